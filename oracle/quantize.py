"""Online activation / offline weight quantization and code packing (oracle, fp64).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

[OQ] Methodology, "Online Activation Quantization", for each row x:
  1. x' = Pi_d x                      (rpbh.rotate)
  2. s = ||x'||_2,  x~' = x' / (s + eps)
  3. codes = q_hat(x~') coordinate-wise, x^' = s * C[codes]
[OQ] Methodology, "Offline Weight Quantization", for each row w of W:
  1. w' = Pi_d w   (W' = W Pi_d^T)
  2. r' = ||w'||_2,  w~' = w' / r'
  3. codes = q_hat(w~'), W^' = diag(r') C[codes]
  4. r' stored in BF16.
q_hat(t) = argmin_{c in C} |t - c|  ([OQ] eq. q_hat; [TQ] slide 16).

Readings of what the pages leave open:
* eps = 1e-12, and the same eps on the weight side (a zero row then gives
  codes of t = 0 and norm 0 instead of 0/0).
* argmin ties go to the lower index (numpy.argmin returns the first index).
* r' is rounded from fp64 to bf16 with round-to-nearest-even; the direction is
  divided by the unrounded r'.
* Packing: the codes of one row form a little-endian bit stream, code i
  occupying bits [i*b, (i+1)*b); rows are padded to whole bytes.  For 4 bits
  this puts element 2j in the low nibble of byte j; for 6 bits, four codes
  share three bytes.
"""

import numpy as np

from .rpbh import rotate, rotate_composed

EPS = 1e-12


def nearest_centroid(T: np.ndarray, centroids: np.ndarray, chunk: int = 1 << 22) -> np.ndarray:
    """Brute-force argmin_k |t - c_k| over every centroid, elementwise."""
    T = np.asarray(T, dtype=np.float64)
    flat = T.reshape(-1)
    out = np.empty(flat.shape, dtype=np.int64)
    c = np.asarray(centroids, dtype=np.float64)
    step = max(1, chunk // len(c))
    for i in range(0, flat.size, step):
        blk = flat[i:i + step]
        out[i:i + step] = np.argmin(np.abs(blk[:, None] - c[None, :]), axis=1)
    return out.reshape(T.shape)


def quantize_rows(X, perm, signs, h, centroids, eps: float = EPS):
    """Rows -> (codes int64[M, d], norms float64[M], t float64[M, d]).

    ``t`` is the normalised rotated row (x~'), returned so that tests can find
    entries that lie near a decision boundary.
    """
    return _quantize_rotated(rotate(X, perm, signs, h), centroids, eps)


def _quantize_rotated(U, centroids, eps):
    s = np.sqrt(np.sum(U * U, axis=-1))
    T = U / (s[..., None] + eps)
    codes = nearest_centroid(T, centroids)
    return codes, s, T


def quantize_rows_composed(X, rounds, h, centroids, eps: float = EPS):
    """quantize_rows with the composed rotation Pi_k ... Pi_1 (rpbh.rotate_composed)."""
    return _quantize_rotated(rotate_composed(X, rounds, h), centroids, eps)


def bf16_round(v) -> np.ndarray:
    """Round fp64 values to the nearest bf16 (8 significant bits), ties to even.

    Returned as float64 holding the bf16 value.  Finite normal inputs only
    (norms of real rows); zero maps to zero.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros_like(v)
    nz = v != 0
    m, e = np.frexp(v[nz])            # v = m * 2^e, 0.5 <= |m| < 1
    scaled = m * 256.0                # 8 significant bits -> integer part
    out[nz] = np.ldexp(np.rint(scaled), e - 8)   # rint: round half to even
    return out


def bf16_bits(v) -> np.ndarray:
    """uint16 bit patterns of values that are exactly representable in bf16."""
    f32 = np.asarray(v, dtype=np.float64).astype(np.float32)
    return (f32.view(np.uint32) >> 16).astype(np.uint16)


def quantize_weight_rows(W, perm, signs, h, centroids, eps: float = EPS):
    """Weight rows -> (codes, r_bf16 as float64, r fp64 unrounded, t)."""
    return _quantize_weight_rotated(rotate(W, perm, signs, h), centroids, eps)


def _quantize_weight_rotated(U, centroids, eps):
    r = np.sqrt(np.sum(U * U, axis=-1))
    T = U / (r[..., None] + eps)
    codes = nearest_centroid(T, centroids)
    return codes, bf16_round(r), r, T


def quantize_weight_rows_composed(W, rounds, h, centroids, eps: float = EPS):
    """quantize_weight_rows with the composed rotation (rpbh.rotate_composed)."""
    return _quantize_weight_rotated(rotate_composed(W, rounds, h), centroids, eps)


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Little-endian bit stream per row: uint8[M, ceil(d*bits/8)]."""
    codes = np.asarray(codes, dtype=np.int64)
    if codes.ndim == 1:
        codes = codes[None, :]
    if np.any(codes < 0) or np.any(codes >= (1 << bits)):
        raise ValueError("code out of range")
    M, d = codes.shape
    bitplanes = (codes[:, :, None] >> np.arange(bits)) & 1      # [M, d, bits], LSB first
    stream = bitplanes.reshape(M, d * bits).astype(np.uint8)
    return np.packbits(stream, axis=1, bitorder="little")


def unpack_codes(packed: np.ndarray, bits: int, d: int) -> np.ndarray:
    """Inverse of pack_codes."""
    packed = np.asarray(packed, dtype=np.uint8)
    if packed.ndim == 1:
        packed = packed[None, :]
    stream = np.unpackbits(packed, axis=1, bitorder="little")[:, : d * bits]
    planes = stream.reshape(packed.shape[0], d, bits).astype(np.int64)
    return np.sum(planes << np.arange(bits), axis=2)


def boundary_distance(T: np.ndarray, boundaries: np.ndarray) -> np.ndarray:
    """min_k |t - beta_k| for every entry (to find near-ties)."""
    T = np.asarray(T, dtype=np.float64)
    b = np.sort(np.asarray(boundaries, dtype=np.float64))
    idx = np.searchsorted(b, T)
    lo = b[np.clip(idx - 1, 0, len(b) - 1)]
    hi = b[np.clip(idx, 0, len(b) - 1)]
    return np.minimum(np.abs(T - lo), np.abs(T - hi))
