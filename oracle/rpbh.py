"""RPBH rotation Pi_d by definition (oracle side, fp64).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

[OQ] Methodology, "Randomized Permuted Block-Hadamard (RPBH) Rotation":

    Pi_d = blkdiag(H_h D_1, ..., H_h D_{d/h}) . P_pi

with H_h an h x h Walsh-Hadamard matrix, D_i diagonal Rademacher signs and
P_pi a uniform random permutation drawn once per dimension; h defaults to the
largest power of two dividing d.

Readings of what the page leaves open:

* Hadamard order and scale: Sylvester (natural) order,
  H_h[j, k] = (-1)^popcount(j & k) / sqrt(h), so that Pi_d is orthogonal as
  the "Offline Weight Quantization" step requires.
* Permutation convention: gather, (P x)_j = x_{pi(j)}, i.e. P[j, pi(j)] = 1.
* Signs act before H inside each block (the literal order H_h D_i).
* Generator: SplitMix64(seed); pi by Fisher-Yates (for i = d-1 .. 1:
  j = next() mod (i+1), swap pi[i], pi[j]), then d sign draws
  sign_j = -1 if the top bit of next() is set else +1.

Composed rounds ([RHT] Methodology; "Key contributions" 1 and 3): the
composition R_k of k randomized Hadamard transforms, each a Hadamard matrix
times its own Rademacher diagonal.  Two rounds make every single coordinate
close to Gaussian for any input, three also decorrelate the coordinates.
Reading for a block rotation: each round is a full RPBH round with its own
permutation and signs, Pi^(k) = Pi_k ... Pi_1 (the permutation is what lets a
later round mix coordinates that an earlier round kept inside one block).
Round 1 is the plain RPBH draw of the seed; round r + 1 continues the same
SplitMix64 stream after round r's draws (Fisher-Yates pass, then d signs).

Everything here is dense and slow on purpose: no butterflies, no fusion.
"""

import numpy as np

from .splitmix64 import SplitMix64


def default_block(d: int) -> int:
    """Largest power of two dividing d ([OQ] RPBH section, last sentence of the eq. paragraph)."""
    if d <= 0:
        raise ValueError("d must be positive")
    return d & (-d)


def _draw_round(g: SplitMix64, d: int):
    perm = list(range(d))
    for i in range(d - 1, 0, -1):
        j = g.next() % (i + 1)
        perm[i], perm[j] = perm[j], perm[i]
    signs = [(-1.0 if (g.next() >> 63) else 1.0) for _ in range(d)]
    return np.array(perm, dtype=np.int64), np.array(signs, dtype=np.float64)


def draw_permutation_and_signs(seed: int, d: int):
    """Fisher-Yates permutation then d Rademacher signs from one SplitMix64 stream.

    Returns (perm int64[d], signs float64[d] in {-1, +1}).
    """
    return _draw_round(SplitMix64(seed), d)


def draw_rounds(seed: int, d: int, rounds: int):
    """[(perm, signs)] of rounds 1..k of the composed rotation, all from one
    SplitMix64(seed) stream in order (round 1 = draw_permutation_and_signs)."""
    if rounds < 1:
        raise ValueError("rounds must be >= 1")
    g = SplitMix64(seed)
    return [_draw_round(g, d) for _ in range(rounds)]


def hadamard(h: int) -> np.ndarray:
    """Dense normalised Walsh-Hadamard matrix in Sylvester order, entry by entry."""
    if h <= 0 or (h & (h - 1)) != 0:
        raise ValueError("h must be a power of two")
    H = np.empty((h, h), dtype=np.float64)
    for j in range(h):
        for k in range(h):
            H[j, k] = -1.0 if bin(j & k).count("1") % 2 else 1.0
    return H / np.sqrt(h)


def permutation_matrix(perm: np.ndarray) -> np.ndarray:
    """P with (P x)_j = x_{perm[j]}."""
    d = len(perm)
    P = np.zeros((d, d), dtype=np.float64)
    P[np.arange(d), perm] = 1.0
    return P


def rpbh_matrix(perm: np.ndarray, signs: np.ndarray, h: int) -> np.ndarray:
    """Dense Pi_d = blkdiag(H_h D_1, ..., H_h D_{d/h}) P_pi (small d only)."""
    d = len(perm)
    if d % h != 0:
        raise ValueError("h must divide d")
    H = hadamard(h)
    B = np.zeros((d, d), dtype=np.float64)
    for i in range(d // h):
        sl = slice(i * h, (i + 1) * h)
        B[sl, sl] = H @ np.diag(signs[sl])
    return B @ permutation_matrix(perm)


def rotate(X: np.ndarray, perm: np.ndarray, signs: np.ndarray, h: int) -> np.ndarray:
    """x' = Pi_d x for every row of X ([OQ] "Online Activation Quantization" step 1).

    Applied as X Pi_d^T for a batch of rows.  Per block: gather by perm, multiply
    by the sign diagonal, then by the dense H_h -- the definition, block by block.
    """
    X = np.asarray(X, dtype=np.float64)
    d = X.shape[-1]
    if d % h != 0 or len(perm) != d:
        raise ValueError("shape mismatch")
    H = hadamard(h)
    Y = X[..., perm]                      # (P x)_j = x_{perm[j]}
    Z = Y * signs                         # D_i
    out = np.empty_like(Z)
    for i in range(d // h):
        sl = slice(i * h, (i + 1) * h)
        out[..., sl] = Z[..., sl] @ H.T   # H_h z_i for each row
    return out


def composed_matrix(rounds, h: int) -> np.ndarray:
    """Dense Pi^(k) = Pi_k ... Pi_1 for rounds [(perm_1, signs_1), ...] (small d only)."""
    d = len(rounds[0][0])
    M = np.eye(d)
    for perm, signs in rounds:
        M = rpbh_matrix(perm, signs, h) @ M
    return M


def rotate_composed(X: np.ndarray, rounds, h: int) -> np.ndarray:
    """x' = Pi_k ( ... (Pi_1 x)) for every row of X: round 1 first."""
    U = np.asarray(X, dtype=np.float64)
    for perm, signs in rounds:
        U = rotate(U, perm, signs, h)
    return U
