"""Seeded synthetic workloads (bf16 activations and weights).

This module only draws random numbers and rounds them to bf16; it holds none
of the quantizer's arithmetic.  Both the CUDA path (tests, bench) and the CPU
oracle take their inputs from here, so the two see the same bytes.

Recipe (one place, so every user draws the same data):

* Rows are drawn in chunks of ``CHUNK`` rows; chunk c of tensor ``tid`` for
  workload ``w`` uses ``numpy.random.Generator(PCG64(SeedSequence([1000*w +
  tid, c])))``.  Any row range can therefore be regenerated on its own, which
  lets a test check sampled rows of a full-size tensor.
* Per-channel properties (log-normal scales, outlier channel ids, sparse
  positions) come from tensor id 5 of the same workload.
* Values are drawn in fp64, rounded to fp32, then to bf16 with
  round-to-nearest-even.  ``bf16`` arrays are ``uint16`` bit patterns.

Workloads (shapes of the DiT layers the OrbitQuant pages evaluate on):

1. single linear  X[64 x 256] N(0,1) with 1% of channels (3) x20;
   W[256 x 256] N(0, 0.02^2).
2. FLUX-like attention projection  X[4608 x 3072] = N(0,1) * exp(N(0,1)) per
   channel, 0.5% of channels (16) x50; fused QKV W[9216 x 3072] N(0, 0.02^2);
   bias N(0, 0.02^2).
3. FLUX-like MLP  X as in 2; fc1 W[12288 x 3072], fc2 W[3072 x 12288].
4. Wan-like video FFN  X[32760 x 1536] Student-t(nu=3); W1[8960 x 1536],
   W2[1536 x 8960].
5. rotate+quantize sweep  X[M x d] N(0,1) rows; the last M/8 rows are
   adversarial: one-hot (+-1 at a random position), then k-sparse rows with
   k in {2, 8, 64} N(0,1) values at random positions, and (optionally) one
   all-zero last row.
"""

import numpy as np

CHUNK = 1024

T_X, T_W, T_W2, T_BIAS, T_CHAN = 1, 2, 3, 4, 5


def _rng(workload: int, tid: int, chunk: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([1000 * workload + tid, chunk])))


def to_bf16_bits(x) -> np.ndarray:
    """fp64 -> fp32 -> bf16 (round to nearest even); returns uint16 bit patterns."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f64(b) -> np.ndarray:
    """Exact values of bf16 bit patterns, as fp64."""
    u = (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16)
    return u.view(np.float32).astype(np.float64)


def _rows(workload, tid, rows, d, draw):
    """Rows [r0, r1) of a chunked tensor; draw(rng, n, d) returns fp64 [n, d]."""
    r0, r1 = rows
    out = np.empty((r1 - r0, d), dtype=np.float64)
    c0, c1 = r0 // CHUNK, (r1 - 1) // CHUNK
    for c in range(c0, c1 + 1):
        lo, hi = c * CHUNK, (c + 1) * CHUNK
        blk = draw(_rng(workload, tid, c), CHUNK, d)
        a, b = max(lo, r0), min(hi, r1)
        out[a - r0:b - r0] = blk[a - lo:b - lo]
    return out


def _normal(scale=1.0):
    return lambda g, n, d: g.standard_normal((n, d)) * scale


def _student_t(nu):
    return lambda g, n, d: g.standard_t(nu, size=(n, d))


def _outlier_channels(workload, d, frac):
    k = int(np.ceil(frac * d))
    return np.sort(_rng(workload, T_CHAN).choice(d, size=k, replace=False))


def activations(workload: int, M: int, d: int, rows=None) -> np.ndarray:
    """bf16 bits of activation rows ``rows`` (default all) of workload 1..5."""
    rows = (0, M) if rows is None else rows
    if workload == 1:
        x = _rows(1, T_X, rows, d, _normal())
        x[:, _outlier_channels(1, d, 0.01)] *= 20.0
    elif workload in (2, 3):
        # workloads 2 and 3 share one activation recipe (same FLUX block input)
        g = _rng(2, T_CHAN, 1)
        scale = np.exp(g.standard_normal(d))
        x = _rows(2, T_X, rows, d, _normal()) * scale
        x[:, _outlier_channels(2, d, 0.005)] *= 50.0
    elif workload == 4:
        x = _rows(4, T_X, rows, d, _student_t(3.0))
    else:
        raise ValueError("use sweep_activations for workload 5")
    return to_bf16_bits(x)


def weights(workload: int, tid: int, N: int, d: int, rows=None) -> np.ndarray:
    """bf16 bits of weight rows, N(0, 0.02^2)."""
    rows = (0, N) if rows is None else rows
    return to_bf16_bits(_rows(workload, tid, rows, d, _normal(0.02)))


def bias(workload: int, N: int) -> np.ndarray:
    return to_bf16_bits(_rng(workload, T_BIAS).standard_normal(N) * 0.02)


def sweep_activations(M: int, d: int, rows=None, zero_last_row: bool = True, seed_offset: int = 0) -> np.ndarray:
    """Workload 5: N(0,1) rows with an adversarial sparse tail of M/8 rows."""
    r0, r1 = (0, M) if rows is None else rows
    wl = 5 + 100 * seed_offset
    x = _rows(wl, T_X, (r0, r1), d, _normal())
    n_adv = M // 8
    adv0 = M - n_adv
    kinds = (1, 2, 8, 64)
    per = max(1, n_adv // len(kinds))
    for r in range(max(r0, adv0), r1):
        j = r - adv0
        kind = kinds[min(j // per, len(kinds) - 1)]
        g = _rng(wl, T_CHAN, 1 + r)
        pos = g.choice(d, size=min(kind, d), replace=False)
        row = np.zeros(d)
        if kind == 1:
            row[pos] = 1.0 if g.random() < 0.5 else -1.0
        else:
            row[pos] = g.standard_normal(len(pos))
        x[r - r0] = row
    if zero_last_row and r1 == M and M > 0:
        x[-1] = 0.0
    return to_bf16_bits(x)
