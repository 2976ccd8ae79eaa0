"""Parity of the flatness check (oq_row_flatness) against the oracle, through
the C ABI.

[RHT] "Quantizing With Randomized Hadamard Transforms", Key contribution 4:
rho3 = sum|x|^3 / ||x||^3 and rhoinf = max|x| / ||x|| per row, and their
batch maxima.  Tolerance: the kernel sums fp32 values of rows rescaled
exactly by a power of two; each lane's accumulator takes at most d/64 terms
(256 at d = 16384), so the sums carry a relative error below 256 * 2^-24
(1.5e-5) in the worst case, the warp reduction adds 5 more roundings, and
rho3 raises the square sum to the 3/2: 1e-4 relative bounds every row.
Zero rows must give exactly 0; the batch maxima must equal the largest
per-row outputs bit for bit (the same values, folded with integer max).
"""

import numpy as np
import pytest
import torch

from calibration_free_rotated_b200 import inputs
from oracle import flatness as ofl

pytestmark = pytest.mark.gpu

TOL = 1e-4


@pytest.fixture(scope="module")
def oq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from calibration_free_rotated_b200 import build
    build.build()
    from calibration_free_rotated_b200 import orbitquant
    return orbitquant


def _dev(bits_u16):
    return torch.from_numpy(np.ascontiguousarray(bits_u16).view(np.int16)).cuda().view(torch.bfloat16)


def _check(oq, X_bits):
    r3, ri, bm = oq.row_flatness(_dev(X_bits))
    torch.cuda.synchronize()
    oq.device_status()
    r3, ri, bm = r3.cpu().numpy(), ri.cpu().numpy(), bm.cpu().numpy()
    e3, ei = ofl.flatness(inputs.bf16_bits_to_f64(X_bits))
    zero = e3 == 0
    assert np.all(r3[zero] == 0) and np.all(ri[zero] == 0)
    nz = ~zero
    assert np.max(np.abs(r3[nz] / e3[nz] - 1), initial=0) < TOL
    assert np.max(np.abs(ri[nz] / ei[nz] - 1), initial=0) < TOL
    if len(r3):
        assert bm[0] == r3.max() and bm[1] == ri.max()
    return r3, ri, bm


@pytest.mark.parametrize("d", [256, 1536, 3072, 8960, 12288, 16384])
def test_sweep_rows(oq, d):
    # N(0,1) rows, then one-hot and k-sparse rows (k in 2, 8, 64) and a zero row;
    # M ragged against the warps of a CTA and the persistent grid
    M = 1001 if d <= 3072 else 301
    X = inputs.sweep_activations(M, d)
    r3, ri, bm = _check(oq, X)
    n_adv = M // 8
    assert bm[0] > 0.99 and bm[1] > 0.99            # the one-hot rows
    dense = r3[: M - n_adv]
    assert np.all(dense < 3.0 / np.sqrt(d))          # flat rows: about 1.6 / sqrt(d)


def test_workload_activations_full_size(oq):
    # FLUX-like projection input X[4608 x 3072] (log-normal channel scales,
    # outlier channels), and the single-linear workload's rows
    _check(oq, inputs.activations(2, 4608, 3072))
    _check(oq, inputs.activations(1, 64, 256))
    _check(oq, inputs.activations(4, 2000, 1536))


def test_extreme_scales(oq):
    # exact power-of-two rescaling keeps every finite bf16 row in range: huge
    # maxima (>= 2^127), subnormal maxima, and rows spanning many decades
    d = 1024
    rng = np.random.default_rng(5)
    base = rng.standard_normal((6, d))
    rows = [base[0] * 2.0 ** 120, base[1] * 1e-40, base[2] * np.exp(rng.uniform(-30, 30, d)),
            base[3] * 1e30, np.where(np.arange(d) == 7, 3.0e38, 0.0), np.where(np.arange(d) < 3, 1e-39, 0.0)]
    X = inputs.to_bf16_bits(np.array(rows))
    assert np.all(np.isfinite(inputs.bf16_bits_to_f64(X)))
    r3, ri, _ = _check(oq, X)
    assert abs(r3[4] - 1.0) < TOL and abs(ri[4] - 1.0) < TOL


def test_batch_only_and_empty(oq):
    X = _dev(inputs.sweep_activations(300, 512))
    bm = torch.full((2,), 7.0, device="cuda")
    _, _, bm = oq.row_flatness(X, batch_max=bm, want_rows=False)
    r3, ri, _ = oq.row_flatness(X)
    torch.cuda.synchronize()
    assert bm[0].item() == r3.max().item() and bm[1].item() == ri.max().item()
    E = torch.empty((0, 512), dtype=torch.bfloat16, device="cuda")
    bm = torch.full((2,), 7.0, device="cuda")
    oq.row_flatness(E, batch_max=bm, want_rows=False)
    torch.cuda.synchronize()
    oq.device_status()
    assert bm.tolist() == [0.0, 0.0]
