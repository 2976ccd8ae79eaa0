"""Parity of the rotate+quantize kernel (oq_quantize_act / oq_quantize_weight)
against the fp64 oracle, through the C ABI.

Rule (stated with the workload): codes are bit-exact except entries whose
normalised rotated value t lies within 1e-5 of a decision boundary; those are
counted and reported, and every mismatch must lie inside that band.  The
oracle decides in fp64, the kernel in fp32, so the only disagreements are
decisions within fp32 rounding of a boundary.  Norms: rel 1e-6 (fp32
activations); bf16 weight norms exact or one bf16 ulp.
"""

import math

import numpy as np
import pytest
import torch

from calibration_free_rotated_b200 import inputs
from oracle import quantize as oqz
from oracle import rpbh as orpbh

pytestmark = pytest.mark.gpu

BAND = 1e-5


@pytest.fixture(scope="module")
def oq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from calibration_free_rotated_b200 import build
    build.build()
    from calibration_free_rotated_b200 import orbitquant
    return orbitquant


_handles = {}


def _lib_handles(oq, seed, d, h, bits, kind="rpbh", rounds=1, cb_d=None):
    key = (seed, d, h, bits, kind, rounds, cb_d)
    if key not in _handles:
        _handles[key] = (oq.Rpbh(seed, d, h, kind=kind, rounds=rounds), oq.Codebook(cb_d or d, bits))
    return _handles[key]


def _to_dev(bits_u16):
    return torch.from_numpy(np.ascontiguousarray(bits_u16).view(np.int16)).cuda().view(torch.bfloat16)


def _check_rows(oq, codebooks, X_bits, d, h, bits, seed=0, weight=False, rows=None, report=None, kind="rpbh",
                rounds=1, cb_d=None):
    """Runs the kernel on all of X_bits; checks rows `rows` (default all) against the oracle.
    cb_d: the codebook's dimension when it is not the row width d."""
    r, cb = _lib_handles(oq, seed, d, h, bits, kind, rounds, cb_d)
    X = _to_dev(X_bits)
    if weight:
        codes, norms = oq.quantize_weight(r, cb, X)
    else:
        codes, norms = oq.quantize_act(r, cb, X)
    torch.cuda.synchronize()
    oq.device_status()
    rows = np.arange(X_bits.shape[0]) if rows is None else np.asarray(rows)
    codes_np = codes.cpu().numpy()[rows]
    if weight:
        norms_np = norms.cpu().view(torch.int16).numpy().view(np.uint16)[rows]
    else:
        norms_np = norms.cpu().numpy()[rows]
    perm, signs = orpbh.draw_permutation_and_signs(seed, d)
    if kind != "rpbh":  # Block-RHT / Full RHT: the same signs, no permutation
        perm = np.arange(d)
    ref = codebooks(cb_d or d, bits)
    xs = inputs.bf16_bits_to_f64(X_bits[rows])
    if rounds > 1:
        R = orpbh.draw_rounds(seed, d, rounds)
        if weight:
            ref_codes, r16, r_exact, T = oqz.quantize_weight_rows_composed(xs, R, h, ref["centroids"])
        else:
            ref_codes, s, T = oqz.quantize_rows_composed(xs, R, h, ref["centroids"])
    elif weight:
        ref_codes, r16, r_exact, T = oqz.quantize_weight_rows(xs, perm, signs, h, ref["centroids"])
    else:
        ref_codes, s, T = oqz.quantize_rows(xs, perm, signs, h, ref["centroids"])
    got = oqz.unpack_codes(codes_np, bits, d)
    mismatch = got != ref_codes
    band = oqz.boundary_distance(T, ref["boundaries"]) < BAND
    outside = mismatch & ~band
    assert not np.any(outside), f"{int(outside.sum())} code mismatches outside the 1e-5 band"
    if report is not None:
        report.append((int(mismatch.sum()), int(band.sum()), mismatch.size))
    if weight:
        ref_bits = oqz.bf16_bits(r16)
        diff = np.abs(norms_np.astype(np.int32) - ref_bits.astype(np.int32))
        assert np.all(diff <= 1), "bf16 row norms differ by more than one ulp"
    else:
        rel = np.abs(norms_np - s) / np.maximum(s, 1e-30)
        assert np.all((s == 0) == (norms_np == 0))
        assert np.max(rel) < 1e-6
    return got, mismatch


@pytest.mark.parametrize("bits", [4, 2, 6])
def test_single_linear_workload_act_and_weight(oq, codebooks, bits):
    # X[64 x 256] with 3 outlier channels x20, W[256 x 256]; block 64, seed 0
    X = inputs.activations(1, 64, 256)
    W = inputs.weights(1, inputs.T_W, 256, 256)
    _check_rows(oq, codebooks, X, 256, 64, bits)
    _check_rows(oq, codebooks, W, 256, 64, bits, weight=True)


@pytest.mark.parametrize("bits", [4, 2])
def test_single_linear_workload_block_codebook(oq, codebooks, bits):
    # The single-linear workload's "4-bit codebook for d=64" read literally:
    # C^(64,b), the block's dimension, on the same rows of width 256.  The rows
    # are unit vectors either way, so the codes are well defined; they crowd
    # into the middle cells (the codebook is built for wider coordinates).
    X = inputs.activations(1, 64, 256)
    W = inputs.weights(1, inputs.T_W, 256, 256)
    got, _ = _check_rows(oq, codebooks, X, 256, 64, bits, cb_d=64)
    _check_rows(oq, codebooks, W, 256, 64, bits, weight=True, cb_d=64)
    assert len(np.unique(got)) >= 2


@pytest.mark.parametrize("d,h", [(256, 64), (8960, 128), (1024, 1024), (512, 32), (1536, 512)])
@pytest.mark.parametrize("bits", [2, 4, 6])
def test_sweep_shapes_with_ragged_tail(oq, codebooks, d, h, bits):
    # widths and blocks beyond the sweep grid: several stages and CTAs, M not
    # a multiple of the rows per stage, sparse tail rows
    M = 300 if d >= 8192 else 1000
    X = inputs.sweep_activations(M, d)
    rep = []
    _check_rows(oq, codebooks, X, d, h, bits, report=rep)
    mism, inband, total = rep[0]
    assert mism <= inband


@pytest.mark.parametrize("d", [1536, 3072, 12288])
@pytest.mark.parametrize("h", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 4, 6])
def test_sweep_grid(oq, codebooks, d, h, bits):
    # The rotate+quantize sweep's whole grid of widths, blocks and code widths
    # (every kernel configuration the sweep launches), each on M = 999 rows:
    # ragged for every rows-per-stage, N(0,1) rows followed by the one-hot and
    # k-sparse tail and a zero last row.
    M = 999
    X = inputs.sweep_activations(M, d)
    rep = []
    _check_rows(oq, codebooks, X, d, h, bits, report=rep)
    mism, inband, total = rep[0]
    assert total == M * d and mism <= inband


@pytest.mark.parametrize("bits", [1, 3, 5])
def test_odd_bit_widths(oq, codebooks, bits):
    X = inputs.sweep_activations(400, 1536)
    _check_rows(oq, codebooks, X, 1536, 128, bits)


def test_edge_rows(oq, codebooks):
    d, h = 3072, 128
    rng = np.random.default_rng(0)
    x = rng.standard_normal((37, d))
    x[0] = 0.0                                  # zero row
    x[1] = 0.0
    x[1, 5] = -3.0                              # one-hot
    x[2] = 1.0                                  # constant row
    x[3] *= 1e-18                               # tiny (squares still normal in fp32)
    x[4] *= 1e15                                # large (squared norm still finite in fp32)
    x[5, :] = 0.0
    x[5, :2] = [1.0, 1.0]                       # two-hot
    X = inputs.to_bf16_bits(x)
    got, _ = _check_rows(oq, codebooks, X, d, h, 4)
    assert np.all(got[0] == 7)                  # t = 0 takes the lower middle centroid
    _check_rows(oq, codebooks, X[:1], d, h, 4)  # M = 1
    _check_rows(oq, codebooks, X, d, h, 4, weight=True)


@pytest.mark.parametrize("d,h,bits", [(64, 64, 4), (3072, 128, 4), (8960, 128, 6), (16384, 256, 2)])
def test_single_row(oq, codebooks, d, h, bits):
    # M = 1 in each row-width configuration of the kernel (one CTA, half a pair)
    X = inputs.to_bf16_bits(np.random.default_rng(d).standard_normal((1, d)))
    _check_rows(oq, codebooks, X, d, h, bits)
    _check_rows(oq, codebooks, X, d, h, bits, weight=True)


def test_empty_batch(oq):
    r, cb = _lib_handles(oq, 0, 256, 64, 4)
    X = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    codes, norms = oq.quantize_act(r, cb, X)
    assert codes.shape == (0, 128)
    oq.device_status()


def test_deterministic(oq):
    r, cb = _lib_handles(oq, 0, 3072, 128, 4)
    X = _to_dev(inputs.activations(2, 4608, 3072, rows=(0, 777)))
    c1, n1 = oq.quantize_act(r, cb, X)
    c2, n2 = oq.quantize_act(r, cb, X)
    assert torch.equal(c1, c2) and torch.equal(n1, n2)


def test_flux_projection_full_size_sampled(oq, codebooks):
    # X[4608 x 3072] (log-normal channel scales + 16 outlier channels x50), h = 128,
    # all rows quantized in one launch, sampled rows checked
    M, d = 4608, 3072
    X = inputs.activations(2, M, d)
    rows = np.linspace(0, M - 1, 48).astype(int)
    _check_rows(oq, codebooks, X, d, 128, 4, rows=rows)
    W = inputs.weights(2, inputs.T_W, 9216, d)
    _check_rows(oq, codebooks, W, d, 128, 4, weight=True, rows=np.linspace(0, 9215, 32).astype(int))


def test_wan_ffn_full_size_sampled(oq, codebooks):
    # X[32760 x 1536] Student-t(3), 6-bit activations; fc2 input width 8960
    M, d = 32760, 1536
    X = inputs.activations(4, M, d)
    rows = np.concatenate([np.linspace(0, M - 1, 40).astype(int), [M - 1]])
    _check_rows(oq, codebooks, X, d, 128, 6, rows=rows)
    W2 = inputs.weights(4, inputs.T_W2, 1536, 8960)
    _check_rows(oq, codebooks, W2, 8960, 128, 4, weight=True, rows=np.linspace(0, 1535, 24).astype(int))


def test_sweep_largest_full_size_sampled(oq, codebooks):
    # 65536 x 12288 bf16 (1.6 GB), the largest sweep point; sparse tail included
    M, d = 65536, 12288
    X = inputs.sweep_activations(M, d)
    rows = np.concatenate([np.linspace(0, M - 1, 24).astype(int), np.arange(M - 8, M)])
    _check_rows(oq, codebooks, X, d, 256, 2, rows=rows)


@pytest.mark.parametrize("d,h,kind,bits", [(3072, 128, "block_rht", 4), (3072, 1024, "full_rht", 4),
                                           (1024, 1024, "full_rht", 2), (256, 64, "block_rht", 6),
                                           (1536, 128, "block_rht", 3), (8960, 128, "block_rht", 4),
                                           (12288, 128, "block_rht", 2), (16384, 1024, "block_rht", 4)])
def test_rotation_variants(oq, codebooks, d, h, kind, bits):
    # [OQ] "Rotation Ablation (Table 3)": Block-RHT (no permutation) and Full RHT
    # against the oracle with the identity permutation and the RPBH signs;
    # ragged tails, sparse rows and a zero row included
    M = 300 if d >= 8192 else 1000
    X = inputs.sweep_activations(M, d)
    rep = []
    _check_rows(oq, codebooks, X, d, h, bits, kind=kind, report=rep)
    assert rep[0][0] <= rep[0][1]
    if d == 3072:
        W = inputs.weights(2, inputs.T_W, 200, d)
        _check_rows(oq, codebooks, W, d, h, bits, weight=True, kind=kind)


def test_widest_rows_rpbh(oq, codebooks):
    # d = 16384, the widest row the kernels take (one row pair per stage)
    X = inputs.sweep_activations(130, 16384)
    _check_rows(oq, codebooks, X, 16384, 256, 4)


@pytest.mark.parametrize("d,h,bits", [(3072, 128, 4), (1536, 64, 2), (12288, 256, 6), (3072, 128, 6)])
def test_empirical_distortion_matches_lloyd_max(oq, codebooks, d, h, bits):
    # [OQ] "Theoretical Basis": after RPBH each coordinate of a unit row follows
    # f_d, so the per-row squared error of the kernel's codes on N(0,1) rows is
    # d * D(d, b), the Lloyd-Max distortion (a property that holds at any M).
    # The rotated rows come from the oracle; the codes from the kernel.
    M = 2048
    X = inputs.sweep_activations(M, d, seed_offset=1)[: M - M // 8]  # the N(0,1) rows only
    r, cb = _lib_handles(oq, 0, d, h, bits)
    codes, _ = oq.quantize_act(r, cb, _to_dev(X))
    torch.cuda.synchronize()
    got = oqz.unpack_codes(codes.cpu().numpy(), bits, d)
    perm, signs = orpbh.draw_permutation_and_signs(0, d)
    U = orpbh.rotate(inputs.bf16_bits_to_f64(X), perm, signs, h)
    T = U / np.linalg.norm(U, axis=1, keepdims=True)
    book = codebooks(d, bits)
    err = np.sum((T - book["centroids"][got]) ** 2, axis=1).mean()
    theory = d * book["distortion"]
    # N(0,1) rows: the error of a row is a mean over d coordinates; 1792 rows
    # bring the sampling spread well below 1%
    assert abs(err / theory - 1.0) < 0.01, (err, theory)


@pytest.mark.parametrize("d,h,bits,rounds", [(256, 64, 4, 2), (3072, 128, 4, 2), (3072, 128, 2, 3), (1536, 256, 6, 2),
                                              (12288, 128, 4, 2), (16384, 1024, 4, 3), (512, 32, 3, 2),
                                              (8960, 128, 5, 3), (1024, 1024, 1, 2),
                                              # block-transposed transform in every round (blocks of 64..256)
                                              (3072, 64, 3, 2), (3072, 64, 6, 3), (1536, 128, 6, 2),
                                              (2048, 256, 4, 2), (2048, 256, 1, 3), (8960, 256, 2, 2)])
def test_composed_rounds(oq, codebooks, d, h, bits, rounds):
    # [RHT] Methodology: Pi_k ... Pi_1, k RPBH rounds from one SplitMix64
    # stream, against the oracle; ragged M, sparse rows and a zero row included
    M = 301 if d >= 8192 else 999
    X = inputs.sweep_activations(M, d)
    rep = []
    _check_rows(oq, codebooks, X, d, h, bits, rounds=rounds, report=rep)
    assert rep[0][0] <= rep[0][1]
    if d == 3072:
        W = inputs.weights(2, inputs.T_W, 200, d)
        _check_rows(oq, codebooks, W, d, h, bits, weight=True, rounds=rounds)


def test_composed_edge_rows(oq, codebooks):
    d, h = 3072, 128
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, d))
    x[0] = 0.0
    x[1] = 0.0
    x[1, 17] = 2.0
    x[2] *= 1e-18
    x[3] *= 1e15
    X = inputs.to_bf16_bits(x)
    got, _ = _check_rows(oq, codebooks, X, d, h, 4, rounds=2)
    assert np.all(got[0] == 7)
    _check_rows(oq, codebooks, X[:1], d, h, 4, rounds=3)  # M = 1


def test_composed_rounds_bring_one_hot_rows_to_the_lloyd_max_distortion(oq, codebooks):
    # [RHT] Key contribution 1: two rounds make each coordinate of any input
    # near-Gaussian, so the kernel's codes of one-hot and 8-sparse rows reach
    # the Lloyd-Max distortion d * D(d, b); one round leaves them far above it.
    d, h, b = 3072, 128, 4
    rng = np.random.default_rng(2)
    M = 512
    x = np.zeros((M, d))
    x[np.arange(M // 2), rng.integers(0, d, M // 2)] = rng.choice([-1.0, 1.0], M // 2)
    for i in range(M // 2, M):
        x[i, rng.choice(d, 8, replace=False)] = rng.standard_normal(8)
    X = inputs.to_bf16_bits(x)
    book = codebooks(d, b)
    theory = d * book["distortion"]
    ratios = {}
    for k in (1, 2, 3):
        r, cb = _lib_handles(oq, 0, d, h, b, rounds=k)
        codes, _ = oq.quantize_act(r, cb, _to_dev(X))
        torch.cuda.synchronize()
        got = oqz.unpack_codes(codes.cpu().numpy(), b, d)
        U = orpbh.rotate_composed(inputs.bf16_bits_to_f64(X), orpbh.draw_rounds(0, d, k), h)
        T = U / np.linalg.norm(U, axis=1, keepdims=True)
        e = np.sum((T - book["centroids"][got]) ** 2, axis=1)
        ratios[k] = (e[: M // 2].mean() / theory, e[M // 2:].mean() / theory)
    assert ratios[1][0] > 10.0 and ratios[1][1] > 2.5
    for k in (2, 3):
        assert 0.6 < ratios[k][0] < 1.3 and 0.8 < ratios[k][1] < 1.2, ratios
