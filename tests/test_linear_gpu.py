"""Parity of the codebook GEMM (oq_linear_codes) and the full layer
(oq_linear) against the fp64 oracle, through the C ABI.

Rule: ||Y_gpu - Y_oracle||_F / ||Y_oracle||_F <= 2e-3 on the same codes and
norms.  The codes and norms come from the oracle (quantized on the CPU) and
are uploaded; the oracle sums in fp64 on the same declared fp16 dequant
table the kernel multiplies.  For oq_linear the GPU quantizes X itself; its
codes may differ from the oracle's only inside the 1e-5 boundary band, so the
same bound applies.
"""

import math

import numpy as np
import pytest
import torch

from calibration_free_rotated_b200 import inputs
from oracle import linear as olin
from oracle import quantize as oqz
from oracle import rpbh as orpbh

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module")
def oq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from calibration_free_rotated_b200 import build
    build.build()
    from calibration_free_rotated_b200 import orbitquant
    return orbitquant


_cb = {}


def _lib_cb(oq, d, bits):
    if (d, bits) not in _cb:
        _cb[(d, bits)] = oq.Codebook(d, bits)
    return _cb[(d, bits)]


def _dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _dev_bf16(bits_u16):
    return torch.from_numpy(np.ascontiguousarray(bits_u16).view(np.int16)).cuda().view(torch.bfloat16)


def _oracle_weight(codebooks, W_bits, d, h, bits, seed=0):
    perm, signs = orpbh.draw_permutation_and_signs(seed, d)
    cw, r16, _, _ = oqz.quantize_weight_rows(inputs.bf16_bits_to_f64(W_bits), perm, signs, h,
                                             codebooks(d, bits)["centroids"])
    return cw, r16


def _oracle_act(codebooks, X_bits, d, h, bits, seed=0):
    perm, signs = orpbh.draw_permutation_and_signs(seed, d)
    ca, s, _ = oqz.quantize_rows(inputs.bf16_bits_to_f64(X_bits), perm, signs, h, codebooks(d, bits)["centroids"])
    return ca, s


def _rel_fro(y, ref):
    return float(np.linalg.norm(y - ref) / np.linalg.norm(ref))


def _run_codes(oq, codebooks, ca, s, cw, r16, d, ba, bw, bias_bits=None, epilogue="none", want_bf16=False):
    cb_a, cb_w = _lib_cb(oq, d, ba), _lib_cb(oq, d, bw)
    a_codes = _dev_u8(oqz.pack_codes(ca, ba))
    a_norm = torch.from_numpy(s.astype(np.float32)).cuda()
    w_codes = _dev_u8(oqz.pack_codes(cw, bw))
    w_norm = _dev_bf16(oqz.bf16_bits(r16))
    bias = None if bias_bits is None else _dev_bf16(bias_bits)
    y32, y16 = oq.linear_codes(d, cb_a, cb_w, a_codes, a_norm, w_codes, w_norm, bias=bias, epilogue=epilogue,
                               want_bf16=want_bf16)
    torch.cuda.synchronize()
    oq.device_status()
    ref = olin.linear_from_codes(ca, s, cw, r16, codebooks(d, ba)["centroids"], codebooks(d, bw)["centroids"], d,
                                 bias=None if bias_bits is None else inputs.bf16_bits_to_f64(bias_bits),
                                 gelu=(epilogue == "gelu"))
    return y32.cpu().double().numpy(), (None if y16 is None else y16.float().cpu().double().numpy()), ref


def test_single_linear_workload_block_codebook(oq, codebooks):
    # The literal reading of the single-linear workload's codebook: C^(64,4)
    # (the block's dimension) for both operands on K = 256.  The dequant table
    # is lut_fp16 / sqrt(64), so the epilogue divides by 64, not by K.
    d, h, dc = 256, 64, 64
    X = inputs.activations(1, 64, d)
    W = inputs.weights(1, inputs.T_W, 256, d)
    book = codebooks(dc, 4)
    perm, signs = orpbh.draw_permutation_and_signs(0, d)
    ca, s, _ = oqz.quantize_rows(inputs.bf16_bits_to_f64(X), perm, signs, h, book["centroids"])
    cw, r16, _, _ = oqz.quantize_weight_rows(inputs.bf16_bits_to_f64(W), perm, signs, h, book["centroids"])
    cb = oq.Codebook(dc, 4)
    # the GEMM on the oracle's codes
    y32, _ = oq.linear_codes(d, cb, cb, _dev_u8(oqz.pack_codes(ca, 4)), torch.from_numpy(s.astype(np.float32)).cuda(),
                             _dev_u8(oqz.pack_codes(cw, 4)), _dev_bf16(oqz.bf16_bits(r16)))
    torch.cuda.synchronize()
    oq.device_status()
    ref = olin.linear_from_codes(ca, s, cw, r16, book["centroids"], book["centroids"], dc)
    assert _rel_fro(y32.cpu().double().numpy(), ref) <= TOL
    # the whole layer: the GPU quantizes both operands with the same handles
    r = oq.Rpbh(0, d, h)
    wc, wn = oq.quantize_weight(r, cb, _dev_bf16(W))
    y, _ = oq.linear(r, cb, cb, _dev_bf16(X), wc, wn)
    torch.cuda.synchronize()
    oq.device_status()
    assert _rel_fro(y.cpu().double().numpy(), ref) <= TOL


@pytest.mark.parametrize("ba,bw", [(4, 4), (4, 2), (6, 4), (2, 2), (6, 6), (2, 4), (3, 3)])
def test_codes_gemm_small_ragged(oq, codebooks, ba, bw):
    # several tiles in both M and N, M and N tails (M=200, N=272), K = 256
    d, h, M, N = 256, 64, 200, 272
    rng = np.random.default_rng(ba * 10 + bw)
    X = inputs.to_bf16_bits(rng.standard_normal((M, d)))
    W = inputs.to_bf16_bits(rng.standard_normal((N, d)) * 0.02)
    ca, s = _oracle_act(codebooks, X, d, h, ba)
    cw, r16 = _oracle_weight(codebooks, W, d, h, bw)
    y, _, ref = _run_codes(oq, codebooks, ca, s, cw, r16, d, ba, bw)
    assert _rel_fro(y, ref) <= TOL


@pytest.mark.parametrize("M,N,d,ba,bw", [(1, 16, 64, 4, 4), (1, 16, 64, 6, 2), (128, 256, 64, 4, 4),
                                          (129, 16, 128, 4, 4), (257, 272, 192, 2, 4), (3, 48, 256, 3, 3)])
def test_codes_gemm_degenerate_shapes(oq, codebooks, M, N, d, ba, bw):
    # the smallest shapes the GEMM accepts (one row, N = 16, K = 64), the
    # largest single-CTA M (128) and the first CTA-pair M (129, one pair with
    # 127 empty rows), and tails in every dimension
    h = 64
    rng = np.random.default_rng(M * 7 + N)
    X = inputs.to_bf16_bits(rng.standard_normal((M, d)))
    W = inputs.to_bf16_bits(rng.standard_normal((N, d)) * 0.02)
    ca, s = _oracle_act(codebooks, X, d, h, ba)
    cw, r16 = _oracle_weight(codebooks, W, d, h, bw)
    y, _, ref = _run_codes(oq, codebooks, ca, s, cw, r16, d, ba, bw)
    assert y.shape == (M, N)
    assert _rel_fro(y, ref) <= TOL


def test_codes_gemm_single_linear_workload(oq, codebooks):
    # X[64 x 256] (3 outlier channels x20), W[256 x 256]; block 64; W4A4
    d, h = 256, 64
    X = inputs.activations(1, 64, d)
    W = inputs.weights(1, inputs.T_W, 256, d)
    ca, s = _oracle_act(codebooks, X, d, h, 4)
    cw, r16 = _oracle_weight(codebooks, W, d, h, 4)
    y, _, ref = _run_codes(oq, codebooks, ca, s, cw, r16, d, 4, 4)
    assert _rel_fro(y, ref) <= TOL
    # and the elementwise view: every output close in absolute terms
    assert np.max(np.abs(y - ref)) <= 5e-3 * np.max(np.abs(ref))


@pytest.mark.parametrize("epilogue", ["none", "gelu"])
def test_codes_gemm_bias_gelu_and_bf16_output(oq, codebooks, epilogue):
    d, h, M, N = 512, 128, 130, 256 + 48
    rng = np.random.default_rng(5)
    X = inputs.to_bf16_bits(rng.standard_normal((M, d)) * 3)
    W = inputs.to_bf16_bits(rng.standard_normal((N, d)) * 0.05)
    bias = inputs.to_bf16_bits(rng.standard_normal(N) * 0.5)
    ca, s = _oracle_act(codebooks, X, d, h, 4)
    cw, r16 = _oracle_weight(codebooks, W, d, h, 4)
    y, y16, ref = _run_codes(oq, codebooks, ca, s, cw, r16, d, 4, 4, bias_bits=bias, epilogue=epilogue,
                             want_bf16=True)
    assert _rel_fro(y, ref) <= TOL
    # bf16 output is the fp32 output rounded to nearest even
    y_as_bf16 = torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(y16, y_as_bf16)


def test_codes_gemm_long_k(oq, codebooks):
    # K = 12288 (FLUX fc2 input width), 2-bit weights, 4-bit activations
    d, h, M, N = 12288, 128, 150, 272
    rng = np.random.default_rng(11)
    X = inputs.to_bf16_bits(rng.standard_normal((M, d)))
    W = inputs.to_bf16_bits(rng.standard_normal((N, d)) * 0.02)
    ca, s = _oracle_act(codebooks, X, d, h, 4)
    cw, r16 = _oracle_weight(codebooks, W, d, h, 2)
    y, _, ref = _run_codes(oq, codebooks, ca, s, cw, r16, d, 4, 2)
    assert _rel_fro(y, ref) <= TOL


def test_zero_rows_give_bias_only(oq, codebooks):
    d, h, M, N = 256, 64, 8, 32
    rng = np.random.default_rng(2)
    X = np.zeros((M, d))
    X[1] = rng.standard_normal(d)
    W = inputs.to_bf16_bits(rng.standard_normal((N, d)) * 0.02)
    bias = inputs.to_bf16_bits(rng.standard_normal(N))
    ca, s = _oracle_act(codebooks, inputs.to_bf16_bits(X), d, h, 4)
    cw, r16 = _oracle_weight(codebooks, W, d, h, 4)
    y, _, ref = _run_codes(oq, codebooks, ca, s, cw, r16, d, 4, 4, bias_bits=bias)
    assert np.array_equal(y[0], inputs.bf16_bits_to_f64(bias).astype(np.float32).astype(np.float64))
    assert _rel_fro(y, ref) <= TOL


def _full_layer(oq, X_bits, W_bits, d, h, ba, bw, bias_bits=None, epilogue="none", want_bf16=False):
    r = oq.Rpbh(0, d, h)
    cb_a, cb_w = _lib_cb(oq, d, ba), _lib_cb(oq, d, bw)
    W = _dev_bf16(W_bits)
    w_codes, w_norm = oq.quantize_weight(r, cb_w, W)
    X = _dev_bf16(X_bits)
    bias = None if bias_bits is None else _dev_bf16(bias_bits)
    y32, y16 = oq.linear(r, cb_a, cb_w, X, w_codes, w_norm, bias=bias, epilogue=epilogue, want_bf16=want_bf16)
    torch.cuda.synchronize()
    oq.device_status()
    return y32, y16


def test_flux_projection_full_size(oq, codebooks):
    # X[4608 x 3072], fused QKV W[9216 x 3072] + bias, block 128, W4A4.
    # GEMM on oracle codes (all rows), checked on sampled rows; then the full layer.
    M, N, d, h = 4608, 9216, 3072, 128
    X = inputs.activations(2, M, d)
    W = inputs.weights(2, inputs.T_W, N, d)
    bias = inputs.bias(2, N)
    ca, s = _oracle_act(codebooks, X, d, h, 4)
    cw, r16 = _oracle_weight(codebooks, W, d, h, 4)
    rows = np.linspace(0, M - 1, 40).astype(int)
    cb_a, cb_w = _lib_cb(oq, d, 4), _lib_cb(oq, d, 4)
    y32, _ = oq.linear_codes(d, cb_a, cb_w, _dev_u8(oqz.pack_codes(ca, 4)), torch.from_numpy(s.astype(np.float32)).cuda(),
                             _dev_u8(oqz.pack_codes(cw, 4)), _dev_bf16(oqz.bf16_bits(r16)), bias=_dev_bf16(bias))
    torch.cuda.synchronize()
    oq.device_status()
    cents = codebooks(d, 4)["centroids"]
    ref = olin.linear_from_codes(ca[rows], s[rows], cw, r16, cents, cents, d, bias=inputs.bf16_bits_to_f64(bias))
    y = y32.cpu().double().numpy()[rows]
    assert _rel_fro(y, ref) <= TOL
    # full layer: the GPU quantizes X and W itself
    y32, _ = _full_layer(oq, X, W, d, h, 4, 4, bias_bits=bias)
    y = y32.cpu().double().numpy()[rows]
    assert _rel_fro(y, ref) <= TOL
    # the method's own W4A4 error against the unquantized product (not a parity bound):
    # about 0.24 on these outlier-heavy rows, well below the size of the output
    exact = inputs.bf16_bits_to_f64(X[rows]) @ inputs.bf16_bits_to_f64(W).T + inputs.bf16_bits_to_f64(bias)
    assert _rel_fro(y, exact) < 0.5


def test_flux_mlp_pair_w2a4(oq, codebooks):
    # fc1 [12288 x 3072] -> GELU -> fc2 [3072 x 12288], W2A4, block 128; sampled rows.
    M, d1, d2, h = 4608, 3072, 12288, 128
    X = inputs.activations(3, M, d1)
    W1 = inputs.weights(3, inputs.T_W, d2, d1)
    W2 = inputs.weights(3, inputs.T_W2, d1, d2)
    rows = np.linspace(0, M - 1, 16).astype(int)
    y1, h1 = _full_layer(oq, X, W1, d1, h, 4, 2, epilogue="gelu", want_bf16=True)
    ca, s = _oracle_act(codebooks, X[rows], d1, h, 4)
    cw1, r1 = _oracle_weight(codebooks, W1, d1, h, 2)
    ref1 = olin.linear_from_codes(ca, s, cw1, r1, codebooks(d1, 4)["centroids"], codebooks(d1, 2)["centroids"], d1,
                                  gelu=True)
    assert _rel_fro(y1.cpu().double().numpy()[rows], ref1) <= TOL
    # fc2 on the oracle's own bf16 fc1 output (each layer judged on its own inputs)
    h1_oracle = inputs.to_bf16_bits(ref1)
    ca2, s2 = _oracle_act(codebooks, h1_oracle, d2, h, 4)
    cw2, r2 = _oracle_weight(codebooks, W2, d2, h, 2)
    y2, _ = _full_layer(oq, h1_oracle, W2, d2, h, 4, 2)
    ref2 = olin.linear_from_codes(ca2, s2, cw2, r2, codebooks(d2, 4)["centroids"], codebooks(d2, 2)["centroids"], d2)
    assert _rel_fro(y2.cpu().double().numpy(), ref2) <= TOL


def test_wan_ffn_w4a6_sampled(oq, codebooks):
    # X[32760 x 1536] Student-t(3), fc1 W[8960 x 1536] with 6-bit activations: M tail tile
    M, d, N, h = 32760, 1536, 8960, 128
    X = inputs.activations(4, M, d)
    W1 = inputs.weights(4, inputs.T_W, N, d)
    y1, _ = _full_layer(oq, X, W1, d, h, 6, 4, epilogue="gelu")
    rows = np.concatenate([np.linspace(0, M - 1, 20).astype(int), [M - 1]])
    ca, s = _oracle_act(codebooks, X[rows], d, h, 6)
    cw, r16 = _oracle_weight(codebooks, W1, d, h, 4)
    ref = olin.linear_from_codes(ca, s, cw, r16, codebooks(d, 6)["centroids"], codebooks(d, 4)["centroids"], d,
                                 gelu=True)
    assert _rel_fro(y1.cpu().double().numpy()[rows], ref) <= TOL


def test_wan_ffn_fc2_w4a6_chain(oq, codebooks):
    # Wan FFN fc2: input width d = 8960 (fc1's GELU output), 6-bit activations,
    # W2 [1536 x 8960] with 4-bit weights.  fc2's input is the oracle's own
    # bf16 fc1 output on 1201 tokens sampled across all 32760 (each layer is
    # judged on its own inputs; 1201 is ragged against the GEMM's 256-row
    # tiles).  Checks, in order: the GPU's 6-bit activation codes at d = 8960
    # against the oracle's (band rule), the (6,4) GEMM on the oracle's codes
    # at K = 8960, and the full fc2 layer (GPU act-quant -> GEMM).
    M, d1, d2, h = 32760, 1536, 8960, 128
    rows = np.linspace(0, M - 1, 1201).astype(int)
    X = inputs.activations(4, M, d1)[rows]
    W1 = inputs.weights(4, inputs.T_W, d2, d1)
    W2 = inputs.weights(4, inputs.T_W2, d1, d2)
    ca1, s1 = _oracle_act(codebooks, X, d1, h, 6)
    cw1, r1 = _oracle_weight(codebooks, W1, d1, h, 4)
    ref1 = olin.linear_from_codes(ca1, s1, cw1, r1, codebooks(d1, 6)["centroids"], codebooks(d1, 4)["centroids"],
                                  d1, gelu=True)
    h1 = inputs.to_bf16_bits(ref1)
    # act-quant of the fc2 input
    perm, signs = orpbh.draw_permutation_and_signs(0, d2)
    book6 = codebooks(d2, 6)
    ca2, s2, T2 = oqz.quantize_rows(inputs.bf16_bits_to_f64(h1), perm, signs, h, book6["centroids"])
    r = oq.Rpbh(0, d2, h)
    cb6 = _lib_cb(oq, d2, 6)
    got_codes, got_norm = oq.quantize_act(r, cb6, _dev_bf16(h1))
    torch.cuda.synchronize()
    oq.device_status()
    got = oqz.unpack_codes(got_codes.cpu().numpy(), 6, d2)
    near = oqz.boundary_distance(T2, book6["boundaries"]) < 1e-5
    assert not np.any((got != ca2) & ~near)
    assert np.max(np.abs(got_norm.cpu().numpy() - s2) / s2) < 1e-6
    # the (6,4) GEMM at K = 8960 on the oracle's codes
    cw2, r2 = _oracle_weight(codebooks, W2, d2, h, 4)
    y, _, ref2 = _run_codes(oq, codebooks, ca2, s2, cw2, r2, d2, 6, 4)
    assert _rel_fro(y, ref2) <= TOL
    # the whole fc2 layer on the GPU
    y2, _ = _full_layer(oq, h1, W2, d2, h, 6, 4)
    assert _rel_fro(y2.cpu().double().numpy(), ref2) <= TOL


def test_empty_shapes(oq):
    cb = _lib_cb(oq, 256, 4)
    a = torch.empty((0, 128), dtype=torch.uint8, device="cuda")
    w = torch.zeros((32, 128), dtype=torch.uint8, device="cuda")
    y32, _ = oq.linear_codes(256, cb, cb, a, torch.empty(0, device="cuda"), w,
                             torch.ones(32, dtype=torch.bfloat16, device="cuda"))
    assert y32.shape == (0, 32)
    oq.device_status()


def test_gelu_epilogue_matches_exact_erf(oq):
    # The GELU epilogue against the exact erf form, 0.5 y (1 + erf(y / sqrt 2)),
    # evaluated in fp64 on the host on the kernel's own pre-activation output
    # (the same launch without the epilogue): isolates the GELU arithmetic.
    # Random codes and norms scaled so that y spans roughly [-12, 12].
    torch.manual_seed(3)
    M, N, d = 200, 272, 256
    ca, cw = _lib_cb(oq, d, 4), _lib_cb(oq, d, 4)
    a = torch.randint(0, 256, (M, d // 2), dtype=torch.uint8, device="cuda")
    w = torch.randint(0, 256, (N, d // 2), dtype=torch.uint8, device="cuda")
    an = torch.rand(M, device="cuda") * 6.0
    wn = (torch.rand(N, device="cuda") * 6.0).to(torch.bfloat16)
    bias = (torch.randn(N, device="cuda") * 2.0).to(torch.bfloat16)
    pre, _ = oq.linear_codes(d, ca, cw, a, an, w, wn, bias=bias, epilogue="none")
    got, _ = oq.linear_codes(d, ca, cw, a, an, w, wn, bias=bias, epilogue="gelu")
    torch.cuda.synchronize()
    oq.device_status()
    y = pre.double().cpu().numpy()
    assert y.min() < -6.0 and y.max() > 6.0
    ref = np.vectorize(lambda v: 0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))))(y)
    err = np.abs(got.double().cpu().numpy() - ref)
    assert err.max() <= 2e-6 * max(1.0, float(np.abs(y).max()))


@pytest.mark.parametrize("kind,h", [("block_rht", 64), ("full_rht", 0)])
def test_full_layer_with_rotation_variants(oq, codebooks, kind, h):
    # The rotation cancels in the product for every orthogonal rotation ([OQ]
    # "Online Activation Quantization", last paragraph): oq_linear with the
    # Block-RHT / Full RHT handles against the oracle on the same rotation
    # (identity permutation, RPBH signs).
    d, M, N = 256, 96, 160
    r = oq.Rpbh(0, d, h, kind=kind)
    hh = r.block
    X = inputs.activations(1, M, d)
    W = inputs.weights(1, inputs.T_W, N, d)
    cb = _lib_cb(oq, d, 4)
    wc, wn = oq.quantize_weight(r, cb, _dev_bf16(W))
    y, _ = oq.linear(r, cb, cb, _dev_bf16(X), wc, wn)
    torch.cuda.synchronize()
    oq.device_status()
    _, signs = orpbh.draw_permutation_and_signs(0, d)
    perm = np.arange(d)
    c = codebooks(d, 4)["centroids"]
    ca, s, T = oqz.quantize_rows(inputs.bf16_bits_to_f64(X), perm, signs, hh, c)
    cw, r16, _, Tw = oqz.quantize_weight_rows(inputs.bf16_bits_to_f64(W), perm, signs, hh, c)
    # rows/columns whose codes all agree with the oracle (in-band flips aside)
    got_a = oqz.unpack_codes(oq.quantize_act(r, cb, _dev_bf16(X))[0].cpu().numpy(), 4, d)
    got_w = oqz.unpack_codes(wc.cpu().numpy(), 4, d)
    rows, cols = (got_a == ca).all(axis=1), (got_w == cw).all(axis=1)
    assert rows.sum() > M // 2 and cols.sum() > N // 2
    ref = olin.linear_from_codes(ca, s, cw, r16, c, c, d)
    assert _rel_fro(y.double().cpu().numpy()[np.ix_(rows, cols)], ref[np.ix_(rows, cols)]) <= TOL


@pytest.mark.parametrize("ba,bw,epilogue,M,N", [(4, 4, "none", 2048, 2560), (4, 2, "gelu", 1000, 2320),
                                                 (6, 4, "gelu", 777, 1216), (2, 2, "none", 300, 272),
                                                 (3, 3, "gelu", 1500, 2576)])
def test_bf16_only_output(oq, codebooks, ba, bw, epilogue, M, N):
    # bf16-only output (the layer's usual call) takes the epilogue that first
    # evacuates the accumulator (spare TMEM columns + raw staging) and converts
    # afterwards; its result must be the fp32 path's output rounded to bf16,
    # bit for bit, over several tiles per CTA pair and ragged M / N tails.
    d, h = 512, 128
    rng = np.random.default_rng(ba * 100 + bw * 10 + M % 7)
    X = inputs.to_bf16_bits(rng.standard_normal((M, d)))
    W = inputs.to_bf16_bits(rng.standard_normal((N, d)) * 0.02)
    bias = inputs.to_bf16_bits(rng.standard_normal(N) * 0.1)
    ca, s = _oracle_act(codebooks, X, d, h, ba)
    cw, r16 = _oracle_weight(codebooks, W, d, h, bw)
    cb_a, cb_w = _lib_cb(oq, d, ba), _lib_cb(oq, d, bw)
    args = (d, cb_a, cb_w, _dev_u8(oqz.pack_codes(ca, ba)), torch.from_numpy(s.astype(np.float32)).cuda(),
            _dev_u8(oqz.pack_codes(cw, bw)), _dev_bf16(oqz.bf16_bits(r16)))
    y32, _ = oq.linear_codes(*args, bias=_dev_bf16(bias), epilogue=epilogue)
    _, y16 = oq.linear_codes(*args, bias=_dev_bf16(bias), epilogue=epilogue, want_f32=False, want_bf16=True)
    torch.cuda.synchronize()
    oq.device_status()
    assert torch.equal(y16, y32.to(torch.bfloat16))
    rows = np.linspace(0, M - 1, 24).astype(int)
    ref = olin.linear_from_codes(ca[rows], s[rows], cw, r16, codebooks(d, ba)["centroids"],
                                 codebooks(d, bw)["centroids"], d, bias=inputs.bf16_bits_to_f64(bias),
                                 gelu=(epilogue == "gelu"))
    # bf16 output: the rounding adds up to 2^-9 relative per element
    assert _rel_fro(y16.double().cpu().numpy()[rows], ref) <= TOL + 2.0 ** -9


def test_full_layer_with_composed_rotation(oq, codebooks):
    # The composed rotation is orthogonal too, so it cancels in the product:
    # oq_linear with a 2-round handle against the oracle on the same rounds.
    d, h, M, N = 512, 64, 200, 272
    r = oq.Rpbh(0, d, h, rounds=2)
    X = inputs.to_bf16_bits(np.random.default_rng(8).standard_normal((M, d)))
    W = inputs.weights(1, inputs.T_W, N, d)
    cb = _lib_cb(oq, d, 4)
    wc, wn = oq.quantize_weight(r, cb, _dev_bf16(W))
    y, _ = oq.linear(r, cb, cb, _dev_bf16(X), wc, wn)
    torch.cuda.synchronize()
    oq.device_status()
    R = orpbh.draw_rounds(0, d, 2)
    c = codebooks(d, 4)["centroids"]
    ca, s, _ = oqz.quantize_rows_composed(inputs.bf16_bits_to_f64(X), R, h, c)
    cw, r16, _, _ = oqz.quantize_weight_rows_composed(inputs.bf16_bits_to_f64(W), R, h, c)
    got_a = oqz.unpack_codes(oq.quantize_act(r, cb, _dev_bf16(X))[0].cpu().numpy(), 4, d)
    got_w = oqz.unpack_codes(wc.cpu().numpy(), 4, d)
    rows, cols = (got_a == ca).all(axis=1), (got_w == cw).all(axis=1)
    assert rows.sum() > M // 2 and cols.sum() > N // 2
    ref = olin.linear_from_codes(ca, s, cw, r16, c, c, d)
    assert _rel_fro(y.double().cpu().numpy()[np.ix_(rows, cols)], ref[np.ix_(rows, cols)]) <= TOL


def test_w3a3_full_layer(oq, codebooks):
    # W3A3 ([OQ] Experiments, Qualitative Results): 3-bit activation and weight
    # codes, whose k-step rows (24 bytes) travel two k-steps per tensor copy.
    # X[2000 x 3072] FLUX-like activations, W[1536 x 3072], bias; sampled rows.
    M, N, d, h = 2000, 1536, 3072, 128
    X = inputs.activations(2, M, d)
    W = inputs.weights(2, inputs.T_W, N, d)
    bias = inputs.bias(2, N)
    y, y16 = _full_layer(oq, X, W, d, h, 3, 3, bias_bits=bias, want_bf16=True)
    rows = np.linspace(0, M - 1, 24).astype(int)
    ca, s = _oracle_act(codebooks, X[rows], d, h, 3)
    cw, r16 = _oracle_weight(codebooks, W, d, h, 3)
    c = codebooks(d, 3)["centroids"]
    ref = olin.linear_from_codes(ca, s, cw, r16, c, c, d, bias=inputs.bf16_bits_to_f64(bias))
    assert _rel_fro(y.cpu().double().numpy()[rows], ref) <= TOL
    assert torch.equal(y16, y.to(torch.bfloat16))


def test_full_layer_replays_from_a_cuda_graph(oq, codebooks):
    # The full layer captured once in a CUDA graph (outputs, workspace and
    # inputs preallocated; one eager call first so that every device table
    # exists) and replayed on new inputs written into the same buffers: the
    # replay equals eager calls bit for bit.
    d, h, M, N = 3072, 128, 640, 1024
    r, cb = oq.Rpbh(0, d, h), oq.Codebook(d, 4)
    wc, wn = oq.quantize_weight(r, cb, _dev_bf16(inputs.weights(2, inputs.T_W, N, d)))
    bias = _dev_bf16(inputs.bias(2, N))
    X = _dev_bf16(inputs.activations(2, 4608, d, rows=(0, M)))
    y16 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty((oq.workspace_bytes(M, d, 4),), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        oq.linear(r, cb, cb, X, wc, wn, bias=bias, out_bf16=y16, want_f32=False, want_bf16=True, workspace=ws,
                  stream=s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        oq.linear(r, cb, cb, X, wc, wn, bias=bias, out_bf16=y16, want_f32=False, want_bf16=True, workspace=ws,
                  stream=s)
    for rows in ((1000, 1000 + M), (3000, 3000 + M)):
        X.copy_(_dev_bf16(inputs.activations(2, 4608, d, rows=rows)))
        g.replay()
        torch.cuda.synchronize()
        _, ref = oq.linear(r, cb, cb, X, wc, wn, bias=bias, want_f32=False, want_bf16=True)
        torch.cuda.synchronize()
        oq.device_status()
        assert torch.equal(y16, ref)


@pytest.mark.parametrize("wl,M,d1,d2,bw,ba", [(3, 4608, 3072, 12288, 2, 4), (4, 3001, 1536, 8960, 4, 6)])
def test_fc2_permutation_folded_into_fc1(oq, codebooks, wl, M, d1, d2, bw, ba):
    # Partial fc1 -> fc2 fusion by reparametrisation: W1's rows (one per fc1
    # output) taken in the order pi_2 of fc2's rotation, so fc1 emits
    # P_2 GELU(.) directly; GELU and bf16 rounding act elementwise, so this is
    # the unfused fc1 output with its columns permuted.  fc2's act-quant then
    # needs blkdiag(H_h D_2) only: the Block-RHT handle of the same seed, with
    # the same signs and no permutation.  The codes, norms and fc2 output must
    # equal the unfused chain's bit for bit (FLUX MLP at full size, Wan FFN on
    # 3001 tokens); the folded fc2 is also checked against the oracle.
    h = 128
    X = _dev_bf16(inputs.activations(wl, M, d1))
    W1 = _dev_bf16(inputs.weights(wl, inputs.T_W, d2, d1))
    W2b = inputs.weights(wl, inputs.T_W2, d1, d2)
    r1, r2 = oq.Rpbh(0, d1, h), oq.Rpbh(0, d2, h)
    r2b = oq.Rpbh(0, d2, h, kind="block_rht")
    ca1, cw1, ca2, cw2 = _lib_cb(oq, d1, ba), _lib_cb(oq, d1, bw), _lib_cb(oq, d2, ba), _lib_cb(oq, d2, bw)
    perm2 = torch.from_numpy(r2.export()[0].astype(np.int64)).cuda()
    w1c, w1n = oq.quantize_weight(r1, cw1, W1)
    w1fc, w1fn = oq.quantize_weight(r1, cw1, W1[perm2].contiguous())
    w2c, w2n = oq.quantize_weight(r2, cw2, _dev_bf16(W2b))
    _, y1 = oq.linear(r1, ca1, cw1, X, w1c, w1n, epilogue="gelu", want_f32=False, want_bf16=True)
    _, y1f = oq.linear(r1, ca1, cw1, X, w1fc, w1fn, epilogue="gelu", want_f32=False, want_bf16=True)
    c2, n2 = oq.quantize_act(r2, ca2, y1)
    c2f, n2f = oq.quantize_act(r2b, ca2, y1f)
    y2, _ = oq.linear_codes(d2, ca2, cw2, c2, n2, w2c, w2n)
    y2f, _ = oq.linear_codes(d2, ca2, cw2, c2f, n2f, w2c, w2n)
    torch.cuda.synchronize()
    oq.device_status()
    assert torch.equal(y1f, y1[:, perm2])
    assert torch.equal(c2f, c2) and torch.equal(n2f, n2)
    assert torch.equal(y2f, y2)
    # the folded fc2 layer against the oracle on sampled rows; its input is the
    # oracle's own bf16 fc1 output, in the folded column order
    rows = np.linspace(0, M - 1, 8).astype(int)
    Xb = inputs.activations(wl, M, d1)[rows]
    ca, s = _oracle_act(codebooks, Xb, d1, h, ba)
    cw1o, r1o = _oracle_weight(codebooks, inputs.weights(wl, inputs.T_W, d2, d1), d1, h, bw)
    h1 = inputs.to_bf16_bits(olin.linear_from_codes(ca, s, cw1o, r1o, codebooks(d1, ba)["centroids"],
                                                     codebooks(d1, bw)["centroids"], d1, gelu=True))
    p2 = perm2.cpu().numpy()
    h1f = h1[:, p2]                                  # what the folded fc1 emits for these rows
    c2o, s2o = _oracle_act(codebooks, h1, d2, h, ba)  # the oracle's fc2 input codes (unfolded, RPBH)
    cw2o, r2o = _oracle_weight(codebooks, W2b, d2, h, bw)
    ref = olin.linear_from_codes(c2o, s2o, cw2o, r2o, codebooks(d2, ba)["centroids"], codebooks(d2, bw)["centroids"],
                                 d2)
    gc, gn = oq.quantize_act(r2b, ca2, _dev_bf16(h1f))
    got, _ = oq.linear_codes(d2, ca2, cw2, gc, gn, w2c, w2n)
    torch.cuda.synchronize()
    assert _rel_fro(got.cpu().double().numpy(), ref) <= TOL
