"""Pins for the oracle's quantizer, packing, bf16 rounding and linear layer (CPU only)."""

import math

import numpy as np
import pytest
import torch

from oracle import linear as olin
from oracle import quantize as oq
from oracle import rpbh


def test_nearest_centroid_equals_boundary_count_away_from_ties(codebooks):
    # argmin |t - c_k| (the definition) equals #{k : t > beta_k} with midpoint boundaries
    cb = codebooks(3072, 4)
    rng = np.random.default_rng(0)
    t = rng.standard_normal(200000) / math.sqrt(3072)
    codes = oq.nearest_centroid(t, cb["centroids"])
    count = np.sum(t[:, None] > cb["boundaries"][None, :], axis=1)
    far = oq.boundary_distance(t, cb["boundaries"]) > 1e-12
    assert np.array_equal(codes[far], count[far])


@pytest.mark.parametrize("bits", [1, 2, 4, 6])
def test_ties_take_lower_centroid(bits, codebooks):
    cb = codebooks(256, bits)
    L = 1 << bits
    # t = 0 sits exactly on the middle boundary of a symmetric codebook
    assert oq.nearest_centroid(np.zeros(3), cb["centroids"]).tolist() == [L // 2 - 1] * 3


def test_zero_row_gives_zero_norm_and_middle_codes(codebooks):
    d, h = 256, 64
    perm, signs = rpbh.draw_permutation_and_signs(0, d)
    cb = codebooks(d, 4)
    codes, s, T = oq.quantize_rows(np.zeros((2, d)), perm, signs, h, cb["centroids"])
    assert np.all(s == 0) and np.all(T == 0)
    assert np.all(codes == 7)


def test_quantized_row_reconstruction_is_scale_invariant(codebooks):
    # codes depend only on the direction: x and 7.5 x give the same codes, norms scale
    d, h = 1536, 128
    perm, signs = rpbh.draw_permutation_and_signs(0, d)
    cb = codebooks(d, 4)
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, d))
    c1, s1, _ = oq.quantize_rows(x, perm, signs, h, cb["centroids"])
    c2, s2, _ = oq.quantize_rows(7.5 * x, perm, signs, h, cb["centroids"])
    assert np.array_equal(c1, c2)
    assert np.allclose(s2, 7.5 * s1, rtol=1e-14)


@pytest.mark.parametrize("d,bits", [(3072, 2), (3072, 4), (1536, 6)])
@pytest.mark.parametrize("kind,tol", [("gauss", 0.03), ("lognormal_channels", 0.15)])
def test_rotated_rows_reach_lloyd_max_distortion(d, bits, kind, tol, codebooks):
    # data-agnostic claim (OrbitQuant "Data-Agnostic Codebook"): after RPBH the
    # per-coordinate error of the normalised row is close to D(d, b).  Rows with
    # log-normal channel scales are not fully Gaussianised by 128-blocks, so
    # their excess is larger (a few percent) -- a property of RPBH itself.
    perm, signs = rpbh.draw_permutation_and_signs(0, d)
    cb = codebooks(d, bits)
    rng = np.random.default_rng(9)
    x = rng.standard_normal((64, d))
    if kind != "gauss":
        x = x * np.exp(rng.standard_normal(d))
    codes, s, T = oq.quantize_rows(x, perm, signs, 128, cb["centroids"])
    mse = np.mean((T - cb["centroids"][codes]) ** 2)
    assert abs(mse / cb["distortion"] - 1) < tol


def test_pack_layout_examples():
    # little-endian bit stream, code i at bits [i*b, (i+1)*b)
    assert oq.pack_codes(np.array([[1, 2, 3, 4]]), 4).tolist() == [[0x21, 0x43]]
    assert oq.pack_codes(np.array([[1, 2, 3, 0]]), 2).tolist() == [[0b00111001]]
    # 6 bits: 1 | 2<<6 | 3<<12 | 4<<18 = 0x103081
    assert oq.pack_codes(np.array([[1, 2, 3, 4]]), 6).tolist() == [[0x81, 0x30, 0x10]]
    assert oq.pack_codes(np.array([[1, 0, 1, 1, 0, 0, 0, 1]]), 1).tolist() == [[0b10001101]]


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6])
def test_pack_roundtrip(bits):
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 1 << bits, size=(5, 96))
    packed = oq.pack_codes(codes, bits)
    assert packed.shape == (5, 96 * bits // 8)
    assert np.array_equal(oq.unpack_codes(packed, bits, 96), codes)


def test_bf16_round_matches_torch_and_ties_to_even():
    rng = np.random.default_rng(2)
    v = np.abs(rng.standard_normal(10000)) * 10.0 ** rng.integers(-3, 4, 10000)
    v32 = v.astype(np.float32).astype(np.float64)           # fp32-representable inputs
    ref = torch.from_numpy(v32.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oq.bf16_round(v32), ref)
    # exact ties: 1 + 2^-8 -> 1 (even), 1 + 3*2^-8 -> 1 + 2^-6 (even)
    assert oq.bf16_round(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8])).tolist() == [1.0, 1 + 2.0 ** -6]


def test_weight_norm_is_bf16(codebooks):
    d, h = 256, 64
    perm, signs = rpbh.draw_permutation_and_signs(0, d)
    rng = np.random.default_rng(4)
    W = rng.standard_normal((16, d)) * 0.02
    codes, r16, r, _ = oq.quantize_weight_rows(W, perm, signs, h, codebooks(d, 4)["centroids"])
    assert np.allclose(r, np.linalg.norm(W, axis=1), rtol=1e-12)
    assert np.all(np.abs(r16 - r) <= r * 2.0 ** -8)
    assert np.array_equal(oq.bf16_round(r16), r16)


def test_rotation_cancels_in_the_product():
    # <Pi w, Pi x> = <w, x> (OrbitQuant "Online Activation Quantization", last line)
    d = 3072
    perm, signs = rpbh.draw_permutation_and_signs(0, d)
    rng = np.random.default_rng(6)
    X = rng.standard_normal((8, d))
    W = rng.standard_normal((5, d))
    Xr = rpbh.rotate(X, perm, signs, 128)
    Wr = rpbh.rotate(W, perm, signs, 128)
    assert np.allclose(Xr @ Wr.T, X @ W.T, rtol=1e-10, atol=1e-10)


def test_linear_equals_product_of_dequantised_rows(codebooks):
    # y = W^' x^' with x^' = s C[codes], W^' = diag(r') C[codes] (steps 3 of both procedures)
    d = 256
    perm, signs = rpbh.draw_permutation_and_signs(0, d)
    cb = codebooks(d, 4)
    rng = np.random.default_rng(8)
    X = rng.standard_normal((6, d))
    W = rng.standard_normal((7, d)) * 0.02
    ca, s, _ = oq.quantize_rows(X, perm, signs, 64, cb["centroids"])
    cw, r16, _, _ = oq.quantize_weight_rows(W, perm, signs, 64, cb["centroids"])
    y = olin.linear_from_codes(ca, s, cw, r16, cb["centroids"], cb["centroids"], d, exact_centroids=True)
    xhat = s[:, None] * cb["centroids"][ca]
    what = r16[:, None] * cb["centroids"][cw]
    for m in range(6):
        for n in range(7):
            assert abs(y[m, n] - float(np.dot(what[n], xhat[m]))) < 1e-12


@pytest.mark.parametrize("bits", [2, 4, 6])
def test_linear_error_matches_codebook_distortion(bits, codebooks):
    # the relative error of y against the unquantised W x is about
    # sqrt(d D_a + d D_w) for Gaussian rows: checks the s and r rescaling
    d = 3072
    perm, signs = rpbh.draw_permutation_and_signs(0, d)
    cb = codebooks(d, bits)
    rng = np.random.default_rng(bits)
    X = rng.standard_normal((32, d))
    W = rng.standard_normal((48, d)) * 0.02
    ca, s, _ = oq.quantize_rows(X, perm, signs, 128, cb["centroids"])
    cw, r16, _, _ = oq.quantize_weight_rows(W, perm, signs, 128, cb["centroids"])
    y = olin.linear_from_codes(ca, s, cw, r16, cb["centroids"], cb["centroids"], d, exact_centroids=True)
    ref = X @ W.T
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    # per-row error of the unit direction is d*D; relative to |<w~, x~>| ~ 1/sqrt(d) it is
    # amplified by sqrt(d): rel ~ sqrt(d * (d D_a + d D_w) / d) = sqrt(2 d D)
    expect = math.sqrt(2 * d * cb["distortion"])
    assert 0.7 * expect < rel < 1.3 * expect


def test_gelu_erf_values():
    # exact-erf GELU: GELU(0) = 0, GELU(x) - GELU(-x) = x, GELU(1) = Phi(1)
    assert olin.gelu_erf(np.array([0.0]))[0] == 0.0
    x = np.linspace(-4, 4, 17)
    assert np.allclose(olin.gelu_erf(x) - olin.gelu_erf(-x), x, atol=1e-15)
    assert abs(olin.gelu_erf(np.array([1.0]))[0] - 0.8413447460685429) < 1e-15


# ---- boundary_distance: decides which code mismatches fall inside the 1e-5 band ----
# The parity rule forgives a code difference only when t lies within 1e-5 of a
# decision boundary beta_k (the midpoints between consecutive centroids that
# define q_hat, OrbitQuant "Theoretical Basis").  These pins fix the distance
# itself: hand-computed values, then brute force against every boundary.

def test_boundary_distance_hand_values():
    b = np.array([-0.5, 0.0, 0.25])
    t = np.array([0.0, -0.5, 0.25,      # exactly on a boundary
                  -1.0, -0.75,          # below the first boundary
                  1.0, 0.5,             # above the last boundary
                  0.125, -0.25,         # midway between two boundaries
                  0.2, -0.1, 0.05])     # nearer one neighbour than the other
    want = [0.0, 0.0, 0.0,
            0.5, 0.25,
            0.75, 0.25,
            0.125, 0.25,
            0.05, 0.1, 0.05]
    got = oq.boundary_distance(t, b)
    assert np.allclose(got, want, rtol=0, atol=1e-15)
    # the boundaries' order must not matter
    assert np.array_equal(oq.boundary_distance(t, b[[2, 0, 1]]), got)
    # shape is kept (a rows x columns matrix of t)
    assert oq.boundary_distance(t.reshape(3, 4), b).shape == (3, 4)


def test_boundary_distance_single_boundary():
    # 1-bit codebook: one boundary at 0, distance is |t|
    t = np.array([-3.0, -1e-7, 0.0, 2e-9, 5.0])
    assert np.array_equal(oq.boundary_distance(t, np.array([0.0])), np.abs(t))


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6])
def test_boundary_distance_equals_brute_force(bits, codebooks):
    d = 256
    beta = codebooks(d, bits)["boundaries"]
    rng = np.random.default_rng(100 + bits)
    # t spread over and beyond the boundaries' range, plus the boundaries
    # themselves and points a hair either side of them
    t = np.concatenate([rng.uniform(-1.0, 1.0, 50000),
                        rng.standard_normal(50000) / math.sqrt(d),
                        beta, np.nextafter(beta, 2.0), np.nextafter(beta, -2.0)])
    brute = np.min(np.abs(t[:, None] - beta[None, :]), axis=1)
    shuffled = beta[rng.permutation(len(beta))]
    assert np.array_equal(oq.boundary_distance(t, beta), brute)
    assert np.array_equal(oq.boundary_distance(t, shuffled), brute)
    assert np.all(oq.boundary_distance(beta, beta) == 0.0)


def test_band_rule_flags_exactly_the_near_ties(codebooks):
    # the parity tests forgive a mismatch where boundary_distance < 1e-5: put
    # points at known offsets from each boundary and check which are flagged
    beta = codebooks(3072, 4)["boundaries"]
    offs = np.array([0.0, 3e-6, -9.9e-6, 1.01e-5, -2e-5, 1e-3])
    t = (beta[:, None] + offs[None, :]).reshape(-1)
    near = oq.boundary_distance(t, beta) < 1e-5
    spacing = np.min(np.diff(beta))
    assert spacing > 2e-3                      # each point's nearest boundary is its own
    assert near.reshape(len(beta), -1).tolist() == [[True, True, True, False, False, False]] * len(beta)
