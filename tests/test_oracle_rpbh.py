"""Pins for the oracle's generator and RPBH rotation (CPU only).

Each check is fixed by the pages or by mathematics, not by the oracle itself:
orthogonality ("Pi_d orthogonal", OrbitQuant "Offline Weight Quantization"),
the Sylvester recursion and an independent butterfly for H_h (the O(d log h)
FWHT of the RPBH section), norm preservation, and the one-hot closed form.
"""

import numpy as np
import pytest

from oracle import rpbh
from oracle.splitmix64 import SplitMix64


def test_splitmix64_known_answer():
    # Reference sequence of SplitMix64 (Steele, Lea & Flood 2014) for seed 1234567,
    # as published with the generator's reference implementation.
    g = SplitMix64(1234567)
    assert [g.next() for _ in range(5)] == [
        6457827717110365317, 3203168211198807973, 9817491932198370423,
        4593380528125082431, 16408922859458223821]


@pytest.mark.parametrize("d", [1, 2, 7, 64, 256, 1536])
def test_permutation_is_bijection_and_signs_are_rademacher(d):
    perm, signs = rpbh.draw_permutation_and_signs(0, d)
    assert sorted(perm.tolist()) == list(range(d))
    assert set(np.unique(signs).tolist()) <= {-1.0, 1.0}


def test_permutation_is_not_trivial_and_depends_on_seed():
    p0, s0 = rpbh.draw_permutation_and_signs(0, 1024)
    p1, s1 = rpbh.draw_permutation_and_signs(1, 1024)
    assert not np.array_equal(p0, np.arange(1024))
    assert not np.array_equal(p0, p1)
    # Rademacher: about half the signs negative (binomial, 6 sigma)
    assert abs(np.sum(s0 < 0) - 512) < 6 * 16


def test_default_block_rule():
    # largest power of two dividing d
    assert rpbh.default_block(3072) == 1024
    assert rpbh.default_block(1536) == 512
    assert rpbh.default_block(8960) == 256
    assert rpbh.default_block(12288) == 4096
    assert rpbh.default_block(256) == 256
    assert rpbh.default_block(6) == 2


@pytest.mark.parametrize("h", [1, 2, 4, 8, 32, 128])
def test_hadamard_orthogonal_and_sylvester(h):
    H = rpbh.hadamard(h)
    assert np.allclose(H @ H.T, np.eye(h), atol=1e-14)
    # Sylvester recursion H_{2n} = [[H, H], [H, -H]] (unnormalised), built with kron
    S = np.array([[1.0]])
    while S.shape[0] < h:
        S = np.kron(np.array([[1.0, 1.0], [1.0, -1.0]]), S)
    assert np.array_equal(H * np.sqrt(h), S)


def _fwht_butterfly(v):
    """Independent in-place iterative butterfly (unnormalised)."""
    v = np.array(v, dtype=np.float64)
    n = v.shape[-1]
    s = 1
    while s < n:
        for i in range(0, n, 2 * s):
            a = v[..., i:i + s].copy()
            b = v[..., i + s:i + 2 * s].copy()
            v[..., i:i + s] = a + b
            v[..., i + s:i + 2 * s] = a - b
        s *= 2
    return v


@pytest.mark.parametrize("h", [32, 64, 256])
def test_dense_hadamard_equals_butterfly(h):
    rng = np.random.default_rng(7)
    v = rng.standard_normal((5, h))
    assert np.allclose(v @ rpbh.hadamard(h).T, _fwht_butterfly(v) / np.sqrt(h), atol=1e-12)


@pytest.mark.parametrize("d,h", [(64, 16), (256, 64), (192, 64), (512, 512)])
def test_dense_rpbh_orthogonal_and_rotate_matches(d, h):
    perm, signs = rpbh.draw_permutation_and_signs(3, d)
    Pi = rpbh.rpbh_matrix(perm, signs, h)
    assert np.allclose(Pi @ Pi.T, np.eye(d), atol=1e-12)
    rng = np.random.default_rng(1)
    X = rng.standard_normal((4, d))
    assert np.allclose(rpbh.rotate(X, perm, signs, h), X @ Pi.T, atol=1e-12)


def test_rpbh_structure_from_definition():
    # Pi = blkdiag(H D) P: column pi(j) of Pi equals sign_j * H column (j mod h) in block j//h
    d, h = 128, 32
    perm, signs = rpbh.draw_permutation_and_signs(11, d)
    Pi = rpbh.rpbh_matrix(perm, signs, h)
    H = rpbh.hadamard(h)
    for j in range(d):
        col = Pi[:, perm[j]]
        b = j // h
        expect = np.zeros(d)
        expect[b * h:(b + 1) * h] = signs[j] * H[:, j % h]
        assert np.allclose(col, expect, atol=1e-15)


@pytest.mark.parametrize("kind", ["gauss", "outlier", "onehot", "sparse"])
def test_norm_preservation(kind):
    d, h = 3072, 128
    perm, signs = rpbh.draw_permutation_and_signs(0, d)
    rng = np.random.default_rng(5)
    X = rng.standard_normal((8, d))
    if kind == "outlier":
        X[:, rng.choice(d, 16, replace=False)] *= 50.0
    elif kind == "onehot":
        X = np.zeros((8, d))
        X[np.arange(8), rng.choice(d, 8)] = 3.0
    elif kind == "sparse":
        X = np.zeros((8, d))
        for r in range(8):
            X[r, rng.choice(d, 8, replace=False)] = rng.standard_normal(8)
    U = rpbh.rotate(X, perm, signs, h)
    assert np.allclose(np.linalg.norm(U, axis=1), np.linalg.norm(X, axis=1), rtol=1e-12)


def test_one_hot_closed_form():
    # x = a e_k: the rotated vector is +-a/sqrt(h) on exactly the h coordinates of the
    # block that holds j = pi^-1(k), and 0 elsewhere.
    d, h, a = 1536, 128, 2.5
    perm, signs = rpbh.draw_permutation_and_signs(0, d)
    inv = np.empty(d, dtype=np.int64)
    inv[perm] = np.arange(d)
    for k in (0, 17, 1535):
        x = np.zeros(d)
        x[k] = a
        u = rpbh.rotate(x[None], perm, signs, h)[0]
        b = inv[k] // h
        blk = u[b * h:(b + 1) * h]
        assert np.allclose(np.abs(blk), a / np.sqrt(h), atol=1e-14)
        rest = np.concatenate([u[:b * h], u[(b + 1) * h:]])
        assert np.all(rest == 0.0)


def test_full_block_identity_permutation_is_textbook_wht():
    # h = d, pi = identity, all signs +: Pi = H_d, so Pi e_k is the k-th WHT column
    d = 64
    perm = np.arange(d)
    signs = np.ones(d)
    S = np.array([[1.0]])
    while S.shape[0] < d:
        S = np.kron(np.array([[1.0, 1.0], [1.0, -1.0]]), S)
    for k in (0, 5, 63):
        e = np.zeros(d)
        e[k] = 1.0
        assert np.allclose(rpbh.rotate(e[None], perm, signs, d)[0], S[:, k] / 8.0, atol=1e-15)


# ---- composed rounds ([RHT] Methodology, Key contributions 1 and 3) ----------

def test_composed_round_one_is_the_rpbh_draw_and_later_rounds_differ():
    d = 512
    rounds = rpbh.draw_rounds(7, d, 3)
    p, s = rpbh.draw_permutation_and_signs(7, d)
    assert np.array_equal(rounds[0][0], p) and np.array_equal(rounds[0][1], s)
    for perm, signs in rounds[1:]:
        assert sorted(perm.tolist()) == list(range(d))
        assert set(np.unique(signs).tolist()) <= {-1.0, 1.0}
    assert not np.array_equal(rounds[1][0], rounds[0][0])
    assert not np.array_equal(rounds[2][0], rounds[1][0])
    # the stream continues: round 2 of a 2-round draw is round 2 of a 3-round draw
    two = rpbh.draw_rounds(7, d, 2)
    assert np.array_equal(two[1][0], rounds[1][0]) and np.array_equal(two[1][1], rounds[1][1])


@pytest.mark.parametrize("d,h,k", [(64, 8, 2), (128, 32, 3), (256, 64, 2)])
def test_composed_rotation_is_orthogonal_and_matches_the_dense_product(d, h, k):
    rounds = rpbh.draw_rounds(3, d, k)
    M = rpbh.composed_matrix(rounds, h)
    assert np.allclose(M @ M.T, np.eye(d), atol=1e-12)
    x = np.random.default_rng(1).standard_normal((5, d))
    assert np.allclose(rpbh.rotate_composed(x, rounds, h), x @ M.T, atol=1e-12)
    assert np.allclose(np.linalg.norm(rpbh.rotate_composed(x, rounds, h), axis=1), np.linalg.norm(x, axis=1))


def test_two_rounds_of_a_one_hot_row_lie_on_the_1_over_h_lattice():
    # Closed form: round 1 turns e_i into h entries of +-1/sqrt(h) (one block);
    # round 2 scatters them, and block b, receiving n_b of them, becomes
    # H_h times n_b entries of +-1/sqrt(h): every entry is k/h with |k| <= n_b
    # and k = n_b (mod 2), and the n_b add up to h.
    d, h = 1024, 32
    rounds = rpbh.draw_rounds(11, d, 2)
    x = np.zeros(d)
    x[123] = 1.0
    u1 = rpbh.rotate(x, *rounds[0], h)
    assert np.count_nonzero(np.abs(u1) > 1e-12) == h
    assert np.allclose(np.abs(u1[np.abs(u1) > 1e-12]), 1.0 / np.sqrt(h))
    moved = u1[rounds[1][0]]                     # round 2's gather
    n_b = (np.abs(moved) > 1e-12).reshape(d // h, h).sum(axis=1)
    assert n_b.sum() == h
    u2 = rpbh.rotate_composed(x, rounds, h)
    k = np.rint(u2 * h).reshape(d // h, h)
    assert np.allclose(u2.reshape(d // h, h) * h, k, atol=1e-9)
    assert np.all(np.abs(k) <= n_b[:, None])
    assert np.all((k - n_b[:, None]) % 2 == 0)


def test_two_and_three_rounds_bring_sparse_rows_to_the_lloyd_max_distortion(codebooks):
    # [RHT] Key contribution 1: after two rounds every coordinate of any input
    # is close to Gaussian, so the Lloyd-Max codebook's distortion d * D(d, b)
    # holds for one-hot and k-sparse rows too; a single block round leaves a
    # one-hot row inside one block and its error many times larger.
    from oracle import quantize as oqz
    d, h, b = 3072, 128, 4
    book = codebooks(d, b)
    c, theory = book["centroids"], d * book["distortion"]
    rng = np.random.default_rng(5)
    M = 48
    onehot = np.zeros((M, d))
    onehot[np.arange(M), rng.integers(0, d, M)] = rng.choice([-1.0, 1.0], M)
    sparse = np.zeros((M, d))
    for i in range(M):
        sparse[i, rng.choice(d, 8, replace=False)] = rng.standard_normal(8)

    def ratio(X, k):
        codes, _, T = oqz.quantize_rows_composed(X, rpbh.draw_rounds(0, d, k), h, c)
        return np.sum((T - c[codes]) ** 2, axis=1).mean() / theory

    assert ratio(onehot, 1) > 10.0 and ratio(sparse, 1) > 2.5
    for k in (2, 3):
        assert 0.6 < ratio(onehot, k) < 1.3
        assert 0.8 < ratio(sparse, k) < 1.25
