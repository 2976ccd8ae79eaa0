"""The composed-rotation kernel's host-built tables, on the CPU.

The library chooses, for every round but the last, where each coordinate of
the round's output is stored in shared memory, so that both the store and the
next round's gather of every half-warp fall on 16 different bank pairs (an
edge colouring of the store-group / gather-group multigraph).  This checks the
tables the library builds (oq_test_composed_tables) without a GPU:

- plumbing: emulating the kernel's data flow through the tables -- round 1
  from the interleaved pair words, each later round from the slots the
  previous round stored to, through the kernel's register orders -- gives the
  composed rotation Pi_k ... Pi_1 x of the oracle exactly;
- layout: every round's store slots are distinct, inside the shared array,
  and every half-warp's store and gather of one register cover 16 distinct
  bank pairs.

The register orders are the kernel's: coordinate order (register r of thread
g holds coordinate 32 g + r), or the block-transposed transform's layouts for
blocks of L = h / 32 lanes (gather: 32 (g - l) + 32 ((r / R) ^ l) + R l + r % R;
output: 32 g + R ((r / R) ^ l) + r % R; R = 32 / L, l = g mod L).
"""

import ctypes

import numpy as np
import pytest

from oracle import rpbh as orpbh


@pytest.fixture(scope="module")
def oq():
    from calibration_free_rotated_b200 import build
    build.build()
    from calibration_free_rotated_b200 import orbitquant
    return orbitquant


def _pair_word_slot(c):
    # the interleave's layout of round 1's input: thread c // 32's run of 32
    # words, 16-byte chunk (c // 4) % 8 at position chunk ^ (thread % 8)
    g = c >> 5
    return (g << 5) | ((((c >> 2) & 7) ^ (g & 7)) << 2) | (c & 3)


def _maps(d, h, xch):
    T = d // 32
    g = np.repeat(np.arange(T), 32)
    r = np.tile(np.arange(32), T)
    if not xch:
        return 32 * g + r, 32 * g + r
    L = h // 32
    R = 32 // L
    l = g & (L - 1)
    gather = 32 * (g - l) + 32 * ((r // R) ^ l) + R * l + r % R
    out = 32 * g + R * ((r // R) ^ l) + r % R
    return gather, out


@pytest.mark.parametrize("d,h,rounds,xch", [(3072, 128, 2, 1), (3072, 128, 3, 0), (1536, 64, 2, 1), (1536, 64, 3, 1),
                                            (8960, 256, 2, 1), (8960, 128, 3, 0), (1024, 32, 2, 0),
                                            (16384, 1024, 2, 0), (2048, 256, 3, 1), (512, 512, 2, 0)])
def test_composed_tables_compose_and_avoid_bank_conflicts(oq, d, h, rounds, xch):
    r = oq.Rpbh(0, d, h, rounds=rounds)
    T, words = d // 32, (d + 31) // 32
    threads = (T + 31) // 32 * 32
    gather = np.zeros(rounds * d, np.uint16)
    store = np.zeros(rounds * d, np.uint16)
    signs = np.zeros(rounds * words, np.uint32)
    rc = oq.lib().oq_test_composed_tables(r.handle, xch, gather.ctypes.data, store.ctypes.data, signs.ctypes.data)
    assert rc == oq.OQ_OK, oq.lib().oq_last_error()
    gmap, omap = _maps(d, h, xch)
    lane16 = np.repeat(np.arange(T), 32) >> 4          # half-warp of each (thread, register)
    reg = np.tile(np.arange(32), T)
    group = lane16 * 32 + reg

    # layout: stores injective and inside the shared array; 16 bank pairs per half-warp access
    for k in range(rounds - 1):
        st = store[k * d:(k + 1) * d].astype(np.int64)
        assert len(np.unique(st)) == d and st.max() < 32 * threads
        for slots in (st, gather[(k + 1) * d:(k + 2) * d].astype(np.int64)):
            for grp in np.unique(group):
                banks = slots[group == grp] % 16
                assert len(np.unique(banks)) == len(banks), (k, grp)

    # plumbing: the kernel's data flow through the tables against Pi_k ... Pi_1 x
    rng = np.random.default_rng(d + rounds)
    x = rng.standard_normal(d)
    H = np.array([[1.0]])
    while H.shape[0] < h:
        H = np.block([[H, H], [H, -H]])
    words_sh = np.zeros(32 * threads)            # round 1: bf16 pair words (4-byte slots)
    words_sh[_pair_word_slot(np.arange(d))] = x
    prev = None
    for k in range(rounds):
        src = words_sh if k == 0 else prev
        sbit = (signs[k * words + np.repeat(np.arange(T), 32)] >> reg.astype(np.uint32)) & 1
        vals = np.where(sbit == 1, -1.0, 1.0) * src[gather[k * d:(k + 1) * d].astype(np.int64)]
        z = np.zeros(d)
        z[gmap] = vals                              # register -> its coordinate of the round
        y = (z.reshape(-1, h) @ H.T).reshape(-1)    # unnormalised block transform
        if k + 1 < rounds:
            prev = np.zeros(32 * threads)
            prev[store[k * d:(k + 1) * d].astype(np.int64)] = y[omap]
    ref = orpbh.rotate_composed(x[None, :], orpbh.draw_rounds(0, d, rounds), h)[0] * h ** (rounds / 2)
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-9)


def test_composed_tables_argument_errors(oq):
    buf = np.zeros(8, np.uint32)
    lib = oq.lib()
    one = oq.Rpbh(0, 256, 64)
    assert lib.oq_test_composed_tables(one.handle, 0, buf.ctypes.data, buf.ctypes.data, buf.ctypes.data) == oq.OQ_ERR_ARG
    two = oq.Rpbh(0, 512, 512, rounds=2)
    assert lib.oq_test_composed_tables(two.handle, 1, buf.ctypes.data, buf.ctypes.data,
                                       buf.ctypes.data) == oq.OQ_ERR_UNSUPPORTED
    assert lib.oq_test_composed_tables(two.handle, 0, None, buf.ctypes.data, buf.ctypes.data) == oq.OQ_ERR_ARG
