"""C-ABI library on the CPU: it loads, exports every declared symbol, and its
host planning (RPBH draw, Lloyd-Max codebook, fp16 table, argument checks)
agrees with the oracle.  No kernel is launched here."""

import ctypes
import math
import os
import re

import numpy as np
import pytest

from oracle import codebook as ocb
from oracle import rpbh as orpbh

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def oq():
    from calibration_free_rotated_b200 import build
    build.build()
    from calibration_free_rotated_b200 import orbitquant
    return orbitquant


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "orbitquant.h")).read()
    return sorted(set(re.findall(r"OQ_API\s+[\w\s\*]+?\b(oq_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(oq):
    names = _declared_symbols()
    assert len(names) >= 16
    lib = oq.lib()
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_empty_error(oq):
    assert oq.lib().oq_version() >= 100


@pytest.mark.parametrize("seed,d,block", [(0, 256, 64), (0, 3072, 128), (7, 1536, 0), (123, 96, 32), (0, 8960, 128)])
def test_rpbh_draw_matches_oracle(oq, seed, d, block):
    r = oq.Rpbh(seed, d, block)
    perm, signs = r.export()
    operm, osigns = orpbh.draw_permutation_and_signs(seed, d)
    assert np.array_equal(perm.astype(np.int64), operm)
    bits = np.array([(signs[j >> 5] >> (j & 31)) & 1 for j in range(d)])
    assert np.array_equal(bits == 1, osigns < 0)
    assert r.block == (block or orpbh.default_block(d))


@pytest.mark.parametrize("d,bits", [(3, 2), (64, 4), (256, 4), (3072, 4), (3072, 2), (3072, 6), (8960, 4),
                                    (1536, 6), (12288, 4), (12288, 2)])
def test_codebook_matches_oracle(oq, codebooks, d, bits):
    lib_cb = oq.Codebook(d, bits).export()
    ref = codebooks(d, bits)
    sd = math.sqrt(d)
    assert np.max(np.abs(lib_cb["centroids"] - ref["centroids"])) * sd < 1e-10
    assert np.max(np.abs(lib_cb["boundaries"] - ref["boundaries"])) * sd < 1e-10
    assert np.array_equal(lib_cb["centroids"], -lib_cb["centroids"][::-1])
    assert abs(lib_cb["distortion"] / ref["distortion"] - 1) < 1e-9
    # the declared fp16 table, bit for bit
    lut = ocb.fp16_lut(ref["centroids"], d).view(np.uint16)
    assert np.array_equal(lib_cb["lut_fp16"], lut)


def test_argument_errors_without_gpu(oq):
    lib = oq.lib()
    h = ctypes.c_void_p()
    assert lib.oq_make_rpbh(0, 0, 0, ctypes.byref(h)) == oq.OQ_ERR_ARG
    assert lib.oq_make_rpbh(0, 96, 64, ctypes.byref(h)) == oq.OQ_ERR_ARG       # 64 does not divide 96
    assert b"power of two" in lib.oq_last_error()
    assert lib.oq_build_codebook(2, 4, ctypes.byref(h)) == oq.OQ_ERR_ARG
    assert lib.oq_build_codebook(64, 9, ctypes.byref(h)) == oq.OQ_ERR_ARG
    r = oq.Rpbh(0, 256, 64)
    cb = oq.Codebook(256, 4)
    cb8 = oq.Codebook(256, 8)
    cb_other = oq.Codebook(512, 4)
    # mismatched d, too many bits, NULL buffers: rejected before any launch
    assert lib.oq_quantize_act(r.handle, cb_other.handle, None, 4, None, None, None) == oq.OQ_ERR_ARG
    assert lib.oq_quantize_act(r.handle, cb8.handle, None, 4, None, None, None) == oq.OQ_ERR_UNSUPPORTED
    assert lib.oq_quantize_act(r.handle, cb.handle, None, 4, None, None, None) == oq.OQ_ERR_ARG
    assert lib.oq_quantize_act(r.handle, cb.handle, None, 0, None, None, None) == oq.OQ_OK  # M == 0: nothing
    # a codebook for the block (C^(64,4) on rows of width 256) passes the dimension check; others do not
    cb_blk = oq.Codebook(64, 4)
    cb128 = oq.Codebook(128, 4)
    assert lib.oq_quantize_act(r.handle, cb_blk.handle, None, 0, None, None, None) == oq.OQ_OK
    assert lib.oq_quantize_act(r.handle, cb128.handle, None, 0, None, None, None) == oq.OQ_ERR_ARG
    assert b"neither" in lib.oq_last_error()
    assert lib.oq_quantize_act(r.handle, cb_other.handle, None, 0, None, None, None) == oq.OQ_ERR_ARG
    assert lib.oq_quantize_act(r.handle, cb.handle, ctypes.c_void_p(8), 4, ctypes.c_void_p(16),
                               ctypes.c_void_p(16), None) == oq.OQ_ERR_ALIGN
    r_small = oq.Rpbh(0, 48, 16)
    cb48 = oq.Codebook(48, 4)
    assert lib.oq_quantize_act(r_small.handle, cb48.handle, None, 4, None, None, None) == oq.OQ_ERR_UNSUPPORTED
    # GEMM constraints
    cb2 = oq.Codebook(256, 2)
    cb3 = oq.Codebook(256, 3)
    args = (None, None, 4, None, None, 32, None, 0, ctypes.c_void_p(16), None, None)
    assert lib.oq_linear_codes(256, cb.handle, cb3.handle, *args) == oq.OQ_ERR_UNSUPPORTED
    assert lib.oq_linear_codes(256, cb.handle, cb2.handle, None, None, 4, None, None, 30, None, 0,
                               ctypes.c_void_p(16), None, None) == oq.OQ_ERR_UNSUPPORTED   # N % 16
    assert lib.oq_linear_codes(256, cb.handle, cb2.handle, None, None, 4, None, None, 32, None, 7,
                               ctypes.c_void_p(16), None, None) == oq.OQ_ERR_ARG           # epilogue
    assert lib.oq_linear_codes(256, cb.handle, cb2.handle, None, None, 4, None, None, 32, None, 0,
                               None, None, None) == oq.OQ_ERR_ARG                          # no output
    assert lib.oq_linear_codes(256, cb.handle, cb2.handle, None, None, 0, None, None, 32, None, 0,
                               None, None, None) == oq.OQ_OK                               # M == 0
    # codebook dimensions: equal, and dividing d
    assert lib.oq_linear_codes(256, cb_blk.handle, cb_blk.handle, None, None, 0, None, None, 32, None, 0,
                               None, None, None) == oq.OQ_OK
    assert lib.oq_linear_codes(256, cb_blk.handle, cb.handle, None, None, 0, None, None, 32, None, 0,
                               None, None, None) == oq.OQ_ERR_ARG
    assert lib.oq_linear_codes(256, cb_other.handle, cb_other.handle, None, None, 0, None, None, 32, None, 0,
                               None, None, None) == oq.OQ_ERR_ARG
    assert b"divide" in lib.oq_last_error()


def test_workspace_bytes(oq):
    assert oq.workspace_bytes(4608, 3072, 4) == 4608 * 3072 // 2 + 4 * 4608
    assert oq.workspace_bytes(3, 64, 6) == 256 + 12
    assert oq.workspace_bytes(0, 64, 4) == 0


@pytest.mark.parametrize("seed,d,block", [(0, 3072, 128), (5, 256, 64), (9, 1536, 0)])
def test_rotation_variants_share_the_rpbh_signs(oq, seed, d, block):
    # [OQ] "Rotation Ablation (Table 3)": Block-RHT is RPBH without P (same
    # draws, so the same signs); Full RHT spans d's largest power-of-two block.
    _, rpbh_signs = oq.Rpbh(seed, d, block).export()
    for kind in ("block_rht", "full_rht"):
        r = oq.Rpbh(seed, d, 0 if kind == "full_rht" else block, kind=kind)
        perm, signs = r.export()
        assert r.kind == kind
        assert np.array_equal(perm, np.arange(d, dtype=np.int32))
        assert np.array_equal(signs, rpbh_signs)
        if kind == "full_rht":
            assert r.block == (d & -d) == orpbh.default_block(d)
        else:
            assert r.block == (block or orpbh.default_block(d))


def test_rotation_variant_errors(oq):
    with pytest.raises(oq.OQError):
        oq.Rpbh(0, 3072, 128, kind="full_rht")  # a full RHT of 3072 has block 1024
    h = ctypes.c_void_p()
    assert oq.lib().oq_make_rotation(0, 256, 64, 7, ctypes.byref(h)) == oq.OQ_ERR_ARG
    assert oq.Rpbh(0, 3072, 1024, kind="full_rht").block == 1024


@pytest.mark.parametrize("seed,d,block,rounds", [(0, 256, 64, 2), (3, 3072, 128, 3), (9, 1536, 0, 2)])
def test_composed_rounds_match_the_oracle_draws(oq, seed, d, block, rounds):
    # Composed rotation ([RHT] Methodology): round 1 is the RPBH draw, later
    # rounds continue the same SplitMix64 stream; the library and the oracle
    # implement the generator independently.
    r = oq.Rpbh(seed, d, block, rounds=rounds)
    assert r.rounds == rounds and r.kind == "rpbh"
    ref = orpbh.draw_rounds(seed, d, rounds)
    p1, s1 = oq.Rpbh(seed, d, block).export()
    assert np.array_equal(r.export()[0], p1) and np.array_equal(r.export()[1], s1)
    for k in range(rounds):
        perm, words = r.export_round(k + 1)
        assert np.array_equal(perm, ref[k][0])
        bits = (words[np.arange(d) // 32] >> (np.arange(d) % 32).astype(np.uint32)) & 1
        assert np.array_equal(np.where(bits == 1, -1.0, 1.0), ref[k][1])
    assert oq.Rpbh(seed, d, block).rounds == 1


def test_composed_rotation_errors(oq):
    h = ctypes.c_void_p()
    for bad in (0, 4, -1):
        assert oq.lib().oq_make_composed_rpbh(0, 256, 64, bad, ctypes.byref(h)) == oq.OQ_ERR_ARG
    r = oq.Rpbh(0, 256, 64, rounds=2)
    with pytest.raises(oq.OQError):
        r.export_round(3)
    with pytest.raises(oq.OQError):
        r.export_round(0)
    with pytest.raises(ValueError):
        oq.Rpbh(0, 256, 64, kind="block_rht", rounds=2)
    # widths and blocks the composed kernel cannot run are refused when the
    # handle is made, with the kernel's own limits (one round has no such limit)
    for d, block in ((32768, 128), (65536, 256), (16416, 32), (240, 16), (4096, 16)):
        assert oq.lib().oq_make_composed_rpbh(0, d, block, 2, ctypes.byref(h)) == oq.OQ_ERR_UNSUPPORTED
        assert "d <= 16384" in oq.lib().oq_last_error().decode()
        assert oq.lib().oq_make_composed_rpbh(0, d, block, 1, ctypes.byref(h)) == oq.OQ_OK
        oq.lib().oq_free_rpbh(h)
    assert oq.lib().oq_make_composed_rpbh(0, 16384, 32, 3, ctypes.byref(h)) == oq.OQ_OK
    oq.lib().oq_free_rpbh(h)


def test_gemm_bit_width_checks(oq):
    # W3A3 needs d % 128 == 0 (two 24-byte k-step rows per tensor copy); 3 bits
    # only for both operands; argument errors are found before any launch.
    lib = oq.lib()
    cb3, cb4 = oq.Codebook(320, 3), oq.Codebook(320, 4)
    null = ctypes.c_void_p()
    assert lib.oq_linear_codes(320, cb3.handle, cb3.handle, null, null, 0, null, null, 0, null, 0, null, null,
                               null) == oq.OQ_ERR_UNSUPPORTED
    assert lib.oq_linear_codes(320, cb4.handle, cb3.handle, null, null, 0, null, null, 0, null, 0, null, null,
                               null) == oq.OQ_ERR_UNSUPPORTED
    cb3b, cb4b = oq.Codebook(384, 3), oq.Codebook(384, 4)
    assert lib.oq_linear_codes(384, cb3b.handle, cb3b.handle, null, null, 0, null, null, 0, null, 0, null, null,
                               null) == 0
    assert lib.oq_linear_codes(384, cb4b.handle, cb4b.handle, null, null, 0, null, null, 0, null, 0, null, null,
                               null) == 0


def test_stall_hook_arguments(oq):
    lib = oq.lib()
    assert lib.oq_test_stall_next(3) == oq.OQ_ERR_ARG
    assert lib.oq_test_stall_next(-1) == oq.OQ_ERR_ARG
    assert lib.oq_test_stall_next(2) == oq.OQ_OK
    assert lib.oq_test_stall_next(0) == oq.OQ_OK  # disarmed again


def test_debug_switch(oq):
    lib = oq.lib()
    assert lib.oq_set_debug(1) == oq.OQ_OK
    assert lib.oq_set_debug(0) == oq.OQ_OK


def test_device_allocation_counter_is_exported(oq):
    # no device here, so nothing has been allocated; the counter never fails
    assert oq.device_allocations() == 0


def test_row_flatness_argument_errors(oq):
    # argument errors are found on the host, before any launch (no GPU here)
    lib = oq.lib()
    out = ctypes.c_void_p(16)
    null = ctypes.c_void_p()
    assert lib.oq_row_flatness(ctypes.c_void_p(16), -1, 256, out, out, out, null) == oq.OQ_ERR_ARG
    assert lib.oq_row_flatness(ctypes.c_void_p(16), 4, 252, out, out, out, null) == oq.OQ_ERR_UNSUPPORTED
    assert lib.oq_row_flatness(ctypes.c_void_p(16), 4, 0, out, out, out, null) == oq.OQ_ERR_UNSUPPORTED
    assert lib.oq_row_flatness(null, 4, 256, out, out, out, null) == oq.OQ_ERR_ARG
    assert lib.oq_row_flatness(ctypes.c_void_p(24), 4, 256, out, out, out, null) == oq.OQ_ERR_ALIGN
    assert lib.oq_row_flatness(ctypes.c_void_p(16), 4, 256, null, null, null, null) == oq.OQ_ERR_ARG
    assert lib.oq_row_flatness(ctypes.c_void_p(16), 4, 256, ctypes.c_void_p(18), null, null, null) == oq.OQ_ERR_ALIGN
    assert "d % 8" in lib.oq_last_error().decode() or "aligned" in lib.oq_last_error().decode()
