"""Failure path on the GPU without a fault: a test hook makes the next launch
of a kernel issue none of its copies, so its bounded waits run out; the kernel
must report OQ_ERR_TIMEOUT through the device status word, leave through its
normal teardown, and leave the context usable (the next launch matches the
oracle).  Nothing traps, hangs or faults."""

import numpy as np
import pytest
import torch

from calibration_free_rotated_b200 import inputs
from oracle import linear as olin
from oracle import quantize as oqz
from oracle import rpbh as orpbh

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def oq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from calibration_free_rotated_b200 import build
    build.build()
    from calibration_free_rotated_b200 import orbitquant
    return orbitquant


def _dev_bf16(bits_u16):
    return torch.from_numpy(np.ascontiguousarray(bits_u16).view(np.int16)).cuda().view(torch.bfloat16)


def _expect_timeout(oq):
    torch.cuda.synchronize()
    with pytest.raises(oq.OQError) as e:
        oq.device_status()
    assert e.value.code == oq.OQ_ERR_TIMEOUT
    oq.device_status()  # read and cleared


def test_rotate_quantize_wait_runs_out_and_context_survives(oq, codebooks):
    d, h, M = 3072, 128, 300
    X = inputs.sweep_activations(M, d)
    r, cb = oq.Rpbh(0, d, h), oq.Codebook(d, 4)
    oq.device_status()
    assert oq.lib().oq_test_stall_next(1) == oq.OQ_OK
    oq.quantize_act(r, cb, _dev_bf16(X))
    _expect_timeout(oq)
    codes, norms = oq.quantize_act(r, cb, _dev_bf16(X))
    torch.cuda.synchronize()
    oq.device_status()
    perm, signs = orpbh.draw_permutation_and_signs(0, d)
    book = codebooks(d, 4)
    ref, s, T = oqz.quantize_rows(inputs.bf16_bits_to_f64(X), perm, signs, h, book["centroids"])
    got = oqz.unpack_codes(codes.cpu().numpy(), 4, d)
    assert np.all((got == ref) | (oqz.boundary_distance(T, book["boundaries"]) < 1e-5))


def test_gemm_wait_runs_out_and_context_survives(oq, codebooks):
    # armed for the GEMM: a rotate+quantize launch in between does not consume it
    d, h, M, N = 512, 128, 300, 272
    rng = np.random.default_rng(4)
    X = inputs.to_bf16_bits(rng.standard_normal((M, d)))
    W = inputs.to_bf16_bits(rng.standard_normal((N, d)) * 0.02)
    r, cb = oq.Rpbh(0, d, h), oq.Codebook(d, 4)
    wc, wn = oq.quantize_weight(r, cb, _dev_bf16(W))
    oq.device_status()
    assert oq.lib().oq_test_stall_next(2) == oq.OQ_OK
    ac, an = oq.quantize_act(r, cb, _dev_bf16(X))
    torch.cuda.synchronize()
    oq.device_status()  # kernel 1 ran normally
    oq.linear_codes(d, cb, cb, ac, an, wc, wn)
    _expect_timeout(oq)
    y, _ = oq.linear_codes(d, cb, cb, ac, an, wc, wn)
    torch.cuda.synchronize()
    oq.device_status()
    ca = oqz.unpack_codes(ac.cpu().numpy(), 4, d)
    cw = oqz.unpack_codes(wc.cpu().numpy(), 4, d)
    r16 = wn.float().cpu().double().numpy()
    c = codebooks(d, 4)["centroids"]
    ref = olin.linear_from_codes(ca, an.cpu().double().numpy(), cw, r16, c, c, d)
    yy = y.double().cpu().numpy()
    assert np.linalg.norm(yy - ref) / np.linalg.norm(ref) <= 2e-3


def test_debug_mode_reports_the_timeout_at_the_launching_call(oq):
    # With synchronous checking on (oq_set_debug / OQ_DEBUG=1), the entry point
    # that launched the kernel returns its give-up itself; normal calls in the
    # same mode return OQ_OK with the same results as asynchronous calls.
    d, M, N = 512, 300, 272
    torch.manual_seed(7)
    cb = oq.Codebook(d, 4)
    a = torch.randint(0, 256, (M, d // 2), dtype=torch.uint8, device="cuda")
    w = torch.randint(0, 256, (N, d // 2), dtype=torch.uint8, device="cuda")
    an = torch.rand(M, device="cuda")
    wn = torch.rand(N, device="cuda").to(torch.bfloat16)
    ref, _ = oq.linear_codes(d, cb, cb, a, an, w, wn)
    torch.cuda.synchronize()
    oq.device_status()
    lib = oq.lib()
    assert lib.oq_set_debug(1) == oq.OQ_OK
    try:
        y, _ = oq.linear_codes(d, cb, cb, a, an, w, wn)
        assert torch.equal(y, ref)
        assert lib.oq_test_stall_next(2) == oq.OQ_OK
        with pytest.raises(oq.OQError) as e:
            oq.linear_codes(d, cb, cb, a, an, w, wn)
        assert e.value.code == oq.OQ_ERR_TIMEOUT
    finally:
        lib.oq_test_stall_next(0)
        lib.oq_set_debug(0)
    oq.device_status()
    y, _ = oq.linear_codes(d, cb, cb, a, an, w, wn)
    torch.cuda.synchronize()
    oq.device_status()
    assert torch.equal(y, ref)
