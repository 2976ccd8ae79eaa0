"""oq_linear_noalloc: the full layer for callers that cannot allocate device
memory (an engine callback that owns every allocation, a loop that cannot
take cudaMalloc's synchronisation).  It keeps its scratch in the library's
static device array instead of a caller workspace.

Checked through the C ABI against the existing entry point (oq_linear with a
workspace) on the same inputs, within the same 2e-3 relative Frobenius bound
the other linear tests use, on two calls in a row -- the second with fewer
rows and different data, so stale scratch contents from the first call
cannot leak into it.  This file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

from calibration_free_rotated_b200 import inputs

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


def _dev_bf16(bits_u16):
    return torch.from_numpy(np.ascontiguousarray(bits_u16).view(np.int16)).cuda().view(torch.bfloat16)


def _rel(a, b):
    a, b = a.double(), b.double()
    return float(torch.linalg.norm(a - b) / torch.linalg.norm(b))


def test_noalloc_matches_linear_on_two_calls(oq):
    torch.cuda.set_device(0)
    d, h, N = 3072, 128, 1024
    r = oq.Rpbh(0, d, h)
    cb = oq.Codebook(d, 4)
    W = _dev_bf16(inputs.weights(2, inputs.T_W, N, d))
    bias = _dev_bf16(inputs.bias(2, N))
    w_codes, w_norm = oq.quantize_weight(r, cb, W)
    for call, (M, rows) in enumerate([(1000, (0, 1000)), (333, (2000, 2333))]):
        X = _dev_bf16(inputs.activations(2, 4608, d, rows=rows))
        ref, _ = oq.linear(r, cb, cb, X, w_codes, w_norm, bias=bias)
        y32 = torch.full((M, N), float("nan"), device="cuda")
        y16 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        allocs = oq.device_allocations()
        oq.linear_noalloc(r, cb, cb, X, w_codes, w_norm, bias=bias, out_f32=y32, out_bf16=y16)
        assert oq.device_allocations() == allocs, "the no-allocation entry point allocated device memory"
        torch.cuda.synchronize()
        oq.device_status()
        assert _rel(y32, ref) <= TOL, f"call {call}"
        assert _rel(y16.float(), ref) <= TOL, f"call {call}"


def test_noalloc_rejects_sizes_beyond_the_static_scratch(oq):
    d = 3072
    r = oq.Rpbh(0, d, 128)
    cb = oq.Codebook(d, 4)
    M = oq.NOALLOC_SCRATCH_BYTES // (d // 2) + 1          # codes alone exceed the array
    X = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((16, d // 2), dtype=torch.uint8, device="cuda")
    wn = torch.ones(16, dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, 16), device="cuda")
    with pytest.raises(oq.OQError) as e:
        oq.linear_noalloc(r, cb, cb, X, w, wn, out_f32=y)
    assert e.value.code == oq.OQ_ERR_UNSUPPORTED
    assert "static scratch" in str(e.value)


def test_noalloc_with_a_composed_rotation(oq):
    # A 2-round composed rotation uploads its round tables when the handle is
    # made (with the device current), so the no-allocation path runs with it.
    torch.cuda.set_device(0)
    d, h, N, M = 1536, 128, 512, 700
    r = oq.Rpbh(0, d, h, rounds=2)
    cb = oq.Codebook(d, 4)
    W = _dev_bf16(inputs.weights(4, inputs.T_W, N, d))
    w_codes, w_norm = oq.quantize_weight(r, cb, W)
    X = _dev_bf16(inputs.activations(4, M, d))
    ref, _ = oq.linear(r, cb, cb, X, w_codes, w_norm)
    y32 = torch.full((M, N), float("nan"), device="cuda")
    oq.linear_noalloc(r, cb, cb, X, w_codes, w_norm, out_f32=y32)
    torch.cuda.synchronize()
    oq.device_status()
    assert torch.equal(y32, ref)  # same kernels on the same inputs
