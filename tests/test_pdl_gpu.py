"""Programmatic dependent launch changes when a kernel's set-up runs, never
what it computes: the same chain of launches (act-quant -> GEMM -> act-quant ->
GEMM, back to back in one stream, so each kernel overlaps the previous one)
gives bit-identical outputs with the launch attribute on and with it off
(OQ_NO_PDL=1, read once per process, hence the child processes)."""

import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
from calibration_free_rotated_b200 import inputs, orbitquant as oq
bf = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).cuda().view(torch.bfloat16)
M, d1, d2, h = 3000, 1536, 3072, 128
r1, r2 = oq.Rpbh(0, d1, h), oq.Rpbh(0, d2, h)
ca1, cw1, ca2, cw2 = oq.Codebook(d1, 6), oq.Codebook(d1, 4), oq.Codebook(d2, 4), oq.Codebook(d2, 2)
w1c, w1n = oq.quantize_weight(r1, cw1, bf(inputs.weights(4, inputs.T_W, d2, d1)))
w2c, w2n = oq.quantize_weight(r2, cw2, bf(inputs.weights(4, inputs.T_W2, d1, d2)))
X = bf(inputs.activations(4, M, d1))
outs = []
for rep in range(3):  # several chains back to back: each launch follows a GEMM or an act-quant
    a1c, a1n = oq.quantize_act(r1, ca1, X)
    _, y1 = oq.linear_codes(d1, ca1, cw1, a1c, a1n, w1c, w1n, epilogue="gelu", want_f32=False, want_bf16=True)
    a2c, a2n = oq.quantize_act(r2, ca2, y1)
    y2, _ = oq.linear_codes(d2, ca2, cw2, a2c, a2n, w2c, w2n)
    outs.append((a1c, a1n, y1, a2c, a2n, y2))
torch.cuda.synchronize()
oq.device_status()
for o in outs[1:]:
    assert all(torch.equal(a, b) for a, b in zip(o, outs[0]))
torch.save([t.cpu() for t in outs[0]], sys.argv[2])
"""


def _run(tmp_path, name, pdl):
    env = dict(os.environ)
    env.pop("OQ_NO_PDL", None)
    if not pdl:
        env["OQ_NO_PDL"] = "1"
    out = str(tmp_path / name)
    r = subprocess.run([sys.executable, "-c", _CHILD, ROOT, out], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return torch.load(out)


def test_outputs_identical_with_and_without_pdl(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from calibration_free_rotated_b200 import build
    build.build()
    on = _run(tmp_path, "on.pt", True)
    off = _run(tmp_path, "off.pt", False)
    for a, b in zip(on, off):
        assert torch.equal(a, b)
