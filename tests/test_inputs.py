"""The seeded workload generator: determinism, row-range independence, bf16 rounding."""

import numpy as np
import torch

from calibration_free_rotated_b200 import inputs


def test_bf16_conversion_matches_torch():
    rng = np.random.default_rng(0)
    v = rng.standard_normal(100000) * 10.0 ** rng.integers(-4, 5, 100000)
    ours = inputs.to_bf16_bits(v)
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(inputs.bf16_bits_to_f64(ours),
                          torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).double().numpy())


def test_row_ranges_regenerate_identically():
    full = inputs.activations(2, 3000, 64)
    part = inputs.activations(2, 3000, 64, rows=(1000, 2100))
    assert np.array_equal(full[1000:2100], part)
    w = inputs.weights(2, inputs.T_W, 2500, 32)
    assert np.array_equal(w[2047:2049], inputs.weights(2, inputs.T_W, 2500, 32, rows=(2047, 2049)))
    s = inputs.sweep_activations(1024, 128)
    assert np.array_equal(s[900:1024], inputs.sweep_activations(1024, 128, rows=(900, 1024)))


def test_sweep_adversarial_tail():
    M, d = 1024, 256
    x = inputs.bf16_bits_to_f64(inputs.sweep_activations(M, d))
    nnz = np.count_nonzero(x, axis=1)
    assert np.all(nnz[: M - M // 8] > d // 2)
    tail = nnz[M - M // 8:]
    assert set(np.unique(tail).tolist()) <= {0, 1, 2, 8, 64}
    assert tail[-1] == 0 and np.sum(tail == 1) >= 30


def test_workload_shapes_and_outliers():
    x = inputs.bf16_bits_to_f64(inputs.activations(1, 64, 256))
    col_rms = np.sqrt(np.mean(x ** 2, axis=0))
    assert np.sum(col_rms > 8) == 3                      # 1% of 256 channels, x20
    assert inputs.weights(1, inputs.T_W, 256, 256).shape == (256, 256)
