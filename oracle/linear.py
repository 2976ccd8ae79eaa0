"""Quantized linear layer (oracle side, fp64).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

[OQ] Methodology, "Online Activation Quantization", last paragraph: the shared
rotation cancels, W^' x^' ~= W Pi^T Pi x = W x, so no inverse rotation is
needed.  With x^' = s C_a[codes_a] and W^' = diag(r') C_w[codes_w]:

    y[m, n] = s_m * r'_n * sum_k v_a[ca[m, k]] * v_w[cw[n, k]]  (+ bias_n)

where v is the dequantisation table.  Reading: v = (declared fp16 LUT of
sqrt(d) c_k) / sqrt(d), so the oracle sums on exactly the values the kernel
multiplies; ``exact_centroids=True`` uses the fp64 centroids instead.

The pages never mention an activation between two linears; where a
configuration places GELU between fc1 and fc2, the reading is the exact erf
form 0.5 y (1 + erf(y / sqrt 2)).
"""

import math

import numpy as np
from scipy.special import erf

from .codebook import fp16_lut


def dequant_table(centroids: np.ndarray, d: int, exact_centroids: bool = False) -> np.ndarray:
    if exact_centroids:
        return np.asarray(centroids, dtype=np.float64)
    return fp16_lut(centroids, d).astype(np.float64) / math.sqrt(d)


def linear_from_codes(codes_a, norms_a, codes_w, norms_w, cent_a, cent_w, d,
                      bias=None, gelu: bool = False, exact_centroids: bool = False):
    """fp64 y[M, N] from unpacked codes (int[M, d], int[N, d]) and norms."""
    va = dequant_table(cent_a, d, exact_centroids)
    vw = dequant_table(cent_w, d, exact_centroids)
    A = va[np.asarray(codes_a)] * np.asarray(norms_a, dtype=np.float64)[:, None]
    B = vw[np.asarray(codes_w)] * np.asarray(norms_w, dtype=np.float64)[:, None]
    y = A @ B.T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    if gelu:
        y = gelu_erf(y)
    return y


def gelu_erf(y):
    y = np.asarray(y, dtype=np.float64)
    return 0.5 * y * (1.0 + erf(y / math.sqrt(2.0)))
