"""Oracle: RMSNorm, the normalization before a Llama block's FFN.

TEST INFRASTRUCTURE ONLY (see the package docstring).

[P5] "Llama 开源模型系列" (docs.ifdog.com), section "RMSNorm：为什么去掉减均值也能
工作": RMSNorm(x) = x / sqrt((1/d) sum_i x_i^2 + eps) * gamma -- no mean
subtraction, only the scaling by the root mean square.
"""
from __future__ import annotations

import numpy as np

from .ffn import bf16_round
from .route import _f64


def rmsnorm(x, gamma, eps: float) -> np.ndarray:
    """RMSNorm of every row of x [T, D] with weights gamma [D].

    Readings (the page gives the formula only): the mean of squares, the
    root and the products are exact (fp64 here); the result is rounded once
    to bf16, as the layer keeps activations in bf16; eps is the caller's
    value.  Returns fp64 values of the bf16 results.
    """
    xf = _f64(x)
    g = _f64(gamma).reshape(1, -1)
    ms = (xf * xf).mean(axis=1, keepdims=True)
    return bf16_round(xf / np.sqrt(ms + float(eps)) * g)
