"""Oracle: SwiGLU experts, the shared expert and the whole MoE FFN layer.

TEST INFRASTRUCTURE ONLY (see the package docstring).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional, Sequence

import numpy as np

from . import quant
from .route import _f64, route


def bf16_round(v) -> np.ndarray:
    """Round fp64 values to the nearest value with 8 significant bits (bf16),
    ties to even.  (Values below bf16's normal range do not occur here.)"""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    return np.ldexp(np.rint(m * 256.0), e - 8)


def silu(z: np.ndarray) -> np.ndarray:
    """Swish(z) = z * sigmoid(z) ([P5] "SwiGLU：门控激活的数学")."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu(x: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """y = (Swish(x W) * (x V)) W2 for rows x[n, D] ([P5] "SwiGLU：门控激活的数学").

    Weights are stored "nt" ([P2] bmm_nt: W[N, K], product x W^T), so
    W = w_gate[F, D], V = w_up[F, D], W2 = w_down[D, F].  Reading: g and u are
    exact (fp64 here); h = silu(g) * u is rounded once to bf16 because the
    layer keeps activations in bf16 ([P1] "FP8 / Int4 混合量化"); y is exact.
    """
    g = x @ w_gate.T
    u = x @ w_up.T
    h = bf16_round(silu(g) * u)
    return h @ w_down.T


def swiglu_fp8(x: np.ndarray, gate, up, down, scale_ub: float = float("inf")) -> np.ndarray:
    """FP8 row-wise expert ([P2] "量化环节做了什么", bmm_nt's FP8 branch).

    Every matmul input is quantized per row to e4m3 with the weight's
    activation-scale bound, then multiplied by the e4m3 row-quantized weight;
    both operands are taken at their dequantized values.  ``gate``, ``up`` and
    ``down`` are (codes uint8 [N, K], row scales fp32 [N]).
    """
    xq, sx = quant.fp8_row_quantize(np.asarray(x, dtype=np.float32), scale_ub=scale_ub)
    xh = quant.dequant_fp8_rows(xq, sx)
    g = xh @ quant.dequant_fp8_rows(*gate).T
    u = xh @ quant.dequant_fp8_rows(*up).T
    h = bf16_round(silu(g) * u)
    hq, sh = quant.fp8_row_quantize(h.astype(np.float32), scale_ub=scale_ub)
    return quant.dequant_fp8_rows(hq, sh) @ quant.dequant_fp8_rows(*down).T


@dataclass
class Layer:
    """One MoE FFN layer as the oracle sees it.

    ``expert(e)`` returns the stored weights of routed expert e as three
    (codes, scales) pairs (gate [F, D], up [F, D], down [D, F]): for "int4"
    unpacked int8 codes with fp32 scales, one per ``group_size`` (128, or
    the smaller 64 / 32) values along K, for "fp8" e4m3 codes
    (uint8) with fp32 row scales.  Router and shared weights are the bf16
    values (any array type; converted to fp64).
    """
    fmt: str
    k: int
    w_router: object
    bias: Optional[np.ndarray]
    expert: Callable[[int], tuple]
    shared: tuple
    act_scale_ub: float = float("inf")
    group_size: int = 128
    rms_weight: object = None      # gamma [D] of an RMSNorm applied to x first, or None
    rms_eps: float = 1e-5

    def expert_output(self, e: int, x_rows: np.ndarray) -> np.ndarray:
        """y = expert e applied to x_rows[n, D] (fp64 values of bf16 inputs)."""
        (qg, sg), (qu, su), (qd, sd) = self.expert(e)
        if self.fmt == "int4":
            G = self.group_size
            return swiglu(x_rows, quant.dequant_int4(qg, sg, G),
                          quant.dequant_int4(qu, su, G), quant.dequant_int4(qd, sd, G))
        if self.fmt == "fp8":
            return swiglu_fp8(x_rows, (qg, sg), (qu, su), (qd, sd), self.act_scale_ub)
        raise ValueError(self.fmt)

    def shared_output(self, x_rows: np.ndarray) -> np.ndarray:
        """The always-on shared expert: SwiGLU with bf16 weights, no gate
        ([P1] "混合专家路由": every token also passes the shared expert)."""
        wg, wu, wd = (_f64(w) for w in self.shared)
        return swiglu(x_rows, wg, wu, wd)


def dense_forward(x, w_gate, w_up, w_down, rms_weight=None, rms_eps: float = 1e-5) -> np.ndarray:
    """A dense SwiGLU FFN layer, the FFN of the dense layers that alternate
    with the MoE layers ([P4] introduction; [P5] "SwiGLU：门控激活的数学"):
    out = bf16(swiglu(x)) with bf16 weights -- the shared expert on its own.
    With ``rms_weight``, x is first replaced by its RMSNorm (norm.rmsnorm).
    Returns fp64 values of the bf16 outputs."""
    if rms_weight is not None:
        from .norm import rmsnorm
        x = rmsnorm(x, rms_weight, rms_eps)
    return bf16_round(swiglu(_f64(x), _f64(w_gate), _f64(w_up), _f64(w_down)))


def moe_forward(layer: Layer, x, tokens: Optional[Sequence[int]] = None) -> dict:
    """The layer for all tokens, or for the listed ``tokens`` only.

    [P1] "混合专家路由" (MoE.forward): router scores -> top-k -> each chosen
    expert runs on its tokens -> scatter_add_ of the expert outputs, weighted
    by their scores, back into their tokens -> plus the shared expert:
        out[t] = bf16( sum_j gate[t, j] * y_{ids[t, j]}(x[t]) + shared(x[t]) ).
    The routing is computed for the whole batch (it is per token anyway).
    With ``layer.rms_weight`` set, x is first replaced by its RMSNorm
    (norm.rmsnorm: the block's normalization in front of the FFN, [P5]
    "RMSNorm：为什么去掉减均值也能工作"), rounded to bf16.
    Returns the routing dict plus ``out`` (fp64 values of the bf16 outputs,
    one row per selected token) and ``tokens``.
    """
    if layer.rms_weight is not None:
        from .norm import rmsnorm
        x = rmsnorm(x, layer.rms_weight, layer.rms_eps)
    xf = _f64(x)
    r = route(x, layer.w_router, layer.bias, layer.k)
    T = xf.shape[0]
    sel = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    ids, gates = r["ids"], r["gates"]
    acc = np.zeros((sel.size, xf.shape[1]), dtype=np.float64)
    sub_ids = ids[sel]
    for e in np.unique(sub_ids):
        rows, js = np.nonzero(sub_ids == e)
        if rows.size == 0:
            continue
        y = layer.expert_output(int(e), xf[sel[rows]])
        acc[rows] += gates[sel[rows], js][:, None] * y
    out = bf16_round(acc + layer.shared_output(xf[sel]))
    r.update(out=out, tokens=sel)
    return r


def moe_forward_dense(layer: Layer, x, E: int) -> np.ndarray:
    """Brute force: every expert on every token, weighted by a gate vector
    that is zero off each token's top-k; must equal :func:`moe_forward`."""
    if layer.rms_weight is not None:
        from .norm import rmsnorm
        x = rmsnorm(x, layer.rms_weight, layer.rms_eps)
    xf = _f64(x)
    r = route(x, layer.w_router, layer.bias, layer.k)
    T = xf.shape[0]
    gate_full = np.zeros((T, E), dtype=np.float64)
    np.put_along_axis(gate_full, r["ids"].astype(np.int64), r["gates"], axis=1)
    acc = np.zeros_like(xf)
    for e in range(E):
        acc += gate_full[:, e:e + 1] * layer.expert_output(e, xf)
    return bf16_round(acc + layer.shared_output(xf))
