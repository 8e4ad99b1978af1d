"""Oracle: router scores, top-k expert choice, gates and token bucketing.

TEST INFRASTRUCTURE ONLY (see the package docstring).
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    """bf16 / fp32 torch tensors or numpy arrays -> fp64 numpy (exact)."""
    if hasattr(a, "detach"):
        a = a.detach().float().numpy()
    return np.asarray(a, dtype=np.float64)


def router_logits(x, w_router, bias=None) -> np.ndarray:
    """logits[t, e] = sum_d x[t, d] * W_r[e, d] (+ b_e), in fp64.

    [P1] "混合专家路由": the router scores every token against every expert;
    [P5] "MoE 架构详解": the router is a linear layer.  The bias term exists
    only for the skewed workload.
    """
    lg = _f64(x) @ _f64(w_router).T
    if bias is not None:
        lg = lg + _f64(bias)[None, :]
    return lg


def topk_select(logits: np.ndarray, k: int) -> np.ndarray:
    """ids[t, j]: the k largest logits of token t, largest first, equal logits
    ordered by lower expert index ([P1] "混合专家路由": torch.topk over the
    router scores; the tie rule and the descending slot order are readings)."""
    order = np.argsort(-logits, axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def gate_values(logits: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """Gate of each chosen slot, fp64.

    k = 1: sigmoid of the chosen logit.  k > 1: softmax over the k chosen
    logits (max subtracted).  [P5] "MoE 架构详解" says "linear layer +
    softmax"; the sigmoid for a single chosen expert is the reading fixed for
    this layer (a softmax over one logit would always be 1).
    """
    chosen = np.take_along_axis(logits, ids.astype(np.int64), axis=1)
    if ids.shape[1] == 1:
        with np.errstate(over="ignore"):
            return 1.0 / (1.0 + np.exp(-chosen))
    z = chosen - chosen.max(axis=1, keepdims=True)
    ez = np.exp(z)
    return ez / ez.sum(axis=1, keepdims=True)


def bucket(ids: np.ndarray, E: int):
    """Group the T*k slots (slot s = t*k + j) by expert.

    counts[e] = number of slots choosing e; offsets = exclusive prefix sum
    (E + 1 entries); perm lists the slots of expert 0, then 1, ..., each in
    ascending slot (hence token) order; inv_perm[s] = position of slot s in perm.
    [P1] "混合专家路由" / [P5] "稀疏激活": only the chosen experts compute,
    so each expert sees just its own tokens; the stable order is a reading.
    """
    flat = ids.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    inv_perm = np.empty_like(perm)
    inv_perm[perm] = np.arange(perm.size, dtype=np.int32)
    return counts, offsets, perm, inv_perm


def topk_margin_ok(logits: np.ndarray, k: int, margin: float = 1e-3) -> np.ndarray:
    """True for tokens whose top-(k+1) sorted logits are pairwise more than
    ``margin`` apart, so fp32 and fp64 evaluations choose the same experts in
    the same order.  (With k = E only the k chosen logits are compared.)"""
    E = logits.shape[1]
    m = min(k + 1, E)
    top = -np.sort(-logits, axis=1)[:, :m]
    if m < 2:
        return np.ones(logits.shape[0], dtype=bool)
    return (np.diff(-top, axis=1) > margin).all(axis=1)


def route(x, w_router, bias, k: int) -> dict:
    """Everything the routing step produces for a batch of tokens."""
    E = _f64(w_router).shape[0]
    lg = router_logits(x, w_router, bias)
    ids = topk_select(lg, k)
    gates = gate_values(lg, ids)
    counts, offsets, perm, inv_perm = bucket(ids, E)
    return dict(logits=lg, ids=ids, gates=gates, counts=counts,
                offsets=offsets, perm=perm, inv_perm=inv_perm)
