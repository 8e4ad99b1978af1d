"""Builds one MoE layer twice from the same seeded inputs: on the GPU through
the library (weights quantized by the library's own kernels) and for the CPU
oracle (weights quantized by the oracle).  Test helper only."""
from __future__ import annotations

import functools
import math
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

import int4_quantized_expert_b200 as moe
import synth
from oracle import ffn as offn
from oracle import quant as oq
from oracle import norm as onorm
from oracle import route as oroute


@dataclass
class Built:
    shape: synth.LayerShape
    x: torch.Tensor                # bf16 [T, D] (CPU)
    gpu: moe.MoELayer
    oracle: offn.Layer
    w_router: torch.Tensor         # bf16 CPU
    bias: Optional[np.ndarray]


def margin_tokens(shape: synth.LayerShape, w_router, bias, seed: int, margin: bool = True, gamma=None,
                  eps: float = 1e-5):
    accept = None
    if margin:
        def accept(x):
            xr = x if gamma is None else onorm.rmsnorm(x, gamma, eps)   # the router sees RMSNorm(x)
            return oroute.topk_margin_ok(oroute.router_logits(xr, w_router, bias), shape.k)
    return synth.tokens(seed, shape.T, shape.D, accept=accept)


def build(shape: synth.LayerShape, seed: int = 0, margin: bool = True, path: int = moe.PATH_AUTO,
          device: str = "cuda", group_size: int = 128, rms: bool = False, rms_eps: float = 1e-5) -> Built:
    E, k, D, F, Fs = shape.E, shape.k, shape.D, shape.F, shape.F_shared
    wr = synth.router_weight(seed, E, D)
    bias = synth.router_bias(shape)
    sg, su, sd = synth.shared_weights(seed, D, Fs)
    gamma = synth.rms_weight(seed, D) if rms else None
    x = margin_tokens(shape, wr, bias, seed, margin, gamma, rms_eps)
    dev = torch.device(device)

    if shape.fmt == "int4":
        alloc = lambda n, kk: (torch.empty(E, n, kk // 2, dtype=torch.uint8, device=dev),
                               torch.empty(E, n, kk // group_size, dtype=torch.float32, device=dev))
        quant = lambda w, out: moe.quantize_int4(w, group_size=group_size, out=out)
        fmt = moe.FMT_INT4
    else:
        alloc = lambda n, kk: (torch.empty(E, n, kk, dtype=torch.uint8, device=dev),
                               torch.empty(E, n, dtype=torch.float32, device=dev))
        quant = lambda w, out: moe.quantize_fp8_rows(w, out=out)
        fmt = moe.FMT_FP8
    gate, up, down = alloc(F, D), alloc(F, D), alloc(D, F)
    for e, g, u, d in synth.iter_expert_weights(seed, range(E), D, F):
        for w, (codes, scales) in ((g, gate), (u, up), (d, down)):
            quant(torch.from_numpy(w).to(dev), (codes[e], scales[e]))
    torch.cuda.synchronize()

    layer = moe.MoELayer(
        E=E, k=k, D=D, F=F, F_shared=Fs, w_router=wr.to(dev),
        router_bias=None if bias is None else torch.from_numpy(bias).to(dev),
        gate=gate, up=up, down=down, shared=(sg.to(dev), su.to(dev), sd.to(dev)),
        fmt=fmt, T_max=shape.T, path=path, group_size=group_size,
        rms_weight=None if gamma is None else gamma.to(dev), rms_eps=rms_eps)

    olayer = oracle_layer(shape, seed, group_size, gamma, rms_eps)
    return Built(shape, x, layer, olayer, wr, bias)


def oracle_layer(shape: synth.LayerShape, seed: int = 0, group_size: int = 128, gamma=None,
                 rms_eps: float = 1e-5) -> offn.Layer:
    """The oracle's view of the layer ``build`` makes: the same seeded
    router, shared and routed weights, the routed ones quantized by the oracle."""
    E, k, D, F, Fs = shape.E, shape.k, shape.D, shape.F, shape.F_shared
    wr = synth.router_weight(seed, E, D)
    bias = synth.router_bias(shape)
    shared = synth.shared_weights(seed, D, Fs)

    @functools.lru_cache(maxsize=4)
    def expert(e):
        ws = synth.expert_weights(seed, e, D, F)
        if shape.fmt == "int4":
            return tuple(oq.int4_row_quantize(w, group_size=group_size) for w in ws)
        return tuple(oq.fp8_row_quantize(w) for w in ws)

    return offn.Layer(shape.fmt, k, wr, bias, expert, shared, group_size=group_size,
                      rms_weight=gamma, rms_eps=rms_eps)


def covering_tokens(ids: np.ndarray, E: int, n_extra: int, seed: int) -> np.ndarray:
    """Tokens to check at full size: for every expert that some token chose,
    one (seeded, random) token that chose it -- taken greedily, so a token
    covers all of its k experts -- plus ``n_extra`` more random tokens."""
    rng = np.random.default_rng(seed)
    T = ids.shape[0]
    chosen, covered = [], set()
    for e in rng.permutation(E):
        if e in covered:
            continue
        cand = np.nonzero((ids == e).any(axis=1))[0]
        if cand.size == 0:
            continue
        t = int(rng.choice(cand))
        chosen.append(t)
        covered.update(int(v) for v in ids[t])
    rest = np.setdiff1d(np.arange(T), chosen)
    extra = rng.choice(rest, min(n_extra, rest.size), replace=False)
    return np.sort(np.concatenate([np.asarray(chosen, dtype=np.int64), extra.astype(np.int64)]))


def _oracle_part(args):
    shape, seed, group_size, x, tokens = args
    layer = oracle_layer(shape, seed, group_size)
    return offn.moe_forward(layer, x, tokens=tokens)["out"]


def oracle_outputs(shape: synth.LayerShape, x, tokens: np.ndarray, ids: np.ndarray, seed: int = 0,
                   group_size: int = 128, workers: int = 0) -> np.ndarray:
    """oracle moe_forward rows of ``tokens``, computed by ``workers`` spawned
    processes (the cost is one weight preparation per distinct expert, so the
    tokens are split into parts with few experts each).  Same values as one
    call: every token's row depends on its own experts only."""
    import multiprocessing as mp
    import os
    from concurrent.futures import ProcessPoolExecutor
    workers = workers or min(16, os.cpu_count() or 1)
    # order the tokens by their first expert so each part touches few experts
    order = np.argsort(ids[tokens, 0], kind="stable")
    parts = [p for p in np.array_split(tokens[order], workers) if p.size]
    with ProcessPoolExecutor(len(parts), mp_context=mp.get_context("spawn")) as ex:
        outs = list(ex.map(_oracle_part, [(shape, seed, group_size, x, p) for p in parts]))
    rows = {}
    for p, o in zip(parts, outs):
        for i, t in enumerate(p):
            rows[int(t)] = o[i]
    return np.stack([rows[int(t)] for t in tokens])


def rel_err(gpu_out: np.ndarray, ref: np.ndarray) -> float:
    """max |gpu - oracle| / max |oracle|."""
    return float(np.abs(gpu_out - ref).max() / max(np.abs(ref).max(), 1e-30))
