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

    @functools.lru_cache(maxsize=4)
    def expert(e):
        ws = synth.expert_weights(seed, e, D, F)
        if shape.fmt == "int4":
            return tuple(oq.int4_row_quantize(w, group_size=group_size) for w in ws)
        return tuple(oq.fp8_row_quantize(w) for w in ws)

    olayer = offn.Layer(shape.fmt, k, wr, bias, expert, (sg, su, sd), group_size=group_size,
                        rms_weight=gamma, rms_eps=rms_eps)
    return Built(shape, x, layer, olayer, wr, bias)


def rel_err(gpu_out: np.ndarray, ref: np.ndarray) -> float:
    """max |gpu - oracle| / max |oracle|."""
    return float(np.abs(gpu_out - ref).max() / max(np.abs(ref).max(), 1e-30))
