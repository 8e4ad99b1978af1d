"""Seeded synthetic inputs for the int4 / FP8 mixture-of-experts FFN layer.

This module is shared by the tests, the benchmark and the CPU oracle's callers.
It only draws random numbers and rounds them to the storage dtypes the layer
takes (bf16 activations, bf16 router and shared-expert weights, fp32 routed
expert weights before quantization).  It performs none of the layer's own
arithmetic: no quantization, no routing, no GEMM.  Where a caller needs inputs
with a property that depends on the layer (top-k margins), it passes an
``accept`` callback and this module only redraws the rows the callback rejects.

Every tensor has its own PCG64 stream, derived from ``SeedSequence(seed,
spawn_key=(stream_id,))``, so any one tensor (for instance one expert's down
projection) can be regenerated alone and in any order.

Distributions (the workloads' stated recipe):
  * x ~ N(0, 1), drawn fp32, rounded to bf16 (round-to-nearest-even).
  * every weight ~ N(0, 0.02) (standard deviation 0.02), drawn fp32.  Router
    and shared-expert weights are rounded to bf16; routed expert weights are
    returned in fp32 and quantized by the caller.
  * the skewed workload adds a router bias b_e = 1.5 * ln(1 / (e + 1)).
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass
from typing import Callable, Iterator, Optional, Sequence

import numpy as np
import torch

__all__ = [
    "LayerShape", "SHAPES", "stream", "tokens", "router_weight", "router_bias",
    "shared_weights", "expert_weights", "iter_expert_weights", "to_bf16", "rms_weight",
    "WEIGHT_STD",
]

WEIGHT_STD = 0.02


@dataclass(frozen=True)
class LayerShape:
    """Sizes of one MoE FFN layer workload.

    T tokens, D model width, F routed-expert hidden width, E routed experts,
    k experts per token, F_shared the shared expert's hidden width, fmt the
    routed-weight storage ("int4" = int4 groups of 128, "fp8" = e4m3 rows).
    """
    name: str
    T: int
    D: int
    F: int
    E: int
    k: int
    F_shared: int
    fmt: str = "int4"
    skewed: bool = False

    def with_tokens(self, T: int) -> "LayerShape":
        return LayerShape(self.name, T, self.D, self.F, self.E, self.k,
                          self.F_shared, self.fmt, self.skewed)


# The workloads: a tiny layer, the Scout-shaped decode and prefill layers
# (16 experts, top-1), the Maverick-shaped FP8 layer (128 experts, top-8), a
# Scout-shaped layer with a Zipf-like router bias, and a 16-expert cut of the
# FP8 layer.
SHAPES = {
    "tiny": LayerShape("tiny", 64, 256, 512, 4, 1, 512, "int4"),
    "scout_decode": LayerShape("scout_decode", 16, 5120, 8192, 16, 1, 8192, "int4"),
    "scout_prefill": LayerShape("scout_prefill", 8192, 5120, 8192, 16, 1, 8192, "int4"),
    "maverick_fp8": LayerShape("maverick_fp8", 4096, 5120, 8192, 128, 8, 8192, "fp8"),
    "skewed": LayerShape("skewed", 32768, 5120, 8192, 16, 1, 8192, "int4", skewed=True),
    # the Maverick-shaped FP8 layer cut to 16 experts and 512 tokens (the same
    # 256 slots per expert on average, 2.3 GB of weights): a case small enough
    # for profiling captures of the FP8 kernels
    "maverick_fp8_e16": LayerShape("maverick_fp8_e16", 512, 5120, 8192, 16, 8, 8192, "fp8"),
}

# Stream ids.  Routed expert e uses ids 16 + 3e + {0: gate, 1: up, 2: down}.
_X, _ROUTER, _SHARED_GATE, _SHARED_UP, _SHARED_DOWN, _RMS = 0, 1, 2, 3, 4, 5


def _routed_stream_id(e: int, which: int) -> int:
    return 16 + 3 * e + which


def stream(seed: int, stream_id: int) -> np.random.Generator:
    """The PCG64 generator of one tensor."""
    return np.random.Generator(
        np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(stream_id,))))


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """Round an fp32 array to a bf16 CPU tensor (round-to-nearest-even)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _normal(g: np.random.Generator, shape, std: float) -> np.ndarray:
    a = g.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def tokens(seed: int, T: int, D: int,
           accept: Optional[Callable[[torch.Tensor], np.ndarray]] = None,
           max_rounds: int = 64) -> torch.Tensor:
    """x [T, D] bf16.

    ``accept(x) -> bool[T]`` marks the rows to keep; rejected rows are redrawn
    from the same stream, in row order, until every row is accepted.
    """
    g = stream(seed, _X)
    x = to_bf16(_normal(g, (T, D), 1.0))
    if accept is None:
        return x
    for _ in range(max_rounds):
        ok = np.asarray(accept(x), dtype=bool)
        bad = np.flatnonzero(~ok)
        if bad.size == 0:
            return x
        x[torch.from_numpy(bad)] = to_bf16(_normal(g, (bad.size, D), 1.0))
    raise RuntimeError("tokens: rows still rejected after %d redraws" % max_rounds)


def router_weight(seed: int, E: int, D: int) -> torch.Tensor:
    """W_r [E, D] bf16."""
    return to_bf16(_normal(stream(seed, _ROUTER), (E, D), WEIGHT_STD))


def rms_weight(seed: int, D: int) -> torch.Tensor:
    """gamma [D] bf16 of an RMSNorm in front of the layer: 1 + N(0, 0.1)
    (trained norm weights sit around 1; the pages give no values)."""
    return to_bf16(np.float32(1.0) + _normal(stream(seed, _RMS), (D,), 0.1))


def router_bias(shape: LayerShape) -> Optional[np.ndarray]:
    """b [E] fp32 for the skewed workload (b_e = 1.5 ln(1/(e+1))), else None."""
    if not shape.skewed:
        return None
    return np.array([1.5 * math.log(1.0 / (e + 1)) for e in range(shape.E)], dtype=np.float32)


def shared_weights(seed: int, D: int, F_shared: int):
    """Shared expert (W_gate [Fs, D], W_up [Fs, D], W_down [D, Fs]) in bf16."""
    return (to_bf16(_normal(stream(seed, _SHARED_GATE), (F_shared, D), WEIGHT_STD)),
            to_bf16(_normal(stream(seed, _SHARED_UP), (F_shared, D), WEIGHT_STD)),
            to_bf16(_normal(stream(seed, _SHARED_DOWN), (D, F_shared), WEIGHT_STD)))


def expert_weights(seed: int, e: int, D: int, F: int):
    """Routed expert e: (W_gate [F, D], W_up [F, D], W_down [D, F]) fp32."""
    return (_normal(stream(seed, _routed_stream_id(e, 0)), (F, D), WEIGHT_STD),
            _normal(stream(seed, _routed_stream_id(e, 1)), (F, D), WEIGHT_STD),
            _normal(stream(seed, _routed_stream_id(e, 2)), (D, F), WEIGHT_STD))


def iter_expert_weights(seed: int, experts: Sequence[int], D: int, F: int,
                        workers: Optional[int] = None,
                        ahead: Optional[int] = None) -> Iterator[tuple]:
    """Yield (e, W_gate, W_up, W_down) for each e, generated by a thread pool
    (numpy's generators release the GIL while they fill an array).

    At most ``ahead`` experts beyond the one being consumed are held in host
    memory (by default enough to keep every worker busy), so a 128-expert
    layer never needs all of its fp32 weights at once.
    """
    workers = workers or min(32, os.cpu_count() or 1)
    ahead = ahead if ahead is not None else max(2, (workers + 2) // 3)
    experts = list(experts)

    def job(e, w):
        shape = (F, D) if w < 2 else (D, F)
        return _normal(stream(seed, _routed_stream_id(e, w)), shape, WEIGHT_STD)

    with ThreadPoolExecutor(max_workers=workers) as ex:
        pending = []
        nxt = 0
        while nxt < len(experts) and len(pending) <= ahead:
            pending.append((experts[nxt], [ex.submit(job, experts[nxt], w) for w in range(3)]))
            nxt += 1
        while pending:
            e, futs = pending.pop(0)
            g, u, d = (f.result() for f in futs)
            if nxt < len(experts):
                pending.append((experts[nxt], [ex.submit(job, experts[nxt], w) for w in range(3)]))
                nxt += 1
            yield e, g, u, d
