"""Expert parallelism for the MoE layer: P ranks, one GPU each, every rank
holding E / P of the routed experts (and the router and shared expert) and
routing its own tokens.

"1 卡跑通 Llama 4" (discosf.com), the closing section on dependencies: the
models are split across GPUs with fairscale's model parallelism; "Llama"
(illegalscreed.cn), introduction: Maverick's 128 routed experts run on one
8-GPU node.  One step of a rank:

  1. route its tokens (moe_route): k (expert, gate) slots per token;
  2. dispatch: an all-to-all sends each slot's token row, the expert's index
     on its owner and the gate to the rank that holds the expert (expert e
     lives on rank e // (E / P)); rows are grouped by destination in slot
     order, so a rank receives each source's rows in the source's slot order;
  3. moe_expert_ffn_forward on the received rows (gate-scaled fp32 y);
  4. combine: an all-to-all returns every y row to its source, where it
     lands at its slot;
  5. moe_shared_ffn_combine: out = bf16(shared(x) + sum_j y[t, j]), the
     slots summed in order, as the one-GPU layer does.

The exchanges are torch.distributed all-to-alls (NCCL between GPUs); a
received row is in this rank's memory before a kernel reads it.  Steps 1, 3
and 5 are callables, so the same bookkeeping runs with the library's kernels
(`library_steps`) or, in tests, with any other implementation of the steps.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist


@dataclass
class Steps:
    """The compute steps the exchanges run around.

    prepare(x) -> the layer's input as every other step sees it (the
        block's RMSNorm, when the layer has one; None: x itself);
    route(x) -> (ids int32 [T, k], gates fp32 [T, k]) over all E experts;
    experts(x_rows, local_ids int32 [n], gates fp32 [n]) -> y fp32 [n, D],
        y[r] = gates[r] * expert(local_ids[r])(x_rows[r]), this rank's experts;
    shared(x, y_slots fp32 [T, k, D]) -> out [T, D].
    """
    route: Callable[[torch.Tensor], Tuple[torch.Tensor, torch.Tensor]]
    experts: Callable[[torch.Tensor, torch.Tensor, torch.Tensor], torch.Tensor]
    shared: Callable[[torch.Tensor, torch.Tensor], torch.Tensor]
    prepare: Optional[Callable[[torch.Tensor], torch.Tensor]] = None


def owners(E: int, world: int) -> int:
    """Experts per rank (E must divide evenly)."""
    if E % world:
        raise ValueError("E = %d experts do not split evenly over %d ranks" % (E, world))
    return E // world


class ExpertParallelLayer:
    """One MoE layer spread over the ranks of `group` (the default group if
    None).  Every rank calls forward() with its own tokens, the same number
    of times and in the same order."""

    def __init__(self, E: int, k: int, D: int, steps: Steps, group=None):
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.E, self.k, self.D = E, k, D
        self.e_local = owners(E, self.world)
        self.steps = steps

    def _exchange(self, recv: torch.Tensor, send: torch.Tensor, recv_counts, send_counts) -> None:
        if self.world == 1:
            recv.copy_(send)
        else:
            dist.all_to_all_single(recv, send, recv_counts, send_counts, group=self.group)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        if self.steps.prepare is not None:
            x = self.steps.prepare(x)
        T, D, k = x.shape[0], self.D, self.k
        ids, gates = self.steps.route(x)
        flat_ids = ids.reshape(-1).to(torch.int64)
        dest = torch.div(flat_ids, self.e_local, rounding_mode="floor")
        # slots grouped by destination rank, in slot order within each
        order = torch.sort(dest, stable=True).indices
        send_counts_t = torch.bincount(dest, minlength=self.world)
        recv_counts_t = torch.empty_like(send_counts_t)
        self._exchange(recv_counts_t, send_counts_t, [1] * self.world, [1] * self.world)
        send_counts = [int(c) for c in send_counts_t.tolist()]
        recv_counts = [int(c) for c in recv_counts_t.tolist()]
        n_recv = sum(recv_counts)

        # dispatch: token rows, local expert indices, gates
        send_x = x.index_select(0, torch.div(order, k, rounding_mode="floor"))
        send_ids = (flat_ids.index_select(0, order) % self.e_local).to(torch.int32)
        send_gates = gates.reshape(-1).index_select(0, order).contiguous()
        recv_x = torch.empty(n_recv, D, dtype=x.dtype, device=x.device)
        recv_ids = torch.empty(n_recv, dtype=torch.int32, device=x.device)
        recv_gates = torch.empty(n_recv, dtype=send_gates.dtype, device=x.device)
        self._exchange(recv_x, send_x, recv_counts, send_counts)
        self._exchange(recv_ids, send_ids, recv_counts, send_counts)
        self._exchange(recv_gates, send_gates, recv_counts, send_counts)

        y_recv = self.steps.experts(recv_x, recv_ids, recv_gates)

        # combine: every y row back to its source rank, at its slot
        y_back = torch.empty(T * k, D, dtype=y_recv.dtype, device=x.device)
        self._exchange(y_back, y_recv.contiguous(), send_counts, recv_counts)
        y_slots = torch.empty_like(y_back)
        y_slots.index_copy_(0, order, y_back)
        return self.steps.shared(x, y_slots.view(T, k, D))

    __call__ = forward


def library_steps(router_weight: torch.Tensor, router_bias: Optional[torch.Tensor], k: int, local_layer,
                  rms_weight: Optional[torch.Tensor] = None, rms_eps: float = 1e-5) -> Steps:
    """The steps on this rank's GPU through the library: moe_route over all
    E experts, moe_expert_ffn_forward with `local_layer` (a MoELayer holding
    this rank's experts and the shared expert, without an RMSNorm of its
    own), and moe_shared_ffn_combine.  With `rms_weight` the tokens are
    normalized once (moe_rmsnorm) and every step sees the normalized rows."""
    from . import rmsnorm, route

    def route_fn(x):
        r = route(x, router_weight, router_bias, k)
        return r["ids"], r["gates"]

    prepare = None
    if rms_weight is not None:
        def prepare(x):
            return rmsnorm(x, rms_weight, rms_eps)

    return Steps(route=route_fn, experts=local_layer.expert_forward, shared=local_layer.shared_combine,
                 prepare=prepare)
