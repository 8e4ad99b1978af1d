"""The expert-parallel layer's bookkeeping on CPU: two ranks over gloo, each
holding half of the experts and routing its own tokens; the compute steps
(route, the rank's experts, shared expert + combine) are the oracle's, so the
ranks' outputs must equal the oracle's one-process layer on the same tokens.
A rank that receives no rows (every token routed to the other rank's experts)
is covered too."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import synth
from oracle import ffn as offn
from oracle import route as oroute
from tests._layers import oracle_layer


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_steps(shape, layer, rank, e_local):
    from int4_quantized_expert_b200.ep import Steps

    def route(x):
        r = oroute.route(x, layer.w_router, layer.bias, shape.k)
        return torch.from_numpy(r["ids"]), torch.from_numpy(r["gates"])

    def experts(rows, local_ids, gates):
        y = torch.zeros(rows.shape[0], shape.D, dtype=torch.float64)
        xr = rows.double().numpy()
        ids = local_ids.numpy()
        for e in np.unique(ids):
            sel = np.nonzero(ids == e)[0]
            out = layer.expert_output(int(rank * e_local + e), xr[sel])      # this rank's expert e
            y[sel] = torch.from_numpy(out) * gates[sel].double()[:, None]
        return y

    def shared(x, y_slots):
        acc = y_slots.sum(dim=1).numpy()       # the slots in order
        return torch.from_numpy(offn.bf16_round(acc + layer.shared_output(x.double().numpy())))

    return Steps(route=route, experts=experts, shared=shared)


def _rank_main(rank, world, port, shape_args, skew, out_q):
    import torch.distributed as dist
    from int4_quantized_expert_b200.ep import ExpertParallelLayer
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shape = synth.LayerShape(*shape_args)
        layer = oracle_layer(shape)
        if skew:   # every token goes to experts of rank 0 only
            wr = torch.zeros(shape.E, shape.D, dtype=torch.bfloat16)
            wr[0] = 0.05
            wr[1] = 0.03
            layer.w_router = wr
        x = synth.tokens(100 + rank, shape.T, shape.D)   # each rank's own tokens
        ep = ExpertParallelLayer(shape.E, shape.k, shape.D, _oracle_steps(shape, layer, rank, shape.E // world))
        got = ep(x).numpy()
        ref = offn.moe_forward(layer, x)["out"]
        out_q.put((rank, got, ref))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("shape_args,skew", [
    (("ep1", 40, 256, 256, 4, 1, 256), False),
    (("ep2", 33, 256, 384, 4, 2, 256), False),
    (("ep_skew", 24, 256, 256, 4, 2, 256), True),
])
def test_two_ranks_match_the_one_process_layer(shape_args, skew):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, shape_args, skew, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, ref in results:
        diff = np.abs(got - ref)
        # the slots are summed in slot order, the oracle's layer in expert
        # order: in fp64 the two differ by ~1e-16, which can move a value
        # across a bf16 rounding boundary (one step) in rare cases
        assert (diff <= np.abs(ref) * 2.0 ** -7 + 1e-30).all(), rank
        assert (diff > 0).mean() < 0.01, rank
