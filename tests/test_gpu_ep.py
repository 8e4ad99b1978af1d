"""The compute steps of the expert-parallel layer on one GPU: the routed
experts on rows with given experts (moe_expert_ffn_forward) and the shared
expert with the combine of given routed outputs (moe_shared_ffn_combine).
With one rank the expert-parallel layer (its bookkeeping is tested over two
gloo ranks on CPU) runs exactly the one-GPU layer's arithmetic."""
import numpy as np
import pytest
import torch

import int4_quantized_expert_b200 as moe
import synth
from int4_quantized_expert_b200.ep import ExpertParallelLayer, library_steps
from oracle import ffn as offn
from tests._layers import build, rel_err

pytestmark = pytest.mark.gpu

SHAPES = [
    synth.SHAPES["tiny"],
    synth.LayerShape("ep_k2", 37, 384, 640, 5, 2, 384),
    synth.LayerShape("ep_fp8", 64, 256, 512, 8, 2, 256, "fp8"),
]


@pytest.mark.parametrize("path", [moe.PATH_DECODE, moe.PATH_PREFILL])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
def test_one_rank_equals_the_layer(shape, path):
    if shape.fmt == "fp8" and path == moe.PATH_DECODE:
        pytest.skip("e4m3 layers run on the tensor-core tiles only")
    b = build(shape)
    b.gpu.set_path(path)
    x = b.x.cuda()
    ref = b.gpu(x)
    assert b.gpu.device_status() == moe.Status.OK
    bias = None if b.bias is None else torch.from_numpy(b.bias).cuda()
    ep = ExpertParallelLayer(shape.E, shape.k, shape.D, library_steps(b.w_router.cuda(), bias, shape.k, b.gpu))
    got = ep(x)
    assert b.gpu.last_call_status() == moe.Status.OK
    if path == moe.PATH_DECODE or shape.k > 1:
        assert torch.equal(got, ref)       # the same kernels, the same sums
    else:
        # with one slot per token the one-GPU tensor-core layer adds gate * y
        # to the shared expert in one fused multiply-add; here y is rounded to
        # fp32 first, so a value may move by one bf16 step
        diff = (got.float() - ref.float()).abs()
        assert (diff <= ref.float().abs() * 2.0 ** -7 + 1e-30).all()
    ref_o = offn.moe_forward(b.oracle, b.x)["out"]
    assert rel_err(got.float().cpu().numpy().astype(np.float64), ref_o) <= 1e-2


def test_experts_on_given_rows_match_the_oracle():
    shape = synth.LayerShape("ep_rows", 24, 256, 512, 6, 1, 256)
    b = build(shape)
    g = torch.Generator().manual_seed(3)
    n = 40
    rows = synth.tokens(31, n, shape.D)
    ids = torch.randint(0, shape.E, (n,), generator=g, dtype=torch.int32)
    gates = torch.rand(n, generator=g, dtype=torch.float32) + 0.25
    y = b.gpu.expert_forward(rows.cuda(), ids.cuda(), gates.cuda())
    assert b.gpu.last_call_status() == moe.Status.OK
    xr = rows.double().numpy()
    ref = np.stack([gates[r].item() * b.oracle.expert_output(int(ids[r]), xr[r:r + 1])[0] for r in range(n)])
    assert rel_err(y.double().cpu().numpy(), ref) <= 1e-2


def test_out_of_range_expert_id_is_reported():
    b = build(synth.SHAPES["tiny"])
    rows = synth.tokens(32, 8, 256).cuda()
    ids = torch.tensor([0, 1, 2, 3, 4, 0, 1, 2], dtype=torch.int32, device="cuda")   # 4 >= E
    gates = torch.ones(8, dtype=torch.float32, device="cuda")
    b.gpu.expert_forward(rows, ids, gates)
    assert b.gpu.last_call_status() == moe.Status.INVALID_ARG
    b.gpu.expert_forward(rows, ids.clamp(max=3), gates)      # the next call is clean again
    assert b.gpu.last_call_status() == moe.Status.OK
