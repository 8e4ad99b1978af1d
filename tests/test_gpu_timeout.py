"""Failure detection without a GPU fault: every pipeline wait in the kernels
is bounded and reports to a device status word.  A lowered wait limit
(moe_set_wait_limit) makes the waits give up on their first miss, so a layer
call must end with MOE_ERR_TIMEOUT in its status word, its kernels must wind
down (their copies in flight drained, tensor memory freed) and return, and the
next call with the default limit must give the normal result again."""
import pytest
import torch

import int4_quantized_expert_b200 as moe
import synth
from tests._layers import build

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny", moe.PATH_DECODE),        # weight-streaming kernels
    ("tiny", moe.PATH_PREFILL),       # tcgen05 int4 / bf16 kernels
    ("fp8", moe.PATH_AUTO),           # tcgen05 e4m3 kernels
]


def _shape(name):
    if name == "fp8":
        return synth.LayerShape("fp8_tiny", 64, 256, 512, 8, 2, 256, "fp8")
    return synth.SHAPES[name]


@pytest.mark.parametrize("name,path", CASES)
def test_waits_time_out_then_the_next_call_recovers(name, path):
    b = build(_shape(name))
    b.gpu.set_path(path)
    x = b.x.cuda()
    ref = b.gpu(x).clone()
    assert b.gpu.device_status() == moe.Status.OK
    moe.set_wait_limit(1)
    try:
        b.gpu(x)
        assert b.gpu.device_status() == moe.Status.TIMEOUT
    finally:
        moe.set_wait_limit(0)
    out = b.gpu(x)
    assert b.gpu.device_status() == moe.Status.OK
    assert torch.equal(out, ref)


def test_noalloc_call_reports_its_timeout():
    b = build(synth.SHAPES["tiny"])
    x = b.x.cuda()
    ref = b.gpu(x).clone()
    moe.set_wait_limit(1)
    try:
        b.gpu.forward_noalloc(x)
        assert moe.noalloc_device_status() == moe.Status.TIMEOUT
    finally:
        moe.set_wait_limit(0)
    out = b.gpu.forward_noalloc(x)
    assert moe.noalloc_device_status() == moe.Status.OK
    assert torch.equal(out, ref)
