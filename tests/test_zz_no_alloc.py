"""moe_ffn_forward_noalloc: the layer forward for callers that cannot
allocate device memory (and so cannot hand the library a workspace), run
through the C ABI and compared with the workspace entry point moe_ffn_forward.

Kept in its own file, collected after the other test files, so that a run
stopping at the first failure has already run everything else.  It builds its
own layers, so it passes alone in a fresh process as well.
"""
import ctypes

import pytest
import torch

import int4_quantized_expert_b200 as moe
import synth
from tests._layers import build

pytestmark = pytest.mark.gpu


def _noalloc(layer, x, out):
    return moe.lib().moe_ffn_forward_noalloc(ctypes.byref(layer.desc), x.data_ptr(), x.shape[0],
                                             out.data_ptr(), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("name", ["tiny", "scout_decode"])
def test_noalloc_matches_workspace_entry_point_twice(name):
    """The kernels are deterministic, so the no-alloc call must give exactly
    the bytes of the workspace call, on two calls in a row (the second finds
    the first call's leftovers in the shared scratch)."""
    b = build(synth.SHAPES[name])
    x = b.x.cuda()
    ref = b.gpu(x)                                   # moe_ffn_forward with a workspace
    assert b.gpu.device_status() == moe.Status.OK
    for _ in range(2):
        out = torch.full_like(x, float("nan"))
        assert _noalloc(b.gpu, x, out) == moe.Status.OK
        assert moe.lib().moe_ffn_noalloc_device_status(torch.cuda.current_stream().cuda_stream) == moe.Status.OK
        assert torch.equal(out, ref)


def test_noalloc_rejects_batches_beyond_its_scratch():
    b = build(synth.SHAPES["tiny"])
    T_big = 8192                                     # needs far more than 8 MiB of scratch
    assert b.gpu.workspace_bytes(T_big) > (8 << 20)
    x = torch.zeros(T_big, b.shape.D, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(x)
    assert _noalloc(b.gpu, x, out) == moe.Status.WORKSPACE_TOO_SMALL
    assert bool((out == 0).all())                   # nothing was launched
