"""RMSNorm on the GPU vs the oracle: the standalone kernel (moe_rmsnorm) and
the layer with the norm as its prologue."""
import numpy as np
import pytest
import torch

import int4_quantized_expert_b200 as moe
import synth
from oracle import ffn as offn
from oracle import norm as onorm
from tests._layers import build, rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,D", [(1, 128), (37, 384), (16, 5120), (300, 8192)])
@pytest.mark.parametrize("eps", [1e-5, 0.0])
def test_rmsnorm_matches_oracle(T, D, eps):
    """fp32 on the GPU, fp64 in the oracle, both rounded once to bf16: an
    element may differ by one bf16 step where the unrounded values straddle
    a rounding boundary; that happens rarely."""
    x = synth.tokens(21, T, D)
    gamma = synth.rms_weight(21, D)
    got = moe.rmsnorm(x.cuda(), gamma.cuda(), eps).float().cpu().numpy().astype(np.float64)
    ref = onorm.rmsnorm(x, gamma, eps)
    ulp = np.abs(ref) * 2.0 ** -7      # one bf16 step at the value's magnitude (upper bound)
    diff = np.abs(got - ref)
    assert (diff <= ulp + 1e-30).all()
    assert (diff > 0).mean() < 0.01


@pytest.mark.parametrize("path", [moe.PATH_DECODE, moe.PATH_PREFILL])
@pytest.mark.parametrize("shape", [synth.SHAPES["tiny"], synth.LayerShape("r", 37, 384, 640, 5, 2, 384),
                                   synth.LayerShape("ks4", 16, 1024, 512, 4, 1, 512),
                                   synth.LayerShape("ks8", 20, 5120, 1024, 8, 2, 512)],
                         ids=["tiny", "ragged", "split4", "split8"])
def test_layer_with_rmsnorm(shape, path):
    """The router normalizes x itself (no launch of its own): with D = 1024
    and 5120 at decode sizes its K range is split over a cluster of 4 / 8
    CTAs that exchange the rows' partial sums of squares."""
    b = build(shape, rms=True)
    b.gpu.set_path(path)
    out = b.gpu(b.x.cuda())
    assert b.gpu.device_status() == moe.Status.OK
    ref = offn.moe_forward(b.oracle, b.x)["out"]
    assert rel_err(out.float().cpu().numpy().astype(np.float64), ref) <= 1e-2


def test_fp8_layer_with_rmsnorm():
    b = build(synth.LayerShape("fp8_rms", 64, 256, 512, 8, 2, 256, "fp8"), rms=True)
    out = b.gpu(b.x.cuda())
    ref = offn.moe_forward(b.oracle, b.x)["out"]
    assert rel_err(out.float().cpu().numpy().astype(np.float64), ref) <= 1e-2


def test_layer_norm_is_not_a_launch():
    b = build(synth.SHAPES["tiny"], rms=True)
    for path in (moe.PATH_DECODE, moe.PATH_PREFILL):
        b.gpu.set_path(path)
        assert "rmsnorm" not in b.gpu.launch_names(64)
