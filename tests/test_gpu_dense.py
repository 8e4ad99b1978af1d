"""The dense SwiGLU layer on the GPU vs the oracle (both paths, with and
without the RMSNorm prologue): max |gpu - oracle| <= 1e-2 * max |oracle|."""
import numpy as np
import pytest
import torch

import int4_quantized_expert_b200 as moe
import synth
from oracle import ffn as offn
from tests._layers import rel_err

pytestmark = pytest.mark.gpu

SHAPES = [(1, 256, 512), (16, 512, 1024), (37, 384, 640), (64, 256, 768), (300, 256, 512)]


@pytest.mark.parametrize("rms", [False, True])
@pytest.mark.parametrize("path", [moe.PATH_AUTO, moe.PATH_DECODE, moe.PATH_PREFILL])
@pytest.mark.parametrize("T,D,F", SHAPES)
def test_dense_layer(T, D, F, path, rms):
    g, u, d = synth.shared_weights(5, D, F)
    gamma = synth.rms_weight(5, D) if rms else None
    x = synth.tokens(5, T, D)
    layer = moe.DenseLayer(D=D, F=F, w_gate=g.cuda(), w_up=u.cuda(), w_down=d.cuda(), path=path, T_max=T,
                           rms_weight=None if gamma is None else gamma.cuda())
    out = layer(x.cuda())
    assert layer.device_status() == moe.Status.OK
    ref = offn.dense_forward(x, g, u, d, rms_weight=gamma)
    assert rel_err(out.float().cpu().numpy().astype(np.float64), ref) <= 1e-2


def test_dense_paths_agree_and_repeat():
    T, D, F = 48, 512, 1024
    g, u, d = (t.cuda() for t in synth.shared_weights(6, D, F))
    x = synth.tokens(6, T, D).cuda()
    a = moe.DenseLayer(D=D, F=F, w_gate=g, w_up=u, w_down=d, path=moe.PATH_DECODE, T_max=T)
    b = moe.DenseLayer(D=D, F=F, w_gate=g, w_up=u, w_down=d, path=moe.PATH_PREFILL, T_max=T)
    o1 = a(x).clone()
    assert torch.equal(o1, a(x))
    assert rel_err(b(x).float().cpu().numpy(), o1.float().cpu().numpy()) <= 1e-2
