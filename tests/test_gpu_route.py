"""GPU routing vs the oracle: ids, counts, offsets and the permutation are
bit-exact on inputs whose top-(k+1) logits are more than 1e-3 apart; gates
agree to within the error of fp32 logits (relative bound below)."""
import numpy as np
import pytest
import torch

import int4_quantized_expert_b200 as moe
import synth
from oracle import route as oroute
from tests._layers import margin_tokens

pytestmark = pytest.mark.gpu

# Gates: the GPU sums each logit in fp32, the oracle in fp64.  A gate's
# relative error is at most its logits' absolute error for the sigmoid
# (d ln sigma = (1 - sigma) dl) and twice it for a softmax (d ln g_j = dl_j -
# sum_i g_i dl_i), plus a few ulps of expf.  The fp32 running sum of a logit
# takes about D / 16 roundings (16 products per MMA step), each at most half
# an ulp of a value below ~10 (4.8e-7); as independent errors they come to
# about sqrt(D / 16) * 4.8e-7, ~9e-6 for D = 5120 at worst, typically a few
# times less.  Measured on a B200 at the workloads' full sizes: at most
# 2.4e-6 relative (Maverick, top-8 softmax), 8.3e-7 absolute.
GATE_RTOL = 1e-5


def _check(shape, seed=0):
    wr = synth.router_weight(seed, shape.E, shape.D)
    bias = synth.router_bias(shape)
    x = margin_tokens(shape, wr, bias, seed)
    bt = None if bias is None else torch.from_numpy(bias).cuda()
    r = moe.route(x.cuda(), wr.cuda(), bt, shape.k)
    ref = oroute.route(x, wr, bias, shape.k)
    assert np.array_equal(r["ids"].cpu().numpy(), ref["ids"])
    assert np.array_equal(r["counts"].cpu().numpy(), ref["counts"])
    assert np.array_equal(r["offsets"].cpu().numpy(), ref["offsets"])
    assert np.array_equal(r["perm"].cpu().numpy(), ref["perm"])
    g = r["gates"].cpu().numpy().astype(np.float64)
    assert (np.abs(g - ref["gates"]) / ref["gates"]).max() <= GATE_RTOL
    if shape.k > 1:
        assert np.allclose(g.sum(axis=1), 1.0, atol=1e-5)
    return ref


@pytest.mark.parametrize("name", ["tiny", "scout_decode", "scout_prefill", "maverick_fp8", "skewed"])
def test_route_workloads(name):
    ref = _check(synth.SHAPES[name])
    if name == "skewed":
        c = ref["counts"] / ref["counts"].sum()
        assert c[0] > 0.4 and (np.diff(c[:6]) < 0).all()      # Zipf-like load


@pytest.mark.parametrize("T,D,E,k", [(1, 128, 4, 1), (37, 384, 5, 2), (65, 256, 256, 8),
                                     (1000, 128, 3, 3), (2049, 256, 64, 4), (130, 640, 200, 1)])
def test_route_ragged(T, D, E, k):
    _check(synth.LayerShape("r", T, D, 128, E, k, 128))


@pytest.mark.parametrize("T,D,E,k", [(16384, 128, 256, 8), (40000, 128, 7, 2)])
def test_route_many_bucket_blocks(T, D, E, k):
    """More than 32 blocks of 2048 slots (131072 and 80000 slots): the
    multi-CTA bucketing's per-expert scans carry across groups of 32 blocks,
    and with 256 experts the expert scans span eight warp passes."""
    _check(synth.LayerShape("r", T, D, 128, E, k, 128))


def test_route_all_tokens_on_one_expert():
    T, D, E = 300, 256, 8
    wr = torch.zeros(E, D, dtype=torch.bfloat16)
    wr[3] = 0.01
    wr[5] = -0.01
    x = torch.ones(T, D, dtype=torch.bfloat16)
    r = moe.route(x.cuda(), wr.cuda(), None, 2)
    ids = r["ids"].cpu().numpy()
    assert (ids[:, 0] == 3).all()
    # the remaining experts tie at 0: the lowest index wins
    assert (ids[:, 1] == 0).all()
    assert r["counts"].cpu().tolist() == [T, 0, 0, T, 0, 0, 0, 0]
    assert r["perm"].cpu().numpy()[:T].tolist() == list(range(1, 2 * T, 2))
