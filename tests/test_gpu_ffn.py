"""The whole layer on the GPU vs the oracle:
max |gpu - oracle| <= 1e-2 * max |oracle| (bf16 output, fp32 accumulation)."""
import numpy as np
import pytest
import torch

import int4_quantized_expert_b200 as moe
import synth
from oracle import ffn as offn
from oracle import route as oroute
from tests._layers import build, covering_tokens, oracle_outputs, rel_err

pytestmark = pytest.mark.gpu

TOL = 1e-2


def _run(b, path=moe.PATH_AUTO, tokens=None):
    b.gpu.set_path(path)
    out = b.gpu(b.x.cuda())
    assert b.gpu.device_status() == moe.Status.OK
    got = out.float().cpu().numpy().astype(np.float64)
    ref = offn.moe_forward(b.oracle, b.x, tokens=tokens)
    sel = ref["tokens"]
    return got[sel], ref["out"]


@pytest.mark.parametrize("path", [moe.PATH_AUTO, moe.PATH_DECODE, moe.PATH_PREFILL])
def test_tiny(path):
    b = build(synth.SHAPES["tiny"])
    got, ref = _run(b, path)
    assert rel_err(got, ref) <= TOL


RAGGED = [
    (1, 256, 512, 512, 4, 1),        # one token
    (37, 384, 640, 384, 5, 2),       # ragged: 3 groups along D, token chunks + tail
    (16, 128, 256, 128, 1, 1),       # a single expert
    (50, 256, 384, 256, 6, 3),
    (16, 512, 1024, 768, 16, 1),
    (300, 256, 256, 128, 3, 2),      # more than one 256-token tile per expert
    (2100, 256, 256, 128, 8, 2),     # 4200 slots: bucketing over several CTAs
]


@pytest.mark.parametrize("path", [moe.PATH_DECODE, moe.PATH_PREFILL])
@pytest.mark.parametrize("T,D,F,Fs,E,k", RAGGED)
def test_ragged(T, D, F, Fs, E, k, path):
    b = build(synth.LayerShape("r", T, D, F, E, k, Fs))
    got, ref = _run(b, path)
    assert rel_err(got, ref) <= TOL


def test_all_tokens_on_one_expert_and_empty_experts():
    shape = synth.LayerShape("one", 40, 256, 512, 4, 1, 256)
    b = build(shape, margin=False)
    wr = torch.zeros(4, 256, dtype=torch.bfloat16)
    wr[2] = 0.02
    b.gpu.tensors[0].copy_(wr.cuda())
    b.oracle.w_router = wr
    b.x = torch.ones(40, 256, dtype=torch.bfloat16) * torch.linspace(0.5, 1.5, 40).to(torch.bfloat16)[:, None]
    for path in (moe.PATH_DECODE, moe.PATH_PREFILL):
        got, ref = _run(b, path)
        assert rel_err(got, ref) <= TOL


def test_repeat_calls_identical():
    b = build(synth.SHAPES["tiny"])
    o1 = b.gpu(b.x.cuda()).clone()
    o2 = b.gpu(b.x.cuda())
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("shape", [synth.LayerShape("k4", 600, 256, 384, 8, 4, 256),
                                   synth.LayerShape("fp8_k8", 512, 256, 512, 16, 8, 256, "fp8")],
                         ids=lambda s: s.name)
def test_repeat_calls_identical_k_slots(shape):
    """k > 1 on the tensor-core path: the last of a token's k down tiles to
    finish sums its slots, in slot order -- bit-identical outputs whichever
    tile is last, call after call."""
    b = build(shape)
    b.gpu.set_path(moe.PATH_PREFILL)
    x = b.x.cuda()
    o1 = b.gpu(x).clone()
    for _ in range(3):
        assert torch.equal(b.gpu(x), o1)
    got, ref = _run(b, moe.PATH_PREFILL)
    assert rel_err(got, ref) <= TOL


def test_host_buffers_match_device_call():
    b = build(synth.SHAPES["tiny"])
    dev = b.gpu(b.x.cuda()).cpu()
    xh = b.x.clone().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    b.gpu.forward_host(xh, oh)
    torch.cuda.synchronize()
    assert torch.equal(oh, dev)


@pytest.mark.slow
def test_scout_decode_full_size():
    """The decode workload at full size (T=16, D=5120, F=8192, 16 experts),
    every token checked against the oracle."""
    b = build(synth.SHAPES["scout_decode"])
    got, ref = _run(b)
    assert rel_err(got, ref) <= TOL


def _sampled(name, n_extra, seed=0):
    """The workload at full size through AUTO; checked on a covering sample:
    one token for every expert that some token chose, plus ``n_extra`` random
    tokens, against the oracle (evaluated by spawned processes)."""
    shape = synth.SHAPES[name]
    b = build(shape)
    ids = oroute.route(b.x, b.w_router, b.bias, shape.k)["ids"]
    tokens = covering_tokens(ids, shape.E, n_extra, seed)
    chosen = set(ids.reshape(-1).tolist())
    assert chosen == set(ids[tokens].reshape(-1).tolist())      # every used expert is checked
    b.gpu.set_path(moe.PATH_AUTO)
    out = b.gpu(b.x.cuda())
    assert b.gpu.device_status() == moe.Status.OK
    got = out.float().cpu().numpy().astype(np.float64)[tokens]
    ref = oracle_outputs(shape, b.x, tokens, ids, seed=0)
    return got, ref


@pytest.mark.slow
def test_scout_prefill_full_size_sampled():
    """The prefill workload at full size (T=8192) through the tensor-core
    path: a token of every expert plus 16 random ones."""
    got, ref = _sampled("scout_prefill", 16)
    assert rel_err(got, ref) <= TOL


@pytest.mark.slow
def test_skewed_full_size_sampled():
    """The Zipf-routed workload at full size (T=32768): a token of every
    expert, the 0.2 %-load tail included, plus 16 random ones."""
    got, ref = _sampled("skewed", 16, seed=1)
    assert rel_err(got, ref) <= TOL


def _decode_takes_groups(D, F, G):
    """The weight-streaming kernels take groups of 64 / 32 when a stage's
    scale box fits a row: K / G a multiple of 4 and at least the groups of a
    stage (256 K for gate/up, 512 K for down)."""
    return all((K // G) % 4 == 0 and K // G >= kst // G for K, kst in ((D, 256), (F, 512)))


@pytest.mark.parametrize("G", [64, 32])
@pytest.mark.parametrize("T,D,F,Fs,E,k", [(64, 256, 512, 512, 4, 1), (37, 384, 640, 384, 5, 2),
                                          (300, 256, 256, 128, 3, 2), (1, 256, 512, 512, 4, 1),
                                          (16, 1024, 1536, 512, 6, 1)])
def test_small_int4_groups(T, D, F, Fs, E, k, G):
    """int4 experts quantized in groups of 64 or 32 ("a smaller group_size"):
    AUTO, the tensor-core tiles and -- where the shape allows -- the
    weight-streaming kernels, whose MMAs then go one 32-K quarter at a time."""
    b = build(synth.LayerShape("g%d" % G, T, D, F, E, k, Fs), group_size=G)
    for path in (moe.PATH_AUTO, moe.PATH_PREFILL):
        got, ref = _run(b, path)
        assert rel_err(got, ref) <= TOL
    b.gpu.set_path(moe.PATH_DECODE)
    if _decode_takes_groups(D, F, G):
        got, ref = _run(b, moe.PATH_DECODE)
        assert rel_err(got, ref) <= TOL
    else:
        with pytest.raises(moe.MoEError):
            b.gpu(b.x.cuda())


@pytest.mark.parametrize("G", [64, 32])
def test_small_int4_groups_wide_range(G):
    """Groups of 64 / 32 on the weight-streaming path with token rows spanning
    30 binades (each group of x and h gets its own power of two)."""
    b = build(synth.LayerShape("wide%d" % G, 24, 512, 1024, 4, 1, 512), margin=False, group_size=G)
    b.x = _wide_range_tokens(b.shape, b.w_router, b.bias, seed=6)
    b.gpu.set_path(moe.PATH_DECODE)
    out = b.gpu(b.x.cuda())
    assert b.gpu.device_status() == moe.Status.OK
    got = out.float().cpu().numpy().astype(np.float64)
    ref = offn.moe_forward(b.oracle, b.x)["out"]
    row_err = np.abs(got - ref).max(axis=1) / np.abs(ref).max(axis=1)
    assert row_err.max() <= TOL, row_err.max()


FP8_SHAPES = [
    synth.LayerShape("fp8_tiny", 64, 256, 512, 8, 2, 256, "fp8"),
    synth.LayerShape("fp8_ragged", 37, 384, 640, 5, 3, 384, "fp8"),
    synth.LayerShape("fp8_one", 1, 256, 256, 4, 4, 128, "fp8"),
]


@pytest.mark.parametrize("shape", FP8_SHAPES, ids=lambda s: s.name)
def test_fp8_layers(shape):
    """e4m3 row-quantized experts (weights and every expert input), bf16
    shared expert, softmax over the top-k gates."""
    b = build(shape)
    got, ref = _run(b)
    assert rel_err(got, ref) <= TOL


@pytest.mark.slow
def test_maverick_fp8_full_size_sampled():
    """The Maverick-shaped FP8 layer at full size (T=4096, 128 experts,
    top-8): a covering sample that checks a token of each of the 128 experts."""
    got, ref = _sampled("maverick_fp8", 0, seed=2)
    assert rel_err(got, ref) <= TOL


def _wide_range_tokens(shape, w_router, bias, seed):
    """bf16 token rows whose elements span 30 binades (magnitudes 2^U(-20, 10),
    random signs), each row also scaled by 2^0, 2^-8 or 2^-16, so some rows --
    and every hidden activation h they produce -- are tiny.  Rows whose top-
    (k+1) logits are closer than 1e-4 of the row's largest logit are redrawn."""
    rng = np.random.default_rng(seed)
    x = np.empty((shape.T, shape.D), dtype=np.float64)
    todo = np.arange(shape.T)
    while todo.size:
        n = todo.size
        mag = np.exp2(rng.uniform(-20.0, 10.0, (n, shape.D)))
        sign = np.where(rng.random((n, shape.D)) < 0.5, -1.0, 1.0)
        row = np.exp2(-8.0 * rng.integers(0, 3, (n, 1)))
        x[todo] = torch.from_numpy(sign * mag * row).to(torch.bfloat16).double().numpy()
        lg = oroute.router_logits(x[todo], w_router, bias)
        m = min(shape.k + 1, shape.E)
        top = -np.sort(-lg, axis=1)[:, :m]
        ok = (np.diff(-top, axis=1) > 1e-4 * np.abs(lg).max(axis=1, keepdims=True)).all(axis=1)
        todo = todo[~ok]
    return torch.from_numpy(x).to(torch.bfloat16)


@pytest.mark.parametrize("path", [moe.PATH_DECODE, moe.PATH_PREFILL])
@pytest.mark.parametrize("T,D,F,Fs,E,k", [(48, 256, 512, 512, 4, 1), (37, 384, 640, 384, 5, 2)])
def test_wide_dynamic_range_rows(T, D, F, Fs, E, k, path):
    """Token rows spanning 30 binades, and rows 2^-16 smaller than others,
    through the weight-streaming path's scaled fp16 re-encoding of x and h
    (and the tensor-core path): every row within 1e-2 of its own largest
    oracle value."""
    b = build(synth.LayerShape("wide", T, D, F, E, k, Fs), margin=False)
    b.x = _wide_range_tokens(b.shape, b.w_router, b.bias, seed=5)
    b.gpu.set_path(path)
    out = b.gpu(b.x.cuda())
    assert b.gpu.device_status() == moe.Status.OK
    got = out.float().cpu().numpy().astype(np.float64)
    ref = offn.moe_forward(b.oracle, b.x)["out"]
    row_err = np.abs(got - ref).max(axis=1) / np.abs(ref).max(axis=1)
    assert row_err.max() <= TOL, row_err.max()
