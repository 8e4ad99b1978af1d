"""Pins for the oracle's SwiGLU experts and the whole layer (CPU only).

Closed forms use permutation-matrix weights, so a transposed operand, a
dropped factor or a wrong sign changes the answer; the brute-force dense
evaluation pins the sparse bookkeeping (bucketing, gates, scatter-add).
"""
import numpy as np
import torch

import synth
from oracle import ffn, quant, route


def test_bf16_round_matches_library_cast():
    rng = np.random.default_rng(10)
    v = (rng.standard_normal(20000) * 10.0 ** rng.integers(-5, 5, 20000)).astype(np.float32)
    ours = ffn.bf16_round(v.astype(np.float64))
    lib = torch.from_numpy(v).to(torch.bfloat16).double().numpy()
    assert (ours == lib).all()
    # ties to even and carries
    assert ffn.bf16_round(1 + 2.0 ** -8) == 1.0
    assert ffn.bf16_round(1 + 3 * 2.0 ** -8) == 1 + 2.0 ** -6
    assert ffn.bf16_round(2 - 2.0 ** -9) == 2.0


def test_silu_closed_forms():
    assert ffn.silu(np.array([0.0]))[0] == 0.0
    assert abs(ffn.silu(np.array([1.0]))[0] - 1 / (1 + np.exp(-1.0))) < 1e-16
    big = ffn.silu(np.array([50.0, -50.0, -1000.0]))
    assert abs(big[0] - 50.0) < 1e-15 and abs(big[1]) < 1e-19 and big[2] == 0.0


def _perm_matrix(n_out, n_in, perm, value):
    w = np.zeros((n_out, n_in), np.float32)
    w[np.arange(n_out), perm] = value
    return w


def _int4_perm_expert(D, F, rng):
    """Weights -P (gate), -0.5 P (up), -P (down): each nonzero is its group's
    largest magnitude and negative, so int4 stores it exactly (code -8)."""
    pg = rng.integers(0, D, F)
    pu = rng.integers(0, D, F)
    pd = rng.integers(0, F, D)
    wg = _perm_matrix(F, D, pg, -1.0)
    wu = _perm_matrix(F, D, pu, -0.5)
    wd = _perm_matrix(D, F, pd, -1.0)
    return (wg, wu, wd), (pg, pu, pd)


def _closed_form_expert(x, pg, pu, pd):
    """y[d] = -h[pd[d]], h[n] = bf16(silu(-x[pg[n]]) * (-0.5 x[pu[n]]))."""
    g = -x[:, pg]
    u = -0.5 * x[:, pu]
    h = ffn.bf16_round(g / (1 + np.exp(-g)) * u)
    return -h[:, pd]


def test_int4_expert_closed_form():
    rng = np.random.default_rng(11)
    D, F = 256, 384
    (wg, wu, wd), (pg, pu, pd) = _int4_perm_expert(D, F, rng)
    stored = tuple(quant.int4_row_quantize(w) for w in (wg, wu, wd))
    for (q, s), w in zip(stored, (wg, wu, wd)):
        assert (quant.dequant_int4(q, s) == w).all()      # exact storage
    x = synth.tokens(0, 5, D).double().numpy()
    lay = ffn.Layer("int4", 1, np.zeros((1, D)), None, lambda e: stored, shared=None)
    y = lay.expert_output(0, x)
    assert (y == _closed_form_expert(x, pg, pu, pd)).all()


def test_fp8_expert_closed_form():
    rng = np.random.default_rng(12)
    D, F = 64, 96
    (wg, wu, wd), (pg, pu, pd) = _int4_perm_expert(D, F, rng)
    stored = tuple(quant.fp8_row_quantize(w) for w in (wg, wu, wd))
    x = synth.tokens(1, 3, D).float().numpy()
    lay = ffn.Layer("fp8", 1, np.zeros((1, D)), None, lambda e: stored, shared=None)
    y = lay.expert_output(0, x.astype(np.float64))
    # closed form: the weights' row scales and codes are exact (-448 * s),
    # the activations pass through the pinned row quantizer.
    sw = [s for _, s in stored]
    xq, sx = quant.fp8_row_quantize(x)
    xh = quant.dequant_fp8_rows(xq, sx)
    g = xh[:, pg] * (-448.0 * sw[0].astype(np.float64))[None, :]
    u = xh[:, pu] * (-448.0 * sw[1].astype(np.float64))[None, :]
    h = ffn.bf16_round(g / (1 + np.exp(-g)) * u)
    hq, sh = quant.fp8_row_quantize(h.astype(np.float32))
    hh = quant.dequant_fp8_rows(hq, sh)
    want = hh[:, pd] * (-448.0 * sw[2].astype(np.float64))[None, :]
    assert np.allclose(y, want, rtol=1e-12, atol=1e-15)
    # the fp8 path really differs from the exact product (activation rounding)
    exact = _closed_form_expert(x.astype(np.float64), pg, pu, pd)
    assert not np.array_equal(y, exact) and np.allclose(y, exact, rtol=0.15, atol=0.05)


def _tiny_layer(E, k, D=256, F=256, Fs=256, seed=0, fmt="int4", zero_expert=None, skew=False):
    wr = synth.router_weight(seed, E, D)
    bias = np.linspace(0.5, -0.5, E).astype(np.float32) if skew else None
    experts = {}
    for e in range(E):
        g, u, d = synth.expert_weights(seed, e, D, F)
        if e == zero_expert:
            g, u, d = (np.zeros_like(a) for a in (g, u, d))
        if fmt == "int4":
            experts[e] = tuple(quant.int4_row_quantize(w) for w in (g, u, d))
        else:
            experts[e] = tuple(quant.fp8_row_quantize(w) for w in (g, u, d))
    shared = synth.shared_weights(seed, D, Fs)
    return ffn.Layer(fmt, k, wr, bias, experts.__getitem__, shared)


def _margin_tokens(layer, T, D, seed=0):
    def accept(x):
        return route.topk_margin_ok(route.router_logits(x, layer.w_router, layer.bias), layer.k)
    return synth.tokens(seed, T, D, accept=accept)


def test_dense_equals_sparse():
    for E, k, fmt, skew in [(4, 1, "int4", False), (6, 2, "int4", True), (5, 3, "fp8", False)]:
        lay = _tiny_layer(E, k, fmt=fmt, skew=skew)
        x = _margin_tokens(lay, 24, 256)
        sparse = ffn.moe_forward(lay, x)["out"]
        dense = ffn.moe_forward_dense(lay, x, E)
        assert np.array_equal(sparse, dense) or np.allclose(sparse, dense, rtol=2 ** -7, atol=0)
        # bf16 outputs may differ by at most one rounding step where the fp64
        # sums differ in their last bits; almost all must be identical
        assert (sparse == dense).mean() > 0.999


def test_token_subset_matches_full():
    lay = _tiny_layer(4, 2)
    x = _margin_tokens(lay, 16, 256)
    full = ffn.moe_forward(lay, x)["out"]
    sub = ffn.moe_forward(lay, x, tokens=[3, 0, 15])["out"]
    assert np.array_equal(sub, full[[3, 0, 15]])


def test_single_expert_reduces_to_gated_ffn_plus_shared():
    lay = _tiny_layer(1, 1)
    x = synth.tokens(3, 8, 256)
    r = ffn.moe_forward(lay, x)
    xf = x.double().numpy()
    l = xf @ lay.w_router.double().numpy().T
    y = lay.expert_output(0, xf)
    want = ffn.bf16_round(1 / (1 + np.exp(-l)) * y + lay.shared_output(xf))
    assert (r["ids"] == 0).all() and np.array_equal(r["out"], want)


def test_zero_expert_gives_shared_only():
    lay = _tiny_layer(2, 1, zero_expert=0)
    lay.w_router = torch.tensor(np.stack([np.ones(256), -np.ones(256)]) * 0.01,
                                dtype=torch.bfloat16)
    x = torch.ones(4, 256, dtype=torch.bfloat16)          # every token picks expert 0
    r = ffn.moe_forward(lay, x)
    assert (r["ids"] == 0).all()
    assert np.array_equal(r["out"], ffn.bf16_round(lay.shared_output(x.double().numpy())))


def test_shared_expert_closed_form():
    rng = np.random.default_rng(13)
    D, F = 128, 256
    (wg, wu, wd), (pg, pu, pd) = _int4_perm_expert(D, F, rng)
    lay = ffn.Layer("int4", 1, np.zeros((1, D)), None, None,
                    shared=tuple(torch.from_numpy(w).to(torch.bfloat16) for w in (wg, wu, wd)))
    x = synth.tokens(4, 6, D).double().numpy()
    assert np.array_equal(lay.shared_output(x), _closed_form_expert(x, pg, pu, pd))
