"""Pins for the oracle's RMSNorm (CPU only): hand-worked rows, the closed
forms that follow from the definition, and the wiring into the layer."""
import os

import numpy as np
import pytest
import torch

import synth
from oracle import ffn as offn
from oracle import norm
from oracle.ffn import bf16_round

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows():
    out = []
    with open(os.path.join(GOLDEN, "rmsnorm_worked_example.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                v = [float(t) for t in line.split()]
                out.append((v[0], v[1:5], v[5:9], v[9:13]))
    return out


@pytest.mark.parametrize("eps,x,g,want", _rows())
def test_worked_rows(eps, x, g, want):
    got = norm.rmsnorm(np.array([x]), np.array(g), eps)
    assert got[0].tolist() == want


def test_power_of_two_scale_invariance():
    """With eps = 0, RMSNorm(2^k x) = RMSNorm(x) exactly: the root scales by
    2^k and every step is exact or rounds the same value."""
    rng = np.random.default_rng(4)
    x = bf16_round(rng.standard_normal((5, 256)))
    g = bf16_round(1 + 0.1 * rng.standard_normal(256))
    base = norm.rmsnorm(x, g, 0.0)
    for k in (-3, 1, 6):
        assert np.array_equal(norm.rmsnorm(x * 2.0 ** k, g, 0.0), base)


def test_unit_root_mean_square():
    """gamma = 1: the output's mean square is ms / (ms + eps) up to the bf16
    rounding of each element (relative 2^-8)."""
    rng = np.random.default_rng(5)
    x = bf16_round(rng.standard_normal((6, 512)) * 3)
    eps = 0.5
    y = norm.rmsnorm(x, np.ones(512), eps)
    ms = (x * x).mean(axis=1)
    assert np.allclose((y * y).mean(axis=1), ms / (ms + eps), rtol=2 * 2.0 ** -8)


def test_sign_of_a_constant_row():
    """A constant row c with eps = 0 normalizes to sign(c) * gamma."""
    g = np.array([0.5, -2.0, 1.5, 3.0] * 32)
    for c in (-7.0, 0.25, 1e3):
        assert np.array_equal(norm.rmsnorm(np.full((1, 128), c), g, 0.0)[0], np.sign(c) * g)


def test_layer_applies_the_norm_first():
    """The layer with an RMSNorm equals the same layer on RMSNorm(x)."""
    shape = synth.SHAPES["tiny"]
    rng = np.random.default_rng(6)
    gamma = torch.from_numpy(bf16_round(1 + 0.1 * rng.standard_normal(shape.D)).astype(np.float32)).to(torch.bfloat16)
    wr = synth.router_weight(0, shape.E, shape.D)
    sh = synth.shared_weights(0, shape.D, shape.F_shared)
    from oracle import quant as oq
    experts = {e: tuple(oq.int4_row_quantize(w) for w in synth.expert_weights(0, e, shape.D, shape.F))
               for e in range(shape.E)}
    x = synth.tokens(0, 8, shape.D)
    with_norm = offn.Layer("int4", 1, wr, None, experts.__getitem__, sh, rms_weight=gamma, rms_eps=1e-5)
    plain = offn.Layer("int4", 1, wr, None, experts.__getitem__, sh)
    xn = norm.rmsnorm(x, gamma, 1e-5)
    a = offn.moe_forward(with_norm, x)
    b = offn.moe_forward(plain, torch.from_numpy(xn.astype(np.float32)).to(torch.bfloat16))
    assert np.array_equal(a["out"], b["out"]) and np.array_equal(a["ids"], b["ids"])
