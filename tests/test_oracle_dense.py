"""Pins for the oracle's dense SwiGLU layer (CPU only): a saturated gate that
reduces it to a plain product of matmuls, zero and scaling cases, and the
identity with the MoE layer's (separately pinned) shared expert."""
import numpy as np
import torch

import synth
from oracle import ffn as offn
from oracle.ffn import bf16_round


def _weights(D=128, F=256, seed=3):
    g, u, d = synth.shared_weights(seed, D, F)
    return g, u, d


def test_saturated_gate_is_a_product_of_matmuls():
    """With every gate pre-activation >= 40, silu(g) = g in fp64, so the layer
    is bf16( bf16((x Wg^T) * (x Wu^T)) Wd^T ): an operand swapped or transposed
    anywhere changes the result."""
    D, F = 128, 256
    rng = np.random.default_rng(7)
    x = bf16_round(rng.uniform(0.5, 1.0, (6, D)))
    wg = np.full((F, D), 0.5)                        # g = 0.5 * sum(x) >= 32 * ... > 40
    wu = bf16_round(rng.standard_normal((F, D)) * 0.02)
    wd = bf16_round(rng.standard_normal((D, F)) * 0.02)
    g = x @ wg.T
    assert g.min() >= 40
    want = bf16_round(bf16_round(g * (x @ wu.T)) @ wd.T)
    assert np.array_equal(offn.dense_forward(x, wg, wu, wd), want)


def test_zero_up_projection_gives_zero():
    g, u, d = _weights()
    x = synth.tokens(1, 5, 128)
    assert (offn.dense_forward(x, g, torch.zeros_like(u), d) == 0).all()


def test_power_of_two_scaling_of_the_down_projection():
    g, u, d = _weights()
    x = synth.tokens(2, 7, 128)
    a = offn.dense_forward(x, g, u, d)
    b = offn.dense_forward(x, g, u, d.float() * 4)
    assert np.array_equal(b, 4 * a)


def test_equals_the_moe_layers_shared_expert():
    g, u, d = _weights()
    x = synth.tokens(3, 9, 128)
    lay = offn.Layer("int4", 1, None, None, None, (g, u, d))
    assert np.array_equal(offn.dense_forward(x, g, u, d), bf16_round(lay.shared_output(x.float().numpy())))
