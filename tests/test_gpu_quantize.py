"""GPU quantizers vs the oracle: int4 codes/scales and e4m3 bytes/scales must be
bit-exact (both sides take every rounding decision in fp32)."""
import math

import numpy as np
import pytest
import torch

import int4_quantized_expert_b200 as moe
import synth
from oracle import quant as oq

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols", [(1, 128), (3, 384), (37, 512), (256, 5120), (130, 8192)])
def test_int4_bit_exact(rows, cols):
    g = synth.stream(11, rows * 7 + cols)
    w = (g.standard_normal((rows, cols), dtype=np.float32) * np.float32(0.02))
    w[0, :128] = 0.0                                      # all-zero group
    if rows > 2:
        w[1, :128] = np.linspace(-1, 1, 128, dtype=np.float32)   # exact .5 quotients
        w[2, 5] = 1e4                                     # one huge value
    codes, scales = moe.quantize_int4(torch.from_numpy(w).cuda())
    q_ref, s_ref = oq.int4_row_quantize(w)
    assert np.array_equal(scales.cpu().numpy(), s_ref)
    assert np.array_equal(codes.cpu().numpy(), oq.pack_int4(q_ref))


@pytest.mark.parametrize("G", [64, 32])
@pytest.mark.parametrize("rows,cols", [(1, 128), (37, 512), (130, 5120)])
def test_int4_small_groups_bit_exact(rows, cols, G):
    """Groups of 64 and 32 (the smaller group_size the lshu.cn page names as
    the int4 path's next step): codes and scales bit-exact."""
    g = synth.stream(13, rows * 7 + cols + G)
    w = (g.standard_normal((rows, cols), dtype=np.float32) * np.float32(0.02))
    w[0, :G] = 0.0                                        # all-zero group
    w[0, G:2 * G] = np.linspace(-1, 1, G, dtype=np.float32)
    codes, scales = moe.quantize_int4(torch.from_numpy(w).cuda(), group_size=G)
    q_ref, s_ref = oq.int4_row_quantize(w, group_size=G)
    assert scales.shape == (rows, cols // G)
    assert np.array_equal(scales.cpu().numpy(), s_ref)
    assert np.array_equal(codes.cpu().numpy(), oq.pack_int4(q_ref))


def test_int4_small_groups_worked_example_on_gpu():
    """The hand-worked row of tests/golden/int4_small_groups_worked_example.txt
    (padded to 128 columns with zeros) on the GPU quantizer."""
    row = np.zeros((1, 128), np.float32)
    idx = [0, 1, 3, 5, 33, 34, 40, 41, 42, 63]
    row[0, idx] = [0.3125, 0.4375, 1.0, -0.1875, 0.15625, 0.21875, -0.5, 0.46875, -0.03125, 0.09375]
    expect = {32: [2, 4, 7, -2, 2, 4, -8, 7, 0, 2], 64: [2, 4, 7, -2, 1, 2, -4, 4, 0, 1]}
    for G in (32, 64):
        codes, scales = moe.quantize_int4(torch.from_numpy(row).cuda(), group_size=G)
        q = oq.unpack_int4(codes.cpu().numpy())
        assert q[0, idx].tolist() == expect[G]
        assert scales.cpu().numpy()[0, :64 // G].tolist() == ([0.125, 0.0625] if G == 32 else [0.125])


def _near_tie_groups(n_groups, seed):
    """Groups whose quotients w / s sit on or within a few ulps of a
    half-integer (the places where a quotient one ulp off would round the
    other way), with scales that are not powers of two."""
    g = synth.stream(seed, 99)
    w = np.zeros((n_groups, 128), np.float32)
    for i in range(n_groups):
        m = np.float32(g.uniform(0.01, 0.05))
        s = np.float32(np.maximum(m, np.float32(1e-6)) / np.float32(8.0))
        k = g.integers(-8, 8, 127).astype(np.float32) + np.float32(0.5)   # half-integers
        v = (k * s).astype(np.float32)                                     # quotients near k + 1/2
        steps = g.integers(-3, 4, 127)
        v = np.array([np.float32(x) for x in v])
        for j in range(127):                                               # move a few ulps either way
            for _ in range(abs(int(steps[j]))):
                v[j] = np.nextafter(v[j], np.float32(np.inf if steps[j] > 0 else -np.inf), dtype=np.float32)
        v = np.clip(v, -m, m)
        w[i, 0] = m                                                        # the group maximum
        w[i, 1:] = v
    return w


def test_int4_bit_exact_near_ties():
    """Quotients on and a few ulps around half-integers: the GPU's rounding
    decisions must be those of the IEEE quotient, as in the oracle."""
    w = _near_tie_groups(512, 5)
    codes, scales = moe.quantize_int4(torch.from_numpy(w).cuda())
    q_ref, s_ref = oq.int4_row_quantize(w)
    assert np.array_equal(scales.cpu().numpy(), s_ref)
    assert np.array_equal(codes.cpu().numpy(), oq.pack_int4(q_ref))


def test_int4_worked_group_on_gpu():
    group = np.zeros((1, 128), np.float32)
    group[0, :6] = [0.3125, 0.4375, -0.0625, 1.0, -1.0, 0.1875]
    codes, scales = moe.quantize_int4(torch.from_numpy(group).cuda())
    q = oq.unpack_int4(codes.cpu().numpy())
    assert q[0, :6].tolist() == [2, 4, 0, 7, -8, 2] and scales.item() == 0.125


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,cols,nv,ub", [(1, 8, 1, math.inf), (33, 5120, 30, math.inf),
                                               (64, 8192, 64, 2.0), (5, 40, 3, 0.5), (7, 3000, 7, math.inf),
                                               (3, 8200, 2, math.inf)])
def test_fp8_rows_bit_exact(dtype, rows, cols, nv, ub):
    g = synth.stream(12, rows * 3 + cols)
    x = g.standard_normal((rows, cols), dtype=np.float32) * np.float32(3.0)
    x[0, :4] = [0.0, -1e-9, 1e-30, -0.0]              # signed zero and underflow
    xt = torch.from_numpy(x).to(dtype)
    q, s = moe.quantize_fp8_rows(xt.cuda(), num_valid_rows=nv, scale_ub=ub)
    q_ref, s_ref = oq.fp8_row_quantize(xt.float().numpy(), num_valid_rows=nv, scale_ub=ub)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def _fp8_near_ties(rows, cols, seed):
    """Rows whose quotients x / s sit on or within a few ulps of the midpoint
    between two e4m3 values (where the rounding decision is taken), across
    the whole e4m3 range including the subnormals."""
    g = synth.stream(seed, 77)
    pos = oq.E4M3_VALUES[:0x7F]
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)     # 4 significant bits: exact in fp32
    x = np.zeros((rows, cols), np.float32)
    for r in range(rows):
        m = np.float32(g.uniform(0.5, 4.0))
        s = np.float32(m / np.float32(448.0))
        v = (g.choice(mids, cols - 1) * np.where(g.integers(0, 2, cols - 1) == 1, 1, -1)).astype(np.float32)
        v = (v * s).astype(np.float32)
        steps = g.integers(-3, 4, cols - 1)
        for j in range(cols - 1):
            for _ in range(abs(int(steps[j]))):
                v[j] = np.nextafter(v[j], np.float32(np.inf if steps[j] > 0 else -np.inf), dtype=np.float32)
        x[r, 0] = m                                              # the row maximum
        x[r, 1:] = np.clip(v, -m, m)
    return x


@pytest.mark.parametrize("cols", [1024, 8192])
def test_fp8_rows_bit_exact_near_ties(cols):
    """e4m3 codes of quotients on and around the format's rounding midpoints:
    the GPU must take the IEEE quotient's rounding decisions, as the oracle."""
    x = _fp8_near_ties(16, cols, 9)
    q, s = moe.quantize_fp8_rows(torch.from_numpy(x).cuda())
    q_ref, s_ref = oq.fp8_row_quantize(x)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.slow
def test_int4_full_size_sampled_experts():
    """int4_row_quantize of a 16-expert Scout-shaped layer at full size (one
    launch over all 2.01 G weights, as timed standalone), checked on sampled
    experts' down projections and gate rows."""
    shape = synth.SHAPES["skewed"]
    E, D, F = shape.E, shape.D, shape.F
    w = torch.empty(E * 3, F * D, dtype=torch.float32, device="cuda")   # 8.05 GB
    for e, g, u, d in synth.iter_expert_weights(0, range(E), D, F):
        w[3 * e].copy_(torch.from_numpy(g).view(-1))
        w[3 * e + 1].copy_(torch.from_numpy(u).view(-1))
        w[3 * e + 2].copy_(torch.from_numpy(d).view(-1))
    rows = E * 3 * F          # gate/up rows have K = D; down rows K = F differ, so view by [rows, D]
    codes, scales = moe.quantize_int4(w.view(-1, D))
    del w
    for e in (0, 7, 15):
        g, u, d = synth.expert_weights(0, e, D, F)
        for which, mat in ((0, g), (2, d)):
            q_ref, s_ref = oq.int4_row_quantize(mat.reshape(-1, D))
            n = mat.size // D
            base = (3 * e + which) * n
            assert np.array_equal(scales[base:base + n].cpu().numpy(), s_ref)
            assert np.array_equal(codes[base:base + n].cpu().numpy(), oq.pack_int4(q_ref))
