"""Pins for the oracle's quantizers (CPU only).

int4 groups: a hand-worked example, brute-force nearest code, invariants.
FP8 e4m3: the format's defining values, the library conversion as a special
case, saturation, and the row-quantization invariants.
"""
import os

import numpy as np
import pytest
import torch

from oracle import quant

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load_worked_example():
    idx, w, q = [], [], []
    scale = None
    with open(os.path.join(GOLDEN, "int4_group_worked_example.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            parts = line.split()
            if parts[0] == "scale":
                scale = float(parts[1])
                continue
            idx.append(int(parts[0]))
            w.append(float(parts[1]))
            q.append(int(parts[3]))
    return idx, w, q, scale


def test_int4_worked_example():
    idx, w, q, scale = _load_worked_example()
    group = np.zeros(128, np.float32)
    group[idx] = w
    codes, scales = quant.int4_row_quantize(group[None, :])
    assert scales.shape == (1, 1) and scales[0, 0] == np.float32(scale)
    assert codes[0, idx].tolist() == q
    rest = np.setdiff1d(np.arange(128), idx)
    assert (codes[0, rest] == 0).all()


def _load_small_groups_example():
    idx, w, q32, q64, sc = [], [], [], [], {}
    with open(os.path.join(GOLDEN, "int4_small_groups_worked_example.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            parts = line.split()
            if parts[0].startswith("scales"):
                sc[int(parts[0][6:])] = [float(v) for v in parts[1:]]
                continue
            idx.append(int(parts[0]))
            w.append(float(parts[1]))
            q32.append(int(parts[2]))
            q64.append(int(parts[3]))
    return idx, w, {32: q32, 64: q64}, sc


@pytest.mark.parametrize("G", [32, 64])
def test_int4_small_groups_worked_example(G):
    idx, w, q, sc = _load_small_groups_example()
    row = np.zeros(64, np.float32)
    row[idx] = w
    codes, scales = quant.int4_row_quantize(row[None, :], group_size=G)
    assert scales.shape == (1, 64 // G)
    assert scales[0].tolist() == sc[G]
    assert codes[0, idx].tolist() == q[G]
    rest = np.setdiff1d(np.arange(64), idx)
    assert (codes[0, rest] == 0).all()
    # dequantization repeats each group's scale over exactly its G values
    wh = quant.dequant_int4(codes, scales, group_size=G)
    assert wh[0, 40] == q[G][idx.index(40)] * sc[G][40 // G]


@pytest.mark.parametrize("G", [128, 64, 32])
def test_int4_brute_force_nearest_code(G):
    """q must be the code in [-8, 7] nearest to fl32(w / s), ties to even."""
    rng = np.random.default_rng(1)
    w = (rng.standard_normal((6, 256)) * rng.uniform(1e-4, 3, (6, 1))).astype(np.float32)
    w[0, :128] = 0.0                         # an all-zero group
    w[1, 5] = 7.5 * np.abs(w[1, :128]).max() / 8  # exactly x.5 quotients occur below
    q, s = quant.int4_row_quantize(w, group_size=G)
    cand = np.arange(-8, 8, dtype=np.float64)
    for r in range(w.shape[0]):
        for c in range(w.shape[1]):
            sc = s[r, c // G]
            v = float(np.float32(w[r, c]) / np.float32(sc))
            d = np.abs(v - cand)
            best = np.flatnonzero(d == d.min())
            if best.size > 1:          # tie: the even code
                best = best[cand[best] % 2 == 0]
            assert q[r, c] == int(cand[best[0]]), (r, c, v)


@pytest.mark.parametrize("G", [128, 64, 32])
def test_int4_invariants(G):
    rng = np.random.default_rng(2)
    w = (rng.standard_normal((32, 512)) * 0.02).astype(np.float32)
    q, s = quant.int4_row_quantize(w, group_size=G)
    assert q.dtype == np.int8 and q.min() >= -8 and q.max() <= 7
    groups = w.reshape(-1, G)
    sg = s.reshape(-1)
    amax = np.abs(groups).max(axis=1)
    # scale * 8 recovers max(amax, 1e-6) exactly (division by 8 is exact)
    assert (sg * np.float32(8) == np.maximum(amax, np.float32(1e-6))).all()
    qg = q.reshape(-1, G)
    for g in range(groups.shape[0]):
        i = np.argmax(np.abs(groups[g]))
        if groups[g, i] > 0:
            assert qg[g, i] == 7                     # w/s = 8 clamps to 7
        else:
            assert qg[g, i] == -8                    # w/s = -8 exactly, no error
    # round trip: error <= s/2 while w/s < 7.5, else <= w - 7 s (<= s)
    wh = quant.dequant_int4(q, s, group_size=G).reshape(-1, G)
    err = np.abs(groups.astype(np.float64) - wh)
    ratio = groups.astype(np.float64) / sg[:, None].astype(np.float64)
    lim = np.where(ratio < 7.5, sg[:, None] / 2.0, groups - 7.0 * sg[:, None])
    assert (err <= lim * (1 + 1e-6) + 1e-12).all()


def test_int4_zero_group_scale():
    q, s = quant.int4_row_quantize(np.zeros((1, 128), np.float32))
    assert s[0, 0] == np.float32(1e-6) / np.float32(8) and (q == 0).all()


def test_int4_rejects_ragged_groups():
    with pytest.raises(ValueError):
        quant.int4_row_quantize(np.zeros((2, 100), np.float32))


def test_pack_layout_hand_example():
    # q = [1, -1, -8, 7]: low nibble = even index, two's complement nibbles
    b = quant.pack_int4(np.array([[1, -1, -8, 7]], np.int8))
    assert b.tolist() == [[0xF1, 0x78]]
    assert quant.unpack_int4(b).tolist() == [[1, -1, -8, 7]]


def test_pack_unpack_roundtrip():
    rng = np.random.default_rng(3)
    q = rng.integers(-8, 8, (7, 256)).astype(np.int8)
    assert (quant.unpack_int4(quant.pack_int4(q)) == q).all()


def test_int4_matches_listing_ops_cross_check():
    """Cross-check only (not a pin): the listing's own torch operators."""
    rng = np.random.default_rng(4)
    w = (rng.standard_normal((8, 384)) * 0.02).astype(np.float32)
    t = torch.from_numpy(w).reshape(-1, 128)
    mx = torch.abs(t).amax(dim=1, keepdim=True)
    sc = mx.clamp(min=1e-6) / 8
    qt = t.div(sc).round().clamp_(-8, 7).to(torch.int8)
    q, s = quant.int4_row_quantize(w)
    assert (q.reshape(-1, 128) == qt.numpy()).all()
    assert (s.reshape(-1, 1) == sc.numpy()).all()


# ---------------------------------------------------------------------------
# FP8 e4m3
# ---------------------------------------------------------------------------

def test_e4m3_defining_values():
    v = quant.E4M3_VALUES
    assert v[0x00] == 0.0 and v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9
    assert v[0x08] == 2.0 ** -6 and v[0x38] == 1.0 and v[0xB8] == -1.0
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0 and v[0x77] == 240.0
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    fin = v[np.isfinite(v)]
    assert fin.max() == 448.0 and len(np.unique(fin)) == 253  # +0 and -0 equal


def test_e4m3_encode_matches_library_conversion():
    """torch's float8_e4m3fn cast (round to nearest even, not saturating)
    agrees on every bf16 bit pattern below 464 in magnitude, the midpoint
    between 448 and the next step 480 above which torch gives NaN."""
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16)
    x = bits.view(torch.bfloat16).float()
    ok = torch.isfinite(x) & (x.abs() < 464)
    xs = x[ok]
    lib = xs.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = quant.fp8_e4m3_encode(xs.numpy())
    assert (lib == ours).all()


def test_e4m3_saturates():
    assert quant.fp8_e4m3_encode(np.array([1e6, -1e6, 448.0, 470.0], np.float32)).tolist() == \
        [0x7E, 0xFE, 0x7E, 0x7E]
    assert quant.fp8_e4m3_encode(np.array([-0.0, -1e-9], np.float32)).tolist() == [0x80, 0x80]


def test_fp8_row_quantize_invariants():
    rng = np.random.default_rng(5)
    x = torch.from_numpy(rng.standard_normal((16, 300)).astype(np.float32)).to(torch.bfloat16)
    xf = x.float().numpy()
    q, s = quant.fp8_row_quantize(xf)
    amax = np.abs(xf).max(axis=1)
    assert (s == np.maximum(amax, np.float32(1e-12)) / np.float32(448)).all()
    # the row's largest magnitude lands on +-448 exactly
    for r in range(16):
        i = np.argmax(np.abs(xf[r]))
        assert q[r, i] & 0x7F == 0x7E
    # error at most half an e4m3 step at |x/s| (relative 2^-4, absolute 2^-10 s)
    deq = quant.dequant_fp8_rows(q, s)
    t = np.abs(xf / s[:, None].astype(np.float64))
    half_step = np.where(t >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(t, 1e-30))) - 4),
                         2.0 ** -10)
    assert (np.abs(deq - xf) <= half_step * s[:, None] * (1 + 1e-6)).all()


def test_fp8_row_quantize_valid_rows_bound_and_zero_row():
    x = np.ones((4, 32), np.float32)
    x[1] = 0.0
    x[2] *= 3.0
    q, s = quant.fp8_row_quantize(x, num_valid_rows=3, scale_ub=2.0)
    assert (q[3] == 0).all() and s[3] == 0.0
    assert (q[1] == 0).all() and s[1] == np.float32(1e-12) / np.float32(448)
    # row 2: amax 3 clamped to the bound 2 -> x/s = 672 saturates to 448
    assert s[2] == np.float32(2.0) / np.float32(448) and (q[2] == 0x7E).all()
    assert (q[0] == 0x7E).all()
