"""The bench's roofline numerators (algorithmic bytes and FLOPs per launch)
against the per-unit figures worked out from the layer's shapes: 66,846,720 B
of int4 codes and scales per touched Scout expert, 251,658,240 B of bf16
shared expert, 503.48 MFLOP per Scout token, 9.12 GB moved by quantizing the
16-expert weight set.  CPU only."""
import synth

import bench


def test_decode_bytes_per_touched_expert():
    s = synth.SHAPES["scout_decode"]
    w12 = bench.kernel_work(s, 12)
    w11 = bench.kernel_work(s, 11)
    gate_up = w12["decode_gate_up"][1] - w11["decode_gate_up"][1]
    down = w12["decode_down"][1] - w11["decode_down"][1]
    assert gate_up + down == 66_846_720                      # codes 62.9 MB + scales 3.93 MB
    assert gate_up == 2 * (8192 * 5120 // 2 + 8192 * 40 * 4)
    # the whole gate/up launch at 12 touched experts: routed + shared + activations
    # (x read; h written as bf16 and, for the routed rows, as fp16 operands)
    assert w12["decode_gate_up"][1] == 703_234_048 + 16 * 8192 * 2


def test_decode_shared_expert_bytes():
    s = synth.SHAPES["scout_decode"]
    w0 = bench.kernel_work(s, 0)
    act_gu = 16 * 5120 * 2 + (16 * 8192 + 16 * 8192) * 2 + 16 * 8192 * 2
    act_dn = (16 * 8192 + 16 * 8192) * 2 + (16 + 16) * 5120 * 4 + 16 * 5120 * 2
    assert (w0["decode_gate_up"][1] - act_gu) + (w0["decode_down"][1] - act_dn) == 251_658_240


def test_prefill_flops_per_token():
    s = synth.SHAPES["scout_prefill"]
    assert bench.layer_flops(s) == 8192 * 503_480_320    # 503.48 MFLOP per token
    w = bench.kernel_work(s, 16)
    assert w["tc_gate_up"] == ("flops", 1_374_389_534_720)
    assert w["tc_down"][1] * 2 == w["tc_gate_up"][1]


def test_quantize_bytes():
    total = sum(bench.quant_bytes(r, c) for _, r, c in bench.quant_matrices())
    assert total == 9_122_611_200                           # 8.05 GB read + 1.07 GB written
    assert sum(bench.quant_bytes(r, c, 32) for _, r, c in bench.quant_matrices()) > total


def test_group_size_changes_only_the_scale_bytes():
    s = synth.SHAPES["scout_decode"]
    a = bench.kernel_work(s, 12, 128)["decode_gate_up"][1]
    b = bench.kernel_work(s, 12, 64)["decode_gate_up"][1]
    assert b - a == 12 * 2 * 8192 * (80 - 40) * 4
