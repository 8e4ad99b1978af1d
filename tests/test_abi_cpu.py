"""The C ABI without a GPU: the library loads, exports every function the
header declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import int4_quantized_expert_b200 as moe

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe_int4.h")


def _declared():
    src = open(HEADER).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(moe.LIB_PATH):
        from int4_quantized_expert_b200 import build
        build.build()
    return moe.lib()


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) == 21
    for n in names:
        assert hasattr(lib, n), n


def test_header_compiles_and_links_as_plain_c(lib, tmp_path):
    """The boundary is a C ABI: a strict C99 program includes the header,
    links the library and calls it, with no Python or C++ involved."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(
        '#include "moe_int4.h"\n#include <stdio.h>\n'
        "int main(void) {\n"
        "    moe_layer_desc d; moe_dense_desc dd; (void)d; (void)dd;\n"
        '    printf("%d %s\\n", moe_abi_version(), moe_status_string(MOE_ERR_TIMEOUT));\n'
        "    return moe_quantize_int4(0, 0, 128, 128, 0, 0, 0) == MOE_OK ? 0 : 1;\n"
        "}\n")
    libdir = os.path.dirname(moe.LIB_PATH)
    exe = tmp_path / "abi"
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.dirname(HEADER), str(src),
                        "-o", str(exe), "-L", libdir, "-lmoe_int4", "-Wl,-rpath," + libdir],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "2 device wait timed out", (r.stdout, r.stderr)


def test_version_and_status_strings(lib):
    assert lib.moe_abi_version() == 2
    assert lib.moe_status_string(0) == b"ok"
    assert lib.moe_status_string(3) == b"workspace too small"
    assert lib.moe_status_string(99) == b"unknown status"


def test_quantize_rejects_bad_arguments(lib):
    S = moe.Status
    fake = 1 << 20           # an aligned non-null address that is never dereferenced
    assert lib.moe_quantize_int4(fake, 4, 256, 16, fake, fake, None) == S.UNSUPPORTED_SHAPE
    assert lib.moe_quantize_int4(fake, 4, 256, 96, fake, fake, None) == S.UNSUPPORTED_SHAPE
    assert lib.moe_quantize_int4(None, 4, 256, 64, fake, fake, None) == S.INVALID_ARG   # 64: accepted size
    assert lib.moe_quantize_int4(None, 4, 256, 32, fake, fake, None) == S.INVALID_ARG   # 32: accepted size
    assert lib.moe_quantize_int4(fake, 4, 100, 128, fake, fake, None) == S.UNSUPPORTED_SHAPE
    assert lib.moe_quantize_int4(None, 4, 256, 128, fake, fake, None) == S.INVALID_ARG
    assert lib.moe_quantize_int4(fake + 4, 4, 256, 128, fake, fake, None) == S.INVALID_ARG
    assert lib.moe_quantize_int4(None, 0, 256, 128, None, None, None) == S.OK   # empty: no-op
    assert lib.moe_quantize_fp8_rows(fake, 7, 4, 16, 4, 1.0, fake, fake, None) == S.INVALID_ARG
    assert lib.moe_quantize_fp8_rows(fake, 0, 4, 12, 4, 1.0, fake, fake, None) == S.UNSUPPORTED_SHAPE
    assert lib.moe_quantize_fp8_rows(fake, 0, 4, 16, 5, 1.0, fake, fake, None) == S.INVALID_ARG
    assert lib.moe_quantize_fp8_rows(fake, 0, 4, 16, 4, 0.0, fake, fake, None) == S.INVALID_ARG
    assert lib.moe_quantize_fp8_rows(fake, 0, 4, 16, 4, float("nan"), fake, fake, None) == S.INVALID_ARG


def test_route_rejects_bad_shapes(lib):
    S = moe.Status
    f = 1 << 20
    args = lambda T, D, E, k: (f, T, D, f, None, E, k, f, f, f, f, f, None)
    assert lib.moe_route(*args(0, 256, 4, 1)) == S.UNSUPPORTED_SHAPE
    assert lib.moe_route(*args(8, 200, 4, 1)) == S.UNSUPPORTED_SHAPE
    assert lib.moe_route(*args(8, 256, 4, 5)) == S.UNSUPPORTED_SHAPE
    assert lib.moe_route(*args(8, 256, 300, 1)) == S.UNSUPPORTED_SHAPE
    assert lib.moe_route(*args(8, 256, 16, 9)) == S.UNSUPPORTED_SHAPE
    a = list(args(8, 256, 4, 1))
    a[7] = None
    assert lib.moe_route(*a) == S.INVALID_ARG


def _desc(**kw):
    d = moe.LayerDesc()
    d.E, d.k, d.D, d.F, d.F_shared = 4, 1, 256, 512, 512
    d.format, d.group_size, d.path = moe.FMT_INT4, 128, moe.PATH_AUTO
    f = 1 << 20
    for name in ("w_router", "w_gate", "s_gate", "w_up", "s_up", "w_down", "s_down",
                 "ws_gate", "ws_up", "ws_down"):
        setattr(d, name, f)
    d.act_scale_ub = float("inf")
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_workspace_size_and_layer_checks(lib):
    d = _desc()
    n16 = lib.moe_ffn_workspace_size(ctypes.byref(d), 16)
    n64 = lib.moe_ffn_workspace_size(ctypes.byref(d), 64)
    assert 0 < n16 < n64 and n16 % 256 == 0
    assert lib.moe_ffn_workspace_size(ctypes.byref(_desc(D=200)), 16) == 0
    assert lib.moe_ffn_workspace_size(ctypes.byref(_desc(k=5)), 16) == 0
    assert lib.moe_ffn_workspace_size(ctypes.byref(_desc(group_size=16)), 16) == 0
    # groups of 64 / 32: with AUTO the workspace covers both paths when the
    # weight-streaming kernels take the shape, the tensor-core path otherwise
    g64 = _desc(group_size=64, D=384)
    pre = _desc(group_size=64, D=384, path=moe.PATH_PREFILL)
    assert lib.moe_ffn_workspace_size(ctypes.byref(g64), 16) == lib.moe_ffn_workspace_size(ctypes.byref(pre), 16)
    assert lib.moe_ffn_workspace_size(ctypes.byref(_desc(group_size=32)), 16) > 0
    assert lib.moe_ffn_workspace_size(ctypes.byref(_desc(w_up=None)), 16) == 0
    assert lib.moe_ffn_workspace_size(ctypes.byref(d), 0) == 0


def test_forward_rejects_small_workspace_and_bad_pointers(lib):
    S = moe.Status
    d = _desc()
    f = 1 << 20
    need = lib.moe_ffn_workspace_size(ctypes.byref(d), 16)
    assert lib.moe_ffn_forward(ctypes.byref(d), f, 16, f, f, 4096, None) == S.WORKSPACE_TOO_SMALL
    assert lib.moe_ffn_forward(ctypes.byref(d), f, 16, f, f + 16, need, None) == S.INVALID_ARG  # ws not 256-aligned
    assert lib.moe_ffn_forward(ctypes.byref(d), None, 16, f, f, need, None) == S.INVALID_ARG
    assert lib.moe_ffn_forward(ctypes.byref(d), f, 0, f, f, need, None) == S.UNSUPPORTED_SHAPE
    assert lib.moe_ffn_forward(None, f, 16, f, f, need, None) == S.INVALID_ARG
    assert lib.moe_ffn_forward_host(ctypes.byref(d), f, 16, f, f, 4096, None) == S.WORKSPACE_TOO_SMALL
    assert lib.moe_ffn_device_status(None, None) == S.INVALID_ARG
    ev = (ctypes.c_void_p * 2)(f, f)
    assert lib.moe_ffn_forward_timed(ctypes.byref(d), f, 16, f, f, need, None, ev, 2) == S.INVALID_ARG


def test_small_groups_on_the_weight_streaming_path(lib):
    """Groups of 64 / 32 run on the weight-streaming kernels when a stage's
    scale box fits a row (K / G a multiple of 4 and at least a stage's
    groups); other shapes are refused there and AUTO takes the tensor cores."""
    S = moe.Status
    f = 1 << 20
    names = (ctypes.c_char_p * 16)()
    ok = _desc(group_size=64, path=moe.PATH_AUTO)                       # D = 256, F = 512
    n = lib.moe_ffn_launch_names(ctypes.byref(ok), 16, names, 16)
    assert "decode_gate_up" in [names[i].decode() for i in range(n)]
    bad = _desc(group_size=64, D=384, path=moe.PATH_DECODE)            # 384 / 64 = 6 scales a row
    need = lib.moe_ffn_workspace_size(ctypes.byref(bad), 16)
    assert need > 0
    assert lib.moe_ffn_forward(ctypes.byref(bad), f, 16, f, f, need, None) == S.UNSUPPORTED_SHAPE
    n = lib.moe_ffn_launch_names(ctypes.byref(_desc(group_size=32, F=256)), 16, names, 16)
    assert "tc_gate_up" in [names[i].decode() for i in range(n)]      # F = 256: 8 < 16 groups a stage


def test_rmsnorm_checks_and_layer_prologue(lib):
    S = moe.Status
    f = 1 << 20
    assert lib.moe_rmsnorm(f, 0, 256, f, 1e-5, f, None) == S.UNSUPPORTED_SHAPE
    assert lib.moe_rmsnorm(f, 4, 200, f, 1e-5, f, None) == S.UNSUPPORTED_SHAPE
    assert lib.moe_rmsnorm(f, 4, 256, None, 1e-5, f, None) == S.INVALID_ARG
    assert lib.moe_rmsnorm(f, 4, 256, f, -1.0, f, None) == S.INVALID_ARG
    assert lib.moe_rmsnorm(f, 4, 256, f, float("nan"), f, None) == S.INVALID_ARG
    # a layer with an RMSNorm: the router normalizes x itself (no launch of its
    # own), and the workspace holds the normalized rows: T x D x 2 more bytes
    plain, normed = _desc(), _desc(rms_weight=f, rms_eps=1e-5)
    for T in (16, 4096):
        n0 = lib.moe_ffn_workspace_size(ctypes.byref(plain), T)
        n1 = lib.moe_ffn_workspace_size(ctypes.byref(normed), T)
        assert n1 >= n0 + T * 256 * 2
        names0 = (ctypes.c_char_p * 16)()
        names1 = (ctypes.c_char_p * 16)()
        n = lib.moe_ffn_launch_names(ctypes.byref(normed), T, names1, 16)
        assert n == lib.moe_ffn_launch_names(ctypes.byref(plain), T, names0, 16)
        assert [names1[i] for i in range(n)] == [names0[i] for i in range(n)]
        assert names1[0] == b"router" and b"rmsnorm" not in [names1[i] for i in range(n)]
    assert lib.moe_ffn_workspace_size(ctypes.byref(_desc(rms_weight=f, rms_eps=-1.0)), 16) == 0
    assert lib.moe_ffn_workspace_size(ctypes.byref(_desc(rms_weight=f + 4, rms_eps=1e-5)), 16) == 0


def test_dense_layer_checks(lib):
    S = moe.Status
    f = 1 << 20
    d = moe.DenseDesc()
    d.D, d.F, d.path = 256, 512, moe.PATH_AUTO
    d.w_gate = d.w_up = d.w_down = f
    d.rms_weight, d.rms_eps = None, 1e-5
    n16 = lib.moe_dense_ffn_workspace_size(ctypes.byref(d), 16)
    n512 = lib.moe_dense_ffn_workspace_size(ctypes.byref(d), 512)
    assert 0 < n16 < n512 and n16 % 256 == 0
    assert lib.moe_dense_ffn_forward(ctypes.byref(d), f, 16, f, f, 4096, None) == S.WORKSPACE_TOO_SMALL
    assert lib.moe_dense_ffn_forward(ctypes.byref(d), f, 0, f, f, n16, None) == S.UNSUPPORTED_SHAPE
    assert lib.moe_dense_ffn_forward(ctypes.byref(d), None, 16, f, f, n16, None) == S.INVALID_ARG
    assert lib.moe_dense_ffn_forward(None, f, 16, f, f, n16, None) == S.INVALID_ARG
    d.F = 200
    assert lib.moe_dense_ffn_workspace_size(ctypes.byref(d), 16) == 0
    d.F, d.w_up = 512, None
    assert lib.moe_dense_ffn_workspace_size(ctypes.byref(d), 16) == 0


def test_launch_names(lib):
    d = _desc()
    n = lib.moe_ffn_launch_names(ctypes.byref(d), 16, None, 0)
    arr = (ctypes.c_char_p * n)()
    assert lib.moe_ffn_launch_names(ctypes.byref(d), 16, arr, n) == n
    names = [arr[i].decode() for i in range(n)]
    assert len(set(names)) == n and "router" in names and "decode_gate_up" in names
    assert names.index("router") < names.index("bucket") < names.index("decode_gate_up")
    assert lib.moe_ffn_launch_names(ctypes.byref(_desc(D=100)), 16, None, 0) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        moe.quantize_int4(torch.zeros(2, 128))


def _scout_decode_desc(**kw):
    """The Scout-shaped decode layer (D=5120, F=8192, 16 experts, top-1), fake
    pointers: only for calls that return before touching the device."""
    return _desc(E=16, k=1, D=5120, F=8192, F_shared=8192, **kw)


def test_noalloc_checks_arguments_before_the_cuda_runtime(lib):
    """Argument errors of moe_ffn_forward_noalloc come back as such, before
    the library looks up its scratch array (which needs a device)."""
    S = moe.Status
    f = 1 << 20
    d = _scout_decode_desc()
    assert lib.moe_ffn_forward_noalloc(ctypes.byref(d), None, 16, f, None) == S.INVALID_ARG
    assert lib.moe_ffn_forward_noalloc(ctypes.byref(d), f, 16, None, None) == S.INVALID_ARG
    assert lib.moe_ffn_forward_noalloc(ctypes.byref(d), f, 16, f + 8, None) == S.INVALID_ARG
    assert lib.moe_ffn_forward_noalloc(ctypes.byref(d), f + 4, 16, f, None) == S.INVALID_ARG
    assert lib.moe_ffn_forward_noalloc(ctypes.byref(d), f, 0, f, None) == S.UNSUPPORTED_SHAPE
    assert lib.moe_ffn_forward_noalloc(None, f, 16, f, None) == S.INVALID_ARG


def test_noalloc_scratch_covers_scout_decode_batches(lib):
    """The no-alloc entry point's 8 MiB scratch holds every batch of the
    Scout-shaped decode layer that takes the weight-streaming path (T * k <=
    4 E, i.e. T <= 64); the first batch past it (T = 65, tensor-core path)
    is refused with WORKSPACE_TOO_SMALL before anything is launched."""
    S = moe.Status
    f = 1 << 20
    scratch = 8 << 20
    dec = _scout_decode_desc(path=moe.PATH_DECODE)
    assert lib.moe_ffn_workspace_size(ctypes.byref(dec), 64) <= scratch
    pre = _scout_decode_desc(path=moe.PATH_PREFILL)
    assert lib.moe_ffn_workspace_size(ctypes.byref(pre), 65) > scratch
    auto = _scout_decode_desc()
    assert lib.moe_ffn_forward_noalloc(ctypes.byref(auto), f, 65, f, None) == S.WORKSPACE_TOO_SMALL
    assert lib.moe_ffn_forward_noalloc(ctypes.byref(auto), f, 4096, f, None) == S.WORKSPACE_TOO_SMALL


def test_expert_parallel_steps_check_arguments(lib):
    """The compute steps of an expert-parallel layer reject bad arguments
    before touching the device; their workspaces follow the rows' count."""
    S = moe.Status
    f = 1 << 20
    d = _desc(k=2)
    n16 = lib.moe_expert_ffn_workspace_size(ctypes.byref(d), 16)
    n512 = lib.moe_expert_ffn_workspace_size(ctypes.byref(d), 512)
    assert 0 < n16 < n512 and n16 % 256 == 0
    assert lib.moe_expert_ffn_workspace_size(ctypes.byref(_desc(D=200)), 16) == 0
    assert lib.moe_expert_ffn_forward(ctypes.byref(d), f, 16, f, f, f, f, 1024, None) == S.WORKSPACE_TOO_SMALL
    assert lib.moe_expert_ffn_forward(ctypes.byref(d), f, 16, None, f, f, f, n16, None) == S.INVALID_ARG
    assert lib.moe_expert_ffn_forward(ctypes.byref(d), f, 16, f, f, f + 8, f, n16, None) == S.INVALID_ARG
    assert lib.moe_expert_ffn_forward(ctypes.byref(d), f, 0, f, f, f, f, n16, None) == S.UNSUPPORTED_SHAPE
    s16 = lib.moe_shared_ffn_workspace_size(ctypes.byref(d), 16)
    assert s16 > 0 and s16 < lib.moe_shared_ffn_workspace_size(ctypes.byref(d), 4096)
    assert lib.moe_shared_ffn_combine(ctypes.byref(d), f, 16, None, f, f, s16, None) == S.INVALID_ARG
    assert lib.moe_shared_ffn_combine(ctypes.byref(d), f, 16, f, f, f, 1024, None) == S.WORKSPACE_TOO_SMALL
