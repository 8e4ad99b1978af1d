"""Compile-time resources of the hot kernels (CPU only: nvcc cross-compiles
for sm_100a): none of them may spill registers to local memory."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "int4_quantized_expert_b200", "csrc")

# kernels (mangled-name fragments) that must not spill
HOT = {
    "ffn_decode.cu": ["decode_ffn_kernel", "act16_kernel"],
    "tc_gemm.cu": ["tc_gemm_kernel", "gather_rows_kernel", "combine_slots_kernel"],
    "quantize.cu": ["quantize_int4_kernel"],
    "norm.cu": ["rmsnorm_kernel"],
}


def _nvcc():
    for c in ("/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    return None


@pytest.mark.parametrize("src", sorted(HOT))
def test_hot_kernels_do_not_spill(src, tmp_path):
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not found")
    r = subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                        "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                        "-Xptxas", "-v", "-c", os.path.join(CSRC, src), "-o", str(tmp_path / "k.o")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    # ptxas prints, per function: "Compiling entry function '<name>'" ... "N bytes spill stores, M bytes spill loads"
    seen = {}
    current = None
    for line in r.stderr.splitlines():
        m = re.search(r"Function properties for (\S+)", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and current:
            seen[current] = (int(m.group(1)), int(m.group(2)))
            current = None
    for frag in HOT[src]:
        hits = {k: v for k, v in seen.items() if frag in k}
        assert hits, "no ptxas report for %s in %s" % (frag, src)
        for name, (st, ld) in hits.items():
            assert st == 0 and ld == 0, "%s spills (%d B stores, %d B loads)" % (name, st, ld)
