"""Compile-time resource checks of every kernel (CPU only: nvcc cross-compiles for sm_100a).

Each library source is compiled with the build's flags plus the assembler's resource report,
and every kernel must run without a stack frame or register spills: local-memory traffic in
the hot loops (the GEMM's producer, loader, MMA and epilogue roles, the quantizer's per-lane
block) would cost far more than any of these kernels' arithmetic.
"""
import os
import re
import subprocess
import tempfile

import pytest

from grouped_sparse_gemm_b200 import _build

FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-fmad=false", "-Xcompiler", "-fPIC",
         "-I" + os.path.join(_build.ROOT, "include"), "--expt-relaxed-constexpr", "-Xptxas", "-v"]

_PROPS = re.compile(r"Function properties for (\S+)\s*\n\s*(\d+) bytes stack frame, (\d+) bytes spill stores, "
                    r"(\d+) bytes spill loads")


def _nvcc():
    try:
        return _build.nvcc_path()
    except RuntimeError:
        return None


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not available")
@pytest.mark.parametrize("src", _build.SOURCES)
def test_no_stack_frame_or_spills(src):
    with tempfile.TemporaryDirectory() as d:
        r = subprocess.run([_nvcc()] + _build.ARCH + FLAGS + ["-c", os.path.join(_build.CSRC, src), "-o",
                                                              os.path.join(d, "k.o")],
                           capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    found = _PROPS.findall(r.stdout + r.stderr)
    with open(os.path.join(_build.CSRC, src)) as f:
        has_kernels = "__global__" in f.read()
    assert found or not has_kernels, "no resource report from the assembler"
    bad = [(name, int(f), int(s), int(l)) for name, f, s, l in found if int(f) or int(s) or int(l)]
    assert not bad, f"kernels with a stack frame or spills: {bad}"
