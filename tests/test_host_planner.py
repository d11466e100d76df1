"""Host-only replay of the planners (no GPU needed).

tests/host/planner_replay.cu includes the dispatcher's source and checks, for
the page workloads, test geometries and every channels-per-thread choice of
the 80 sweep shapes: the streaming kernel's stage layout and TMA box
coordinates, that every output is written exactly once, and on small shapes
its arithmetic on an emulated staged tile against a naive convolution; and
the implicit GEMM's plans (shared memory, MMA N extent, tap-row folding,
weight-slice residency).  It links the library's objects for the launch
symbols it never calls.
"""
import glob
import json
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not available")
def test_planner_replay(tmp_path):
    from depthwise_convolution_fp32_b200 import build as b
    b.build()
    shapes = json.load(open(os.path.join(ROOT, "depthwise_convolution_fp32_b200", "sweep80.json")))["shapes"]
    inc = tmp_path / "sweep80.inc"
    inc.write_text("\n".join("{%d,%d,%d,%d}," % tuple(s) for s in shapes) + "\n")
    objs = [o for o in glob.glob(os.path.join(b.BUILD_DIR, "*.o")) if not o.endswith("gconv_api.o")]
    exe = tmp_path / "planner_replay"
    cmd = [_nvcc()] + b.ARCH + ["-O2", "-std=c++17", "--expt-relaxed-constexpr", "-diag-suppress", "177",
                                "-I", b.INCLUDE, "-I", b.CSRC, "-I", b.BUILD_DIR,
                                f'-DSWEEP_INC="{inc}"',
                                os.path.join(ROOT, "tests", "host", "planner_replay.cu")] + objs + ["-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "ALL OK" in r.stdout, r.stdout[-4000:] + r.stderr[-2000:]
