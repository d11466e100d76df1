"""Build libgconv.so in-tree with nvcc for sm_100a.

    python -m depthwise_convolution_fp32_b200.build [--force]

Each .cu under csrc/ compiles to an object in parallel; the objects link into
depthwise_convolution_fp32_b200/libgconv.so (static CUDA runtime, no torch).
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libgconv.so")
PEAKS_SRC = os.path.join(PKG, "peaks", "peaks.cu")
PEAKS_LIB = os.path.join(PKG, "libgconv_peaks.so")
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
              "--expt-relaxed-constexpr", "-diag-suppress", "177", "-Xcompiler", "-fvisibility=hidden"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libgconv.so")


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def headers() -> list[str]:
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    hs += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return hs


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


TABLE_JSON = os.path.join(PKG, "dispatch_table.json")
TABLE_INC = os.path.join(BUILD_DIR, "gconv_dispatch_table.inc")
TABLE_FAMILIES = {"direct_stream": 1, "direct_blocked": 2, "igemm_split": 3, "winograd": 4, "igemm_fused": 5}


def write_dispatch_table() -> str:
    """dispatch_table.json (per-shape kernel choices measured on B200) as the
    C initialiser list the dispatcher compiles in."""
    import json
    lines = ["/* generated from dispatch_table.json by build.py */"]
    if os.path.exists(TABLE_JSON):
        for e in json.load(open(TABLE_JSON))["entries"]:
            fam, _, kt = e["best"].partition(":kt")
            key = list(e["shape"]) + [1 if e.get("chain") else 0]
            assert len(key) == 12 and fam in TABLE_FAMILIES, e
            lines.append("{{%s}, %d, %d}," % (", ".join(str(int(v)) for v in key), TABLE_FAMILIES[fam],
                                              int(kt) if kt else 0))
    text = "\n".join(lines) + "\n"
    if not os.path.exists(TABLE_INC) or open(TABLE_INC).read() != text:
        with open(TABLE_INC, "w") as f:
            f.write(text)
    return TABLE_INC


def _compile(src: str, extra: list[str]) -> str:
    obj = os.path.join(BUILD_DIR, os.path.basename(src)[:-3] + ".o")
    if _stale(obj, [src] + headers() + [TABLE_INC]):
        cmd = [nvcc()] + ARCH + NVCC_FLAGS + extra + ["-I", INCLUDE, "-I", CSRC, "-I", BUILD_DIR, "-c", src, "-o",
                                                      obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj


def build_peaks(force: bool = False) -> str:
    """The benchmark's roofline microbenchmarks (FP32 FMA, tcgen05 tf32 / bf16
    MMA rates) as libgconv_peaks.so; measurement tooling, not the C ABI."""
    deps = [PEAKS_SRC, os.path.join(PKG, "peaks", "peaks.h"), os.path.join(CSRC, "device_utils.cuh")]
    if not force and not _stale(PEAKS_LIB, deps):
        return PEAKS_LIB
    tmp = PEAKS_LIB + f".tmp{os.getpid()}"
    cmd = [nvcc()] + ARCH + NVCC_FLAGS + ["-shared", PEAKS_SRC, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {PEAKS_SRC}:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, PEAKS_LIB)
    return PEAKS_LIB


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every CUDA source and link libgconv.so (and the benchmark's
    libgconv_peaks.so); returns libgconv.so's path."""
    os.makedirs(BUILD_DIR, exist_ok=True)
    build_peaks(force)
    write_dispatch_table()
    srcs = sources()
    if not force and not _stale(LIB, srcs + headers() + [TABLE_INC]):
        return LIB
    if force:
        for f in os.listdir(BUILD_DIR):
            if f.endswith(".o"):
                os.remove(os.path.join(BUILD_DIR, f))
    extra = ["-Xptxas", "-v"] if verbose else []
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra), srcs))
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc()] + ARCH + ["-shared", "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
