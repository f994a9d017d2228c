"""Builds libplx.so and libplx_synth.so in-tree with nvcc for sm_100a.

    python -m local_linear_attention_streamed_b200._build [--force]

The shared libraries are written next to this file so that they travel with
the source tree; nothing is installed elsewhere.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
ROOT = os.path.dirname(PKG)
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
NVCC = os.path.join(CUDA_HOME, "bin", "nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
          "-I", os.path.join(ROOT, "include")]

LIBS = {
    "libplx.so": {
        "srcs": ["plx_api.cu", "simt.cu", "decode_mma.cu", "prefill_tc.cu", "norm_rope.cu",
                 "decode_noalloc.cu", "decode_gqa.cu", "decode_gqa_tc.cu", "backward_tc.cu", "fp8_linear.cu", "decode_fp8kv.cu"],
        "deps": ["plx_internal.cuh", "sm100.cuh", "decode_tc_common.cuh"],
        "link": ["-lcublas", "-lcublasLt", f"-Xlinker", f"-rpath={os.path.join(CUDA_HOME, 'lib64')}"],
    },
    "libplx_synth.so": {
        "srcs": ["synth.cu"],
        "deps": [],
        "link": [],
    },
}


def _stale(target, inputs):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(p) > t for p in inputs)


def build(force: bool = False, verbose: bool = False) -> list[str]:
    """Compiles every library whose sources changed; returns the built paths."""
    out = []
    headers = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))]
    for name, spec in LIBS.items():
        target = os.path.join(PKG, name)
        srcs = [os.path.join(CSRC, s) for s in spec["srcs"]]
        deps = srcs + [os.path.join(CSRC, s) for s in spec["deps"]] + headers + [__file__]
        if not force and not _stale(target, deps):
            out.append(target)
            continue
        objs = []
        for src in srcs:
            obj = os.path.join(PKG, "_objs", os.path.basename(src) + ".o")
            os.makedirs(os.path.dirname(obj), exist_ok=True)
            cmd = [NVCC, *ARCH, *COMMON, "-c", src, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
            subprocess.run(cmd, check=True)
            objs.append(obj)
        tmp = target + ".tmp"
        subprocess.run([NVCC, *ARCH, "-shared", "-o", tmp, *objs, *spec["link"]], check=True)
        os.replace(tmp, target)
        out.append(target)
    return out


if __name__ == "__main__":
    for p in build(force="--force" in sys.argv, verbose="-v" in sys.argv):
        print(p)
