"""Builds libhh.so in-tree for sm_100a (nvcc), and the input-generator library.

    python -m full_attention_gated_b200.build [--verbose]

Every CUDA source is compiled with -gencode arch=compute_100a,code=sm_100a and
-lineinfo; objects are linked with the static CUDA runtime into a shared
library that exports only the C ABI of include/hh.h.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden", "--expt-relaxed-constexpr",
          "-I", os.path.join(ROOT, "include"), "-I", CSRC]

LIBS = {
    "libhh.so": ["abi.cpp", "status.cu", "gdn_decode.cu", "gdn_chunk.cu", "gdn_bwd.cu", "attn_fwd.cu", "attn_fwd_tc.cu", "attn_fwd_tc2.cu", "attn_decode.cu",
                 "attn_decode_noalloc.cu", "phba.cu"],
    "libhh_gen.so": ["gen_inputs.cu"],
}


def _compile(src: str, verbose: bool) -> str:
    os.makedirs(BUILD, exist_ok=True)
    obj = os.path.join(BUILD, os.path.basename(src) + ".o")
    path = os.path.join(CSRC, src)
    deps = [path] + [os.path.join(CSRC, h) for h in os.listdir(CSRC) if h.endswith((".cuh", ".h"))]
    deps.append(os.path.join(ROOT, "include", "hh.h"))
    if os.path.exists(obj) and os.path.getmtime(obj) >= max(os.path.getmtime(d) for d in deps):
        return obj
    cmd = [NVCC] + ARCH + CFLAGS + (["-Xptxas", "-v"] if verbose and src.endswith(".cu") else []) + ["-c", path, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and r.stderr:
        sys.stderr.write(r.stderr)
    return obj


def build(verbose: bool = False) -> list[str]:
    out = []
    with cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        objs = {lib: [ex.submit(_compile, s, verbose) for s in srcs] for lib, srcs in LIBS.items()}
        for lib, futs in objs.items():
            files = [f.result() for f in futs]
            target = os.path.join(PKG, lib)
            if not os.path.exists(target) or os.path.getmtime(target) < max(os.path.getmtime(f) for f in files):
                cmd = [NVCC] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-o", target] + files + ["-lcudart_static", "-ldl", "-lrt", "-lpthread"]
                r = subprocess.run(cmd, capture_output=True, text=True)
                if r.returncode != 0:
                    raise RuntimeError(f"link of {lib} failed:\n{r.stdout}\n{r.stderr}")
            out.append(target)
    return out


if __name__ == "__main__":
    for p in build(verbose="--verbose" in sys.argv):
        print(p)
