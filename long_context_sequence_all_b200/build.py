"""Build ``libulysses.so`` (all CUDA sources, sm_100a) in-tree with nvcc.

    python -m long_context_sequence_all_b200.build [--force] [--verbose]

Objects go to ``_build/``; the shared library lands next to this file so it
travels with the source tree.  nvcc cross-compiles for sm_100a without a GPU.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import re
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libulysses.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

SOURCES = ["api.cu", "prof.cu", "permute.cu", "loss.cu", "loss_noalloc.cu", "attn_f32.cu", "attn_fwd_sm100.cu",
           "attn_bwd_sm100.cu", "attn_bwd_fused_sm100.cu", "proj_sm100.cu", "kv_copy.cu", "labels.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
         "-Xcompiler", "-Wall", "-I", INCLUDE]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps_mtime() -> float:
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "ulysses.h")]
    return max(os.path.getmtime(f) for f in files)


# Kernels that split their register pool between warpgroups with setmaxnreg:
# the split only adds up when the kernel launches with exactly this many
# registers per thread; any other count would make setmaxnreg.inc wait forever.
REGISTER_SPLIT_KERNELS = {
    "attn_fwd_sm100.cu": [("attn_fwd_sm100_kernel", 168)],
    "attn_bwd_sm100.cu": [("attn_dkdv_sm100_kernel", 168), ("attn_dq_sm100_kernel", 168)],
    "attn_bwd_fused_sm100.cu": [("attn_bwd_sm100_kernel", 128)],
}


def _check_register_split(src: str, ptxas_log: str):
    lines = ptxas_log.splitlines()
    for kernel, want in REGISTER_SPLIT_KERNELS[src]:
        found = False
        # every instance of the kernel (template instantiations included)
        for i, line in enumerate(lines):
            if "Compiling entry function" in line and kernel in line:
                for nxt in lines[i + 1:i + 6]:
                    m = re.search(r"Used (\d+) registers", nxt)
                    if m:
                        if int(m.group(1)) != want:
                            raise RuntimeError(f"{kernel} uses {m.group(1)} registers, its warpgroup register "
                                               f"split needs exactly {want}; refusing to build")
                        found = True
                        break
        if not found:
            raise RuntimeError(f"ptxas report for {kernel} not found; refusing to build")


def _compile(src: str, verbose: bool) -> str:
    obj = os.path.join(BUILD, src.replace(".cu", ".o"))
    cmd = [nvcc(), *ARCH, *FLAGS, "-c", os.path.join(CSRC, src), "-o", obj]
    if verbose or src in REGISTER_SPLIT_KERNELS:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if src in REGISTER_SPLIT_KERNELS:
        _check_register_split(src, r.stdout + r.stderr)
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, file=sys.stderr)
    return obj


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= _deps_mtime():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose), SOURCES))
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static", "-ldl", "-lrt", "-lpthread"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
