"""Builds the four C-ABI libraries (and the synthetic-input device library) for sm_100a.

Run ``python top_kv_routing_b200/build.py``; the shared objects land in-tree under
``top_kv_routing_b200/lib`` and ``msa_synth/`` so they travel with the source tree.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "lib")
INCLUDE = os.path.join(ROOT, "include")
SYNTH = os.path.join(ROOT, "msa_synth")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v",
         "-I" + INCLUDE, "-I" + CSRC]

TARGETS = {
    os.path.join(LIB, "libmsa_pool.so"): ["pool.cu"],
    os.path.join(LIB, "libmsa_route.so"): ["route.cu", "route_tc.cu", "route_proj.cu"],
    os.path.join(LIB, "libmsa_gather.so"): ["gather.cu"],
    os.path.join(LIB, "libmsa_decode.so"): ["decode.cu"],
    os.path.join(LIB, "libmsa_prefill.so"): ["prefill.cu", "prefill_tc.cu"],
    os.path.join(LIB, "libmsa_bank.so"): ["bank.cu"],
}
SYNTH_TARGET = os.path.join(SYNTH, "libmsa_synth.so")

LIBRARIES = {"pool": "libmsa_pool.so", "route": "libmsa_route.so", "gather": "libmsa_gather.so",
             "decode": "libmsa_decode.so", "prefill": "libmsa_prefill.so",
             "bank": "libmsa_bank.so"}


def nvcc() -> str:
    for c in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _deps(srcs):
    deps = list(srcs) + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    deps += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    return deps


def _stale(out, deps):
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(out, srcs, extra_inc=(), force=False, verbose=False):
    deps = _deps(srcs)
    if not force and not _stale(out, deps):
        return out, ""
    cmd = [nvcc()] + ARCH + FLAGS + [f"-I{p}" for p in extra_inc] + ["-o", out] + list(srcs)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {os.path.basename(out)}:\n{r.stdout}\n{r.stderr}")
    return out, r.stderr


def build(force: bool = False, verbose: bool = False) -> list[str]:
    os.makedirs(LIB, exist_ok=True)
    jobs = [(out, [os.path.join(CSRC, s) for s in srcs], ()) for out, srcs in TARGETS.items()]
    jobs.append((SYNTH_TARGET, [os.path.join(SYNTH, "csrc", "synth_dev.cu")], (os.path.join(SYNTH, "csrc"),)))
    with ThreadPoolExecutor(max_workers=len(jobs)) as ex:
        res = list(ex.map(lambda j: _compile(j[0], j[1], j[2], force, verbose), jobs))
    if verbose:
        for out, log in res:
            if log:
                print(f"== {os.path.basename(out)}\n{log}")
    return [r[0] for r in res]


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
