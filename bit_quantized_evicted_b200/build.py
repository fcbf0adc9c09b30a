"""Build libminikv.so in-tree with nvcc for sm_100a.

    python -m bit_quantized_evicted_b200.build [--force] [--verbose-ptxas]
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libminikv.so")
# The same library with the flash-attention pipeline's bounded waits cut to one
# poll: its waits give up while their copies are in flight, which exercises the
# abort path (drain, status word) without any fault.  Only the tests load it.
WAIT_PROBE_LIB = os.path.join(PKG, "libminikv_waitprobe.so")
SOURCES = ["minikv_api.cu", "pack.cu", "prefill.cu", "topk.cu", "decode.cu", "decode_static.cu"]
HEADERS = ["common.cuh", "tc.cuh"]
NVCC = os.environ.get("NVCC", "nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-I", os.path.join(ROOT, "include"),
]


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "minikv.h")]
    objs, jobs = [], []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(o)
        if force or ptxas_verbose or _stale(o, [s, *hdrs]):
            cmd = [NVCC, *FLAGS, "-c", s, "-o", o]
            if ptxas_verbose:
                cmd += ["-Xptxas", "-v"]
            jobs.append(cmd)
    probe_src = os.path.join(CSRC, "prefill.cu")
    probe_obj = os.path.join(BUILD, "prefill_waitprobe.o")
    if force or _stale(probe_obj, [probe_src, *hdrs]):
        jobs.append([NVCC, *FLAGS, "-DMINIKV_WAIT_LIMIT=1", "-c", probe_src, "-o", probe_obj])
    with cf.ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        for res in ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), jobs):
            if res.returncode != 0:
                raise RuntimeError(f"nvcc failed:\n{res.stdout}\n{res.stderr}")
            if ptxas_verbose:
                print(res.stderr)
    probe_objs = [probe_obj if o.endswith(os.sep + "prefill.o") else o for o in objs]
    for lib, parts in ((LIB, objs), (WAIT_PROBE_LIB, probe_objs)):
        if force or jobs or _stale(lib, parts):
            tmp = lib + f".tmp{os.getpid()}"
            cmd = [NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp, *parts, "-lcudart"]
            res = subprocess.run(cmd, capture_output=True, text=True)
            if res.returncode != 0:
                raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
            os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, ptxas_verbose=args.verbose_ptxas))
