"""Build the CUDA libraries in-tree for sm_100a with nvcc.

    python -m kv_cache_serving_ws_b200.build [--force] [--ptxas-info]

produces, next to this file:
  libws.so        the unit-step library (include/ws.h)
  libws_synth.so  the device input generator (include/ws_synth.h)
and, with --debug (or build(debug=True)):
  libws_debug.so  the same library with device index checks (-DWS_DEBUG_CHECKS):
                  every computed cache row, output row, partial slot and merge
                  counter is tested against its buffer's bounds; a failing check
                  skips the access and ws_sync reports WS_ERR_DEVICE_CHECK.
                  Loaded instead of libws.so when WS_LIBRARY=debug.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
         "--expt-relaxed-constexpr", "-I", INCLUDE]

WS_SOURCES = ["ws_api.cu", "unit_graph.cu", "attention.cu", "attention_pair.cu", "copy_kernels.cu", "euler.cu",
              "noalloc.cu"]
LIBS = {
    "libws.so": (WS_SOURCES, []),
    "libws_synth.so": (["synth.cu"], []),
}
DEBUG_LIBS = {"libws_debug.so": (WS_SOURCES, ["-DWS_DEBUG_CHECKS"])}
HEADERS = ["kernels.cuh", "cache_state.cuh", "sm100.cuh", "tmem_ldst.cuh", "attn_common.cuh"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libws")


def _stale(out: str, deps: list[str]) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_info: bool = False, verbose: bool = False, debug: bool = False) -> list[str]:
    built = []
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, h) for h in ("ws.h", "ws_synth.h")]
    libs = dict(LIBS, **(DEBUG_LIBS if debug else {}))
    for lib, (srcs, defines) in libs.items():
        out = os.path.join(HERE, lib)
        src_paths = [os.path.join(CSRC, s) for s in srcs]
        if not force and not ptxas_info and not _stale(out, src_paths + hdrs + [__file__]):
            continue
        cmd = [nvcc()] + ARCH + FLAGS + defines + (["-Xptxas", "-v"] if ptxas_info else []) + src_paths + ["-o", out]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed for {lib}:\n{res.stdout}\n{res.stderr}")
        if ptxas_info:
            print(res.stderr, file=sys.stderr)
        built.append(out)
    return built


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    ap.add_argument("--debug", action="store_true", help="also build libws_debug.so (device index checks)")
    a = ap.parse_args()
    for p in build(force=a.force, ptxas_info=a.ptxas_info, verbose=True, debug=a.debug):
        print("built", p)
