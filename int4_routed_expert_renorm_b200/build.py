"""Build the in-tree CUDA libraries for sm_100a with nvcc.

    python -m int4_routed_expert_renorm_b200.build [--force] [-v]

Produces ``int4_routed_expert_renorm_b200/libcolimoe.so`` (the C-ABI library of
``include/coli_moe.h``) and ``synth/libcolisynth.so`` (the seeded input fill
kernels).  Rebuilds only when a source is newer than its library.
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
          "-Xptxas", "-warn-spills"]

TARGETS = {
    "libcolimoe": dict(
        out=os.path.join(PKG, "libcolimoe.so"),
        main=os.path.join(PKG, "csrc", "coli_moe.cu"),
        deps=glob.glob(os.path.join(PKG, "csrc", "*")) + [os.path.join(ROOT, "include", "coli_moe.h")],
        inc=[os.path.join(ROOT, "include"), os.path.join(PKG, "csrc")],
    ),
    "libcolisynth": dict(
        out=os.path.join(ROOT, "synth", "libcolisynth.so"),
        main=os.path.join(ROOT, "synth", "csrc", "synth_fill.cu"),
        deps=glob.glob(os.path.join(ROOT, "synth", "csrc", "*")),
        inc=[],
    ),
}


def _stale(t) -> bool:
    if not os.path.exists(t["out"]):
        return True
    m = os.path.getmtime(t["out"])
    return any(os.path.getmtime(d) > m for d in t["deps"] + [t["main"], __file__])


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> list[str]:
    built = []
    for name, t in TARGETS.items():
        if not force and not _stale(t):
            continue
        tmp = f"{t['out']}.{os.getpid()}.tmp"     # concurrent builds each write their own, then rename
        cmd = [NVCC, *ARCH, *COMMON, *(f"-I{d}" for d in t["inc"]), t["main"], "-o", tmp]
        if ptxas_info:
            cmd[1:1] = ["-Xptxas", "-v"]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {name}:\n{r.stdout}\n{r.stderr}")
        if verbose or ptxas_info:
            sys.stderr.write(r.stderr)
        os.replace(tmp, t["out"])
        built.append(t["out"])
    return built


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / spills / shared memory")
    a = ap.parse_args()
    for p in build(a.force, a.verbose, a.ptxas_info):
        print("built", p)
