"""Build the in-tree shared libraries for sm_100a with nvcc.

  libw4a16.so    the C-ABI library declared in include/w4a16.h (every csrc/*.cu except synth.cu)
  libw4synth.so  the device half of the seeded input generators (csrc/synth.cu)

Usage: python -m w4a16_group_quantized_w4_b200.build [--force]
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
BUILD = os.path.join(ROOT, "_build")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-Xptxas", "-warn-spills"]

LIB = os.path.join(PKG, "libw4a16.so")
SYNTH_LIB = os.path.join(PKG, "libw4synth.so")


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources(names=None):
    srcs = sorted(f for f in os.listdir(CSRC) if f.endswith(".cu"))
    return [os.path.join(CSRC, f) for f in srcs if (names is None or f in names)]


def _deps() -> list[str]:
    out = [os.path.join(ROOT, "include", "w4a16.h")]
    out += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    return out


def _stale(target: str, inputs: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(p) > t for p in inputs)


def _compile(src: str, verbose: bool) -> str:
    obj = os.path.join(BUILD, os.path.basename(src).replace(".cu", ".o"))
    if _stale(obj, [src] + _deps()):
        cmd = [_nvcc(), *ARCH, *FLAGS, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{res.stdout}\n{res.stderr}")
        if verbose and res.stderr.strip():
            print(res.stderr, flush=True)
    return obj


def _link(objs: list[str], target: str, verbose: bool) -> None:
    if _stale(target, objs):
        cmd = [_nvcc(), *ARCH, "-shared", "-o", target, *objs, "-lcudart"]
        if verbose:
            print(" ".join(cmd), flush=True)
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"link failed for {target}:\n{res.stdout}\n{res.stderr}")


def build(verbose: bool = False, force: bool = False) -> None:
    os.makedirs(BUILD, exist_ok=True)
    if force:
        for f in os.listdir(BUILD):
            if f.endswith(".o"):
                os.remove(os.path.join(BUILD, f))
    main = [s for s in _sources() if not s.endswith("synth.cu")]
    synth = _sources(["synth.cu"])
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose), main + synth))
    _link(objs[: len(main)], LIB, verbose)
    if synth:
        _link(objs[len(main):], SYNTH_LIB, verbose)


if __name__ == "__main__":
    build(verbose=True, force="--force" in sys.argv)
    print("built", LIB)
