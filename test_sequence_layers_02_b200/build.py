"""Build ``libttt_scan.so`` (the C-ABI scan library) in-tree for sm_100a."""

from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
LIB = PKG / "libttt_scan.so"
# Objects, compiled in parallel and linked into one shared library: (source,
# object stem, extra defines). simt.cu is built once per input dtype and mode.
UNITS = [(CSRC / "ttt_scan.cu", "ttt_scan", ()),
         (CSRC / "cluster.cu", "cluster", ()),
         (CSRC / "backward.cu", "backward", ()),
         (CSRC / "probe.cu", "probe", ()),
         (CSRC / "tc_many.cu", "tc_many", ()),
         (CSRC / "host_scan.cu", "host_scan", ())]
UNITS += [(CSRC / "simt.cu", f"simt_{dt}_{md}",
           (f"-DTTT_SIMT_BF16={int(dt == 'bf16')}", f"-DTTT_SIMT_MINIBATCH={int(md == 'mb')}"))
          for dt in ("f32", "bf16") for md in ("tok", "mb")]
SOURCES = sorted({src for src, _, _ in UNITS})
HEADERS = sorted(CSRC.glob("*.cuh")) + sorted(CSRC.glob("*.h")) + sorted((ROOT / "include").glob("*.h"))

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = [
    *ARCH, "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr",
    "-I", str(ROOT / "include"), "-I", str(CSRC),
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def stale() -> bool:
    if not LIB.exists():
        return True
    t = LIB.stat().st_mtime
    return any(p.stat().st_mtime > t for p in SOURCES + HEADERS if p.exists())


def build(force: bool = False, verbose: bool = False, extra=()) -> Path:
    if not force and not stale():
        return LIB
    tag = f"{os.getpid()}"
    objs, procs = [], []
    try:
        for src, stem, defs in UNITS:
            obj = LIB.parent / f".{stem}.{tag}.o"
            cmd = [_nvcc(), *NVCC_FLAGS, *defs, *extra, "-c", str(src), "-o", str(obj)]
            if verbose:
                print(" ".join(cmd), file=sys.stderr)
            objs.append(obj)
            procs.append((stem, subprocess.Popen(cmd)))
        failed = [stem for stem, pr in procs if pr.wait() != 0]
        if failed:
            raise RuntimeError(f"nvcc failed on {', '.join(failed)}")
        tmp = LIB.with_suffix(f".so.tmp{tag}")
        link = [_nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", *map(str, objs), "-o", str(tmp)]
        if verbose:
            print(" ".join(link), file=sys.stderr)
        subprocess.run(link, check=True)
        os.replace(tmp, LIB)
    finally:
        for obj in objs:
            if obj.exists():
                obj.unlink()
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
