"""In-tree build of the native libraries for sm_100a (B200).

``build_all()`` compiles
  * ``libcachegen.so`` -- the codec (csrc/*.cu, C ABI in include/cachegen.h);
  * ``synth/libkvsynth.so`` -- the seeded synthetic-KV generator.
Both are plain ``nvcc -shared`` builds; nothing is JIT-compiled or installed
outside the package directory, so the built files travel with the source tree.
"""
from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
INCLUDE = ROOT / "include"

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# -fmad=false: no multiply-add contraction anywhere (the codec's float path
# uses explicit IEEE round-to-nearest intrinsics as well).
NVCC_FLAGS = ARCH + [
    "-O3", "-lineinfo", "-std=c++17", "-fmad=false",
    "-Xcompiler", "-fPIC,-O2", "-shared",
]

CODEC_SOURCES = ["csrc/capi.cu", "csrc/encode.cu", "csrc/decode.cu", "csrc/static_ws.cu",
                 "csrc/context.cu"]
CODEC_HEADERS = ["csrc/cg_common.cuh"]
SYNTH_SOURCES = ["synth/kvsynth.cu"]

LIB_CODEC = PKG / "libcachegen.so"
LIB_SYNTH = PKG / "synth" / "libkvsynth.so"


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _stale(target: Path, deps: list[Path]) -> bool:
    if not target.exists():
        return True
    t = target.stat().st_mtime
    return any(d.stat().st_mtime > t for d in deps)


def _run(cmd: list[str]) -> None:
    res = subprocess.run(cmd, cwd=PKG, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed ({res.returncode}): {' '.join(cmd)}")
    if os.environ.get("CG_BUILD_VERBOSE"):
        sys.stderr.write(res.stdout + res.stderr)


def build_codec(force: bool = False, verbose_ptxas: bool = False) -> Path:
    deps = [PKG / s for s in CODEC_SOURCES + CODEC_HEADERS] + [INCLUDE / "cachegen.h"]
    if force or _stale(LIB_CODEC, deps):
        extra = ["-Xptxas", "-v"] if verbose_ptxas else []
        _run([_nvcc(), *NVCC_FLAGS, *extra, f"-I{INCLUDE}", "-o", str(LIB_CODEC),
              *CODEC_SOURCES])
    return LIB_CODEC


def build_synth(force: bool = False) -> Path:
    deps = [PKG / s for s in SYNTH_SOURCES]
    if force or _stale(LIB_SYNTH, deps):
        _run([_nvcc(), *NVCC_FLAGS, "-o", str(LIB_SYNTH), *SYNTH_SOURCES])
    return LIB_SYNTH


def build_all(force: bool = False) -> None:
    build_codec(force)
    build_synth(force)


if __name__ == "__main__":
    build_all(force="--force" in sys.argv)
    print(LIB_CODEC, LIB_SYNTH)
