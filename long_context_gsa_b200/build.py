"""Build libgsa.so in-tree with nvcc for sm_100a (B200).

    python -m long_context_gsa_b200.build [--force]

The library is one translation unit (csrc/gsa_api.cu includes the kernel
headers).  It is rebuilt when any source under csrc/ or include/ is newer
than the library.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
LIB = PKG / "libgsa.so"
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _sources() -> list[Path]:
    return sorted(CSRC.glob("*.cu")) + sorted(CSRC.glob("*.cuh")) + sorted((ROOT / "include").glob("*.h"))


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and Path(cand).exists():
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libgsa.so")


def needs_build() -> bool:
    if not LIB.exists():
        return True
    t = LIB.stat().st_mtime
    return any(s.stat().st_mtime > t for s in _sources())


def build_library(force: bool = False, verbose: bool = False) -> Path:
    if not force and not needs_build():
        return LIB
    tmp = LIB.with_suffix(f".so.{os.getpid()}.tmp")
    cmd = [nvcc(), *NVCC_FLAGS, str(CSRC / "gsa_api.cu"), "-o", str(tmp)]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stderr[-8000:]}")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, LIB)
    return LIB


def build_variant(out: Path, defines: dict) -> Path:
    """Build a copy of the library with extra preprocessor definitions (for
    tests that need a shortened wait limit, say) at `out`; rebuilt when any
    source is newer than it."""
    out = Path(out)
    if out.exists() and not any(s.stat().st_mtime > out.stat().st_mtime for s in _sources()):
        return out
    tmp = out.with_suffix(f".so.{os.getpid()}.tmp")
    flags = [f"-D{k}={v}" for k, v in defines.items()]
    res = subprocess.run([nvcc(), *NVCC_FLAGS, *flags, str(CSRC / "gsa_api.cu"), "-o", str(tmp)], capture_output=True,
                         text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stderr[-8000:]}")
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build_library(force="--force" in sys.argv, verbose="-v" in sys.argv))
