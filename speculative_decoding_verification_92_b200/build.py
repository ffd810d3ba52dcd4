"""Build libspecverify.so in-tree with nvcc for sm_100a.

``python -m speculative_decoding_verification_92_b200.build`` (or
``build()``) compiles ``csrc/spec_verify.cu`` (which includes the kernel
headers) and the host-side ``csrc/*.cpp`` into
``speculative_decoding_verification_92_b200/libspecverify.so``.
The library is rebuilt only when the sources or the public header change
(content hash stored beside the library).
"""
from __future__ import annotations

import hashlib
import os
import shutil
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
INCLUDE = ROOT / "include"
LIB = PKG / "libspecverify.so"
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and Path(cand).exists():
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libspecverify.so")


def sources() -> list[Path]:
    return (sorted(CSRC.glob("*.cu")) + sorted(CSRC.glob("*.cuh")) + sorted(CSRC.glob("*.cpp"))
            + sorted(INCLUDE.glob("*.h")))


def kernel_sources() -> list[Path]:
    """The sources the GPU kernels and their launches are built from (the
    host-only components in csrc/*.cpp and include/sv_host.h excluded)."""
    return sorted(CSRC.glob("*.cu")) + sorted(CSRC.glob("*.cuh")) + [INCLUDE / "spec_verify.h"]


def kernel_source_hash() -> str:
    """Hash of kernel_sources(): profiles of a kernel stay valid while it is
    unchanged."""
    h = hashlib.sha256()
    for s in kernel_sources():
        h.update(s.name.encode())
        h.update(s.read_bytes())
    h.update(" ".join(ARCH).encode())
    return h.hexdigest()


def row_stats_source_hash() -> str:
    """Hash of what the row-statistics kernel is built and launched from: its
    header, the shared device helpers and the launch function in
    spec_verify.cu.  DRAM counters taken on that kernel stay valid while this
    is unchanged (edits to the other kernels do not touch them)."""
    h = hashlib.sha256()
    for s in (CSRC / "sv_row_stats.cuh", CSRC / "sv_common.cuh"):
        h.update(s.name.encode())
        h.update(s.read_bytes())
    cu = (CSRC / "spec_verify.cu").read_text()
    start = cu.index("cudaError_t launch_stats(")
    h.update(cu[start:cu.index("\n}\n", start)].encode())
    h.update(" ".join(ARCH).encode())
    return h.hexdigest()


def source_hash() -> str:
    h = hashlib.sha256()
    for s in sources():
        h.update(s.name.encode())
        h.update(s.read_bytes())
    h.update(" ".join(ARCH).encode())
    return h.hexdigest()


def _stamp(lib: Path) -> Path:
    return lib.with_name(lib.name + ".srchash")


def is_stale(lib: Path = LIB) -> bool:
    """True unless the library exists and was built from the current sources
    (content hash, so copies that reset file times do not force a rebuild)."""
    stamp = _stamp(lib)
    if not lib.exists() or not stamp.exists():
        return True
    return stamp.read_text().strip() != source_hash()


def nvcc_command(out: Path, extra=()) -> list[str]:
    return [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "--shared",
            "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
            "-I", str(INCLUDE), "-I", str(CSRC), *extra,
            "-o", str(out), str(CSRC / "spec_verify.cu"), *[str(p) for p in sorted(CSRC.glob("*.cpp"))]]


def build(force: bool = False, verbose: bool = False, extra=(), out: Path | None = None) -> Path:
    """Compile the library (to ``out``, default the in-tree LIB) unless it is
    up to date; ``extra`` are additional nvcc flags."""
    if out is not None and Path(out) != LIB:
        cmd = nvcc_command(Path(out), extra)
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)
        return Path(out)
    if not force and not is_stale():
        return LIB
    tmp = LIB.with_suffix(f".so.tmp{os.getpid()}")
    cmd = nvcc_command(tmp, extra)
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    if list(extra) in ([], ["-Xptxas", "-v"]):
        _stamp(LIB).write_text(source_hash() + "\n")
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else ())
