"""Build libfa.so (the CUDA kernels and the C ABI) in-tree for sm_100a with nvcc.

Usage: ``python -m io_aware_exact_17_b200.build [--force] [--verbose]``.
Rebuilds only when a source under csrc/ or include/ is newer than the library.
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
LIB = PKG / "libfa.so"
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and Path(cand).exists():
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[Path]:
    return sorted(CSRC.glob("*.cu")) + sorted(CSRC.glob("*.cuh")) + sorted(CSRC.glob("*.h")) + sorted(
        (ROOT / "include").glob("*.h"))


# The test build: the same sources with the test hooks compiled in (a forward
# launch can be made to leave out one software mbarrier arrival) and a 5 ms
# wait limit, so that a test can make a bounded wait run out and check that the
# kernel returns with FA_ERR_TIMEOUT. Only tests load it.
TEST_LIB = PKG / "libfa_testhooks.so"
TEST_DEFINES = ["-DFA_TEST_HOOKS", "-DFA_WAIT_LIMIT_NS=5000000ull"]


def needs_build_of(lib: Path) -> bool:
    if not lib.exists():
        return True
    t = lib.stat().st_mtime
    return any(s.stat().st_mtime > t for s in sources())


def needs_build() -> bool:
    return needs_build_of(LIB)


def _compile(lib: Path, defines: list[str], verbose: bool) -> Path:
    tmp = lib.with_suffix(".so.tmp")
    cmd = [
        _nvcc(), *ARCH_FLAGS, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
        "--expt-relaxed-constexpr", *defines, "-o", str(tmp), str(CSRC / "fa_api.cu"),
    ]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> Path:
    if not force and not needs_build():
        return LIB
    return _compile(LIB, [], verbose)


def build_test_hooks(force: bool = False, verbose: bool = False) -> Path:
    """Build libfa_testhooks.so (see TEST_DEFINES); tests only."""
    if not force and not needs_build_of(TEST_LIB):
        return TEST_LIB
    return _compile(TEST_LIB, TEST_DEFINES, verbose)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    build_test_hooks(force="--force" in sys.argv)
    print(LIB)
