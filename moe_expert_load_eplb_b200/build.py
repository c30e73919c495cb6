"""Build libeplb.so in-tree with nvcc for sm_100a (B200).

Usage:  python -m moe_expert_load_eplb_b200.build [--force] [--verbose] [--checks]

--checks builds the checking library libeplb_checks.so instead (-DEPLB_CHECKS:
internal index checks that report EPLB_ERR_INTERNAL through the status word;
same ABI and results, slower).  EPLB_LIBRARY=checks makes the binding load it.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libeplb.so")
CHECKS_LIB = os.path.join(PKG, "libeplb_checks.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libeplb.so")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> list[str]:
    return sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        [os.path.join(ROOT, "include", "eplb.h"), os.path.abspath(__file__)]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def _compile(cmd: list[str]) -> subprocess.CompletedProcess:
    return subprocess.run(cmd, capture_output=True, text=True)


def build(force: bool = False, verbose: bool = False, checks: bool = False) -> str:
    """Compile every CUDA source into one shared library (static cudart):
    one nvcc per source file, in parallel, then one link.  ``checks`` builds
    the checking library instead."""
    lib = CHECKS_LIB if checks else LIB
    if not force and up_to_date(lib):
        return lib
    import tempfile
    from concurrent.futures import ThreadPoolExecutor
    common = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "--use_fast_math",
              "-Xcompiler", "-fPIC,-O3", "-I", os.path.join(ROOT, "include")]
    if verbose:
        common.insert(1, "-Xptxas=-v")
    if checks:
        common.append("-DEPLB_CHECKS")
    with tempfile.TemporaryDirectory(prefix="eplb_build_") as tmpdir:
        objs = [os.path.join(tmpdir, os.path.basename(src) + ".o") for src in sources()]
        cmds = [common + ["-c", src, "-o", obj] for src, obj in zip(sources(), objs)]
        with ThreadPoolExecutor(max_workers=max(1, min(len(cmds), os.cpu_count() or 1))) as ex:
            results = list(ex.map(_compile, cmds))
        for cmd, res in zip(cmds, results):
            if res.returncode != 0:
                raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
            if verbose:
                sys.stderr.write(res.stdout + res.stderr)
        tmp = lib + f".tmp{os.getpid()}"
        link = [_nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
        res = _compile(link)
        if res.returncode != 0:
            raise RuntimeError("nvcc link failed:\n" + " ".join(link) + "\n" + res.stdout + res.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                checks="--checks" in sys.argv))
