"""Build the CUDA library in-tree with nvcc for sm_100a.

    python -m selective_state_space_55_b200.build [--force] [--verbose]

Produces ``selective_state_space_55_b200/libmamba_ssm.so`` (cudart linked
statically, so the library does not depend on the Python environment's CUDA
runtime).  Host compilation needs no GPU.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
INCLUDE = ROOT / "include"
LIBRARY = PKG / "libmamba_ssm.so"
SOURCES = [CSRC / "mamba_ssm.cu"]
DEPENDS = SOURCES + sorted(CSRC.glob("*.cuh")) + sorted(INCLUDE.glob("*.h"))

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and Path(cand).exists():
            return cand
    raise FileNotFoundError("nvcc not found (set NVCC or put CUDA's bin on PATH)")


def build_command(output: Path, verbose: bool = False) -> list[str]:
    cmd = [nvcc_path(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC,-fvisibility=hidden", "-cudart", "static",
           f"-I{INCLUDE}", f"-I{CSRC}", *map(str, SOURCES), "-o", str(output)]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def up_to_date() -> bool:
    if not LIBRARY.exists():
        return False
    built = LIBRARY.stat().st_mtime
    return all(p.stat().st_mtime <= built for p in DEPENDS)


def build(force: bool = False, verbose: bool = False) -> Path:
    if not force and not verbose and up_to_date():
        return LIBRARY
    tmp = LIBRARY.with_name(f".libmamba_ssm.{os.getpid()}.so")
    cmd = build_command(tmp, verbose)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libmamba_ssm.so")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, LIBRARY)
    return LIBRARY


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas resource usage")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose))


if __name__ == "__main__":
    main()
