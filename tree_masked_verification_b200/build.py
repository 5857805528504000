"""Build liblongspec_hta.so in-tree with nvcc for sm_100a.

    python -m tree_masked_verification_b200.build [--force] [--out PATH] [-D KNOB=VALUE ...]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "liblongspec_hta.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-shared",
]


def sources() -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps() -> list:
    return (sources() + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _deps())


def build(force: bool = False, verbose: bool = False, out: str = None, defines=()) -> str:
    """Compile every .cu of csrc/ into one shared library for sm_100a.

    With `out` or `defines` (["HTA_KV_STAGES_D128=2", ...], the tuning knobs
    of csrc/hta_kernels.h) the library is always rebuilt, into `out`
    (default: the in-tree path); load such a build with LONGSPEC_HTA_LIB."""
    target = os.path.abspath(out) if out else LIB
    if not force and not defines and target == LIB and up_to_date():
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    os.makedirs(os.path.dirname(target), exist_ok=True)
    tmp = target + f".{os.getpid()}.tmp"
    cmd = [nvcc, *NVCC_FLAGS, *[f"-D{d}" for d in defines], "-I", INCLUDE, "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, target)
    return target


def _main(argv) -> None:
    import argparse
    ap = argparse.ArgumentParser(description=__doc__.strip().splitlines()[0])
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--out", default=None, help="write the library here instead of in-tree")
    ap.add_argument("-D", dest="defines", action="append", default=[],
                    help="tuning knob NAME=VALUE (HTA_KV_STAGES_D128, HTA_EXP2_POLY_EVERY)")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=True, out=a.out, defines=a.defines))


if __name__ == "__main__":
    _main(sys.argv[1:])
