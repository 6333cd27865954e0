"""Build libgla.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m gated_linear_attention_frame_b200.build [--force] [--verbose]
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG_DIR, "libgla.so")

SOURCES = [os.path.join(CSRC, "gla_api.cu")]
DEPENDS = SOURCES + [
    os.path.join(CSRC, n)
    for n in ("sm100_ptx.cuh", "gla_common.cuh", "gla_increment.cuh", "gla_scan.cuh",
              "gla_output.cuh", "gla_bwd_q.cuh", "gla_scan_bwd.cuh", "gla_bwd_kv.cuh",
              "gla_rope.cuh", "gla_gdn_scan.cuh", "gla_softmax_anchor.cuh")
] + [os.path.join(INCLUDE, "gla.h")]

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libgla.so")
    return cand


def nvcc_command(output: str = LIB_PATH, extra: list[str] | None = None) -> list[str]:
    return [
        nvcc_path(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v" if os.environ.get("GLA_PTXAS_V") else "-O3",
        "-I", INCLUDE, "-I", CSRC,
        *SOURCES, "-o", output, *(extra or []),
    ]


def up_to_date(lib: str = LIB_PATH) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in DEPENDS)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libgla.so unless it is newer than every source; return its path."""
    if not force and up_to_date():
        return LIB_PATH
    cmd = nvcc_command(LIB_PATH + ".tmp")
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stdout.write(res.stdout)
        sys.stderr.write(res.stderr)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed building libgla.so (exit %d)" % res.returncode)
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    return LIB_PATH


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose))


if __name__ == "__main__":
    main()
