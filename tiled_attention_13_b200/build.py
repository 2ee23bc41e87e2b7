"""Build the in-tree CUDA library ``libfa_b200.so`` for sm_100a with nvcc.

    python -m tiled_attention_13_b200.build [--force] [--verbose]

nvcc cross-compiles without a GPU.  The CUDA runtime is linked statically and
the driver's tensor-map encoder is looked up at run time, so the library loads
(and its symbols can be listed) on a machine without a GPU.
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libfa_b200.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)

SOURCES = ["fa_api.cu"]
DEPS = ["fa_api.cu", "tc_common.cuh", "fa_fwd_tc2.cuh", "fa_decode.cuh", "fa_bwd.cuh", "fa_fwd_tile1.cuh", "fa_fwd_short.cuh", "fa_fwd_short_wg.cuh", "fa_fwd_tc.cuh", "fa_fwd_simt.cuh", "fa_splitkv_merge.cuh", "pdl.cuh", "ptx.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2",
    "-shared", "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or install the CUDA toolkit)")


def _stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    inputs = [os.path.join(CSRC, f) for f in DEPS] + [os.path.join(INCLUDE, "fa.h"), __file__]
    return any(os.path.getmtime(p) > t for p in inputs)


def build_variant(out_path: str, defines: dict) -> str:
    """Compile the library with extra preprocessor definitions (compile-time
    kernel options, e.g. {"FA_POLY_EVERY": 4}) to ``out_path``; load it in a
    process of its own by setting $FA_B200_LIB."""
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-o", out_path]
    cmd += [f"-D{k}={v}" for k, v in defines.items()]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    subprocess.run(cmd, check=True)
    return out_path


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if any source is newer than it; return its path."""
    if not force and not _stale():
        return LIB_PATH
    tmp = LIB_PATH + ".tmp"
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-o", tmp]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed ({res.returncode})")
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))


if __name__ == "__main__":
    main()
