"""Build libdkv.so in-tree with nvcc for sm_100a.

    python decode_attention_host_b200/build.py [--verbose]

Run it by path: importing the package itself needs the built library.
"""
from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
LIB = PKG / "libdkv.so"
SOURCES = [CSRC / "dkv_api.cu", CSRC / "dkv_noalloc.cu", CSRC / "dkv_host.cpp"]
HEADERS = [CSRC / "dkv_kernels.cuh", CSRC / "dkv_append.cuh", CSRC / "dkv_multi.cuh", CSRC / "dkv_error.h",
           CSRC / "dkv_plan.h", CSRC / "dkv_tma.h", ROOT / "include" / "dkv.h"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared", "-cudart", "static",
         f"-I{ROOT / 'include'}", f"-I{CSRC}"]


def up_to_date() -> bool:
    if not LIB.exists():
        return False
    t = LIB.stat().st_mtime
    return all(p.stat().st_mtime <= t for p in SOURCES + HEADERS + [Path(__file__)])


def build(force: bool = False, verbose: bool = False, out: Path = LIB, defines: tuple[str, ...] = ()) -> Path:
    """Compile the library to ``out``; ``defines`` are extra -D build-time knobs (e.g. DKV_DEV_STAGES=2)."""
    out = Path(out)
    if not force and not defines and out == LIB and up_to_date():
        return LIB
    tmp = out.with_suffix(f".{os.getpid()}.tmp.so")
    cmd = [NVCC, *FLAGS, *(f"-D{d}" for d in defines), *(["-Xptxas", "-v"] if verbose else []), "-o", str(tmp),
           *map(str, SOURCES)]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    args = sys.argv[1:]
    out = Path(args[args.index("--out") + 1]) if "--out" in args else LIB
    defines = tuple(a[2:] for a in args if a.startswith("-D"))
    print(build(force=True, verbose="--verbose" in args, out=out, defines=defines))
