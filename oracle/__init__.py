"""fp64 CPU oracle for zero-copy split-KV decode attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` are the only callers.  The
product library never imports, links or runs anything here, and nothing here
imports the product package.  The arithmetic lives in ``dkv_oracle.c`` (plain
C, fp64, OpenMP over independent (batch, kv-head) groups); this module only
builds it with gcc and marshals numpy arrays through ctypes.

What is computed, and the readings taken where the pages are silent, is
stated in the header of ``dkv_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
SRC = HERE / "dkv_oracle.c"
BUILD_DIR = HERE / "_build"
LIB_PATH = BUILD_DIR / "liboracle.so"

KV_F16 = 0
KV_BF16 = 1

_lib = None


def build(force: bool = False, src: Path = SRC, out: Path = LIB_PATH) -> Path:
    """Compile ``src`` into a shared library at ``out`` (gcc, -O2, OpenMP)."""
    out = Path(out)
    if out.exists() and not force and out.stat().st_mtime >= Path(src).stat().st_mtime:
        return out
    out.parent.mkdir(parents=True, exist_ok=True)
    tmp = out.with_suffix(f".{os.getpid()}.tmp.so")
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(tmp), str(src), "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    c = ctypes
    lib.oracle_f16_to_f64.argtypes = [c.c_uint16]
    lib.oracle_f16_to_f64.restype = c.c_double
    lib.oracle_bf16_to_f64.argtypes = [c.c_uint16]
    lib.oracle_bf16_to_f64.restype = c.c_double
    lib.oracle_rope.argtypes = [c.c_void_p, c.c_int, c.c_double, c.c_double, c.c_void_p]
    lib.oracle_rope.restype = None
    lib.oracle_decode.argtypes = [c.c_int, c.c_int, c.c_int, c.c_int, c.c_int64, c.c_void_p, c.c_void_p,
                                  c.c_void_p, c.c_void_p, c.c_int, c.c_double, c.c_double, c.c_void_p,
                                  c.c_void_p]
    lib.oracle_decode.restype = c.c_int
    lib.oracle_project.argtypes = [c.c_int, c.c_int, c.c_int, c.c_void_p, c.c_void_p, c.c_int, c.c_void_p]
    lib.oracle_project.restype = c.c_int
    return lib


def load(path: str | os.PathLike | None = None) -> ctypes.CDLL:
    """Load the oracle library (building the default one if needed).

    ``path`` lets a test load a separately compiled variant of the oracle.
    """
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(str(path)))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(str(build())))
    return _lib


def num_threads() -> int:
    """Threads the OpenMP loop of the oracle uses (OMP_NUM_THREADS, else all cores)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env:
        return int(env)
    return len(os.sched_getaffinity(0))


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def f16_to_f64(bits: int, lib=None) -> float:
    return (lib or load()).oracle_f16_to_f64(int(bits))


def bf16_to_f64(bits: int, lib=None) -> float:
    return (lib or load()).oracle_bf16_to_f64(int(bits))


def rope(x: np.ndarray, pos: float, base: float, lib=None) -> np.ndarray:
    """NeoX rotate-half RoPE of one vector ``x[D]`` at position ``pos`` (fp64)."""
    lib = lib or load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    assert x.ndim == 1 and x.shape[0] % 2 == 0
    y = np.empty_like(x)
    lib.oracle_rope(_ptr(x), x.shape[0], float(pos), float(base), _ptr(y))
    return y


def decode(q: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray, seq_lens: np.ndarray, kv_dtype: int,
           rope_base: float, scale: float = 0.0, group_mask: np.ndarray | None = None,
           out: np.ndarray | None = None, lib=None) -> np.ndarray:
    """Exact decode attention over the LOGICAL token sequence, in fp64.

    q        float32 [B, Hq, D]
    k_bits   uint16  [B, Hkv, Lmax, D]  (raw fp16 / bf16 bit patterns, un-rotated)
    v_bits   uint16  [B, Hkv, Lmax, D]
    seq_lens int32   [B]
    group_mask  optional uint8 [B, Hkv]: compute only those (batch, kv head) groups
    returns  float64 [B, Hq, D]
    """
    lib = lib or load()
    q = np.ascontiguousarray(q, dtype=np.float32)
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v_bits = np.ascontiguousarray(v_bits, dtype=np.uint16)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Hq, D = q.shape
    Bk, Hkv, Lmax, Dk = k_bits.shape
    assert Bk == B and Dk == D and v_bits.shape == k_bits.shape and seq_lens.shape == (B,)
    if out is None:
        out = np.zeros((B, Hq, D), dtype=np.float64)
    gm = None
    if group_mask is not None:
        gm = np.ascontiguousarray(group_mask, dtype=np.uint8).reshape(B * Hkv)
    rc = lib.oracle_decode(B, Hq, Hkv, D, Lmax, _ptr(q), _ptr(k_bits), _ptr(v_bits), _ptr(seq_lens),
                           int(kv_dtype), float(rope_base), float(scale),
                           _ptr(gm) if gm is not None else None, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_decode failed with code {rc}")
    return out


def project(x: np.ndarray, w_bits: np.ndarray, kv_dtype: int, lib=None) -> np.ndarray:
    """y[b][r] = sum_h w[r][h] x[b][h] in fp64.  x float32 [B, H]; w uint16 [R, H]; returns float64 [B, R]."""
    lib = lib or load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    w_bits = np.ascontiguousarray(w_bits, dtype=np.uint16)
    B, H = x.shape
    R, H2 = w_bits.shape
    assert H2 == H
    y = np.empty((B, R), dtype=np.float64)
    rc = lib.oracle_project(B, R, H, _ptr(x), _ptr(w_bits), int(kv_dtype), _ptr(y))
    if rc != 0:
        raise ValueError(f"oracle_project failed with code {rc}")
    return y
