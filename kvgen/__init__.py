"""Seeded synthetic decode-attention workloads.

This module only draws inputs: the query vectors, the un-rotated K/V values
of every logical token, the ragged context lengths and the outlier pattern.
It holds none of the method's arithmetic (no RoPE, no attention, no paging or
placement), so both the fp64 oracle and the CUDA library can be fed from it
without sharing code.  Placement of blocks between host and device memory is
the partitioner's job (a product routine) and is not drawn here.

Workload recipe (shapes and distributions of the five benchmark settings):

========  ======================================================================
name      recipe
========  ======================================================================
tiny_gqa  B=1, Hq=4, Hkv=1, D=64, L=512, fp16 K/V ~ N(0,1), q fp32 ~ N(0,1),
          RoPE base 1e4, 16-token blocks, tokens 0..255 host / 256..511 HBM,
          seed 0
llama3_8b B=8, Hq=32, Hkv=8, D=128, L=32768, bf16 K/V ~ N(0,1), base 5e5,
          16-token blocks, half the blocks of each sequence on the host at
          random, seed 1
long_ctx  B=1, Hq=32, Hkv=8, D=128, L=1,048,576, bf16 ~ N(0,1), base 5e5,
          64-token blocks, oldest 90% of blocks host, newest 10% HBM, seed 2
opt_6_7b  B=16, Hq=Hkv=32 (MHA), D=128, L_b ~ U{1024..16384}, fp16 K/V with
          standard deviation 0.5, base 1e4 (and a no-RoPE variant), 16-token
          blocks, shuffled block ids, 75% host at random, seed 3
sweep     B=4, Hq=32, Hkv=8, D=128, bf16, 32-token blocks,
          L in {4k, 16k, 64k, 256k} x host fraction {0, .25, .5, .75, 1};
          K/V ~ N(0,1), each token independently an outlier with p = 0.01 whose
          stored key is multiplied by 8 (exact in bf16); seed 5 + cell index
========  ======================================================================

Values are drawn in fp32 and rounded to the 16-bit storage type with
round-to-nearest-even; the stored 16-bit values are the ground truth for
every consumer.  Each (tensor, batch, kv head) slice has its own numpy
Generator stream keyed by (seed, tensor id, b, h), so any slice can be redrawn
on its own.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Iterator

import numpy as np

F16 = "f16"
BF16 = "bf16"

# stream ids inside a seed
_Q, _K, _V, _LENS, _OUTLIER = 0, 1, 2, 3, 4


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    ctx: int | tuple[int, int]          # fixed length, or inclusive (lo, hi) for ragged lengths
    kv_dtype: str
    kv_std: float
    rope_base: float
    block_size: int
    placement: str                      # "prefix_host" | "random"
    host_fraction: float
    shuffle: bool
    seed: int
    outlier_p: float = 0.0
    outlier_scale: float = 1.0

    @property
    def group_size(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_ctx(self) -> int:
        return self.ctx[1] if isinstance(self.ctx, tuple) else self.ctx

    def max_blocks_per_seq(self) -> int:
        return -(-self.max_ctx // self.block_size)

    def kv_bytes_per_token(self) -> int:
        """K + V bytes of one token over all KV heads (16-bit storage)."""
        return 2 * self.num_kv_heads * self.head_dim * 2

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


TINY_GQA = Workload("tiny_gqa", 1, 4, 1, 64, 512, F16, 1.0, 1e4, 16, "prefix_host", 0.5, False, 0)
LLAMA3_8B = Workload("llama3_8b", 8, 32, 8, 128, 32768, BF16, 1.0, 5e5, 16, "random", 0.5, False, 1)
LONG_CTX = Workload("long_ctx", 1, 32, 8, 128, 1 << 20, BF16, 1.0, 5e5, 64, "prefix_host", 0.9, False, 2)
OPT_6_7B = Workload("opt_6_7b", 16, 32, 32, 128, (1024, 16384), F16, 0.5, 1e4, 16, "random", 0.75, True, 3)

SWEEP_CTX = (4096, 16384, 65536, 262144)
SWEEP_HOST_FRACTION = (0.0, 0.25, 0.5, 0.75, 1.0)


def sweep_cells() -> list[Workload]:
    """The 20 cells of the context x host-fraction sweep (seed 5 + cell index)."""
    cells = []
    for i, (ctx, f) in enumerate((c, f) for c in SWEEP_CTX for f in SWEEP_HOST_FRACTION):
        cells.append(Workload(f"sweep_L{ctx}_f{f:g}", 4, 32, 8, 128, ctx, BF16, 1.0, 5e5, 32, "random", f,
                              False, 5 + i, outlier_p=0.01, outlier_scale=8.0))
    return cells


CONFIGS = {w.name: w for w in (TINY_GQA, LLAMA3_8B, LONG_CTX, OPT_6_7B)}


def get(name: str) -> Workload:
    if name in CONFIGS:
        return CONFIGS[name]
    for w in sweep_cells():
        if w.name == name:
            return w
    raise KeyError(name)


# ----------------------------------------------------------------------------- rounding

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bfloat16 (nearest, ties to even); returns the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to IEEE binary16 (numpy's nearest-even conversion); returns the bits."""
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def bits_to_f32(bits: np.ndarray, kv_dtype: str) -> np.ndarray:
    """Widen 16-bit storage to fp32 (exact)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if kv_dtype == BF16:
        return (bits.astype(np.uint32) << 16).view(np.float32)
    return bits.view(np.float16).astype(np.float32)


def to_bits(x: np.ndarray, kv_dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(x) if kv_dtype == BF16 else f32_to_f16_bits(x)


# ----------------------------------------------------------------------------- draws

def _rng(w: Workload, stream: int, *key: int) -> np.random.Generator:
    return np.random.default_rng([w.seed, stream, *key])


def gen_q(w: Workload) -> np.ndarray:
    """Query vectors, fp32 [B, Hq, D] ~ N(0, 1)."""
    return _rng(w, _Q).standard_normal((w.batch, w.num_q_heads, w.head_dim), dtype=np.float32)


def gen_seq_lens(w: Workload) -> np.ndarray:
    """Context length of each sequence, int32 [B]."""
    if isinstance(w.ctx, tuple):
        lo, hi = w.ctx
        return _rng(w, _LENS).integers(lo, hi + 1, size=w.batch).astype(np.int32)
    return np.full(w.batch, w.ctx, dtype=np.int32)


def outlier_tokens(w: Workload, b: int, length: int) -> np.ndarray:
    """Boolean [length]: tokens of sequence b whose stored keys (all KV heads) are scaled."""
    if w.outlier_p <= 0.0:
        return np.zeros(length, dtype=bool)
    return _rng(w, _OUTLIER, b).random(length) < w.outlier_p


def gen_kv_slice(w: Workload, tensor: str, b: int, h: int, length: int, chunk: int = 1 << 22,
                 out: np.ndarray | None = None) -> np.ndarray:
    """Stored bits of K or V for (b, h), tokens 0..length-1: uint16 [length, D] (written into ``out``
    when given)."""
    stream = _K if tensor == "k" else _V
    rng = _rng(w, stream, b, h)
    if out is None:
        out = np.empty((length, w.head_dim), dtype=np.uint16)
    assert out.shape == (length, w.head_dim) and out.dtype == np.uint16 and out.flags.c_contiguous
    flat = out.reshape(-1)
    n = flat.size
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        x = rng.standard_normal(e - s, dtype=np.float32)
        if w.kv_std != 1.0:
            x *= np.float32(w.kv_std)
        flat[s:e] = to_bits(x, w.kv_dtype)
    if tensor == "k" and w.outlier_p > 0.0:
        mask = outlier_tokens(w, b, length)
        if mask.any():
            scaled = bits_to_f32(out[mask], w.kv_dtype) * np.float32(w.outlier_scale)
            out[mask] = to_bits(scaled, w.kv_dtype)   # a power-of-two scale is exact
    return out


def gen_kv(w: Workload, seq_lens: np.ndarray | None = None, lmax: int | None = None
           ) -> tuple[np.ndarray, np.ndarray]:
    """Logical K and V bits, uint16 [B, Hkv, Lmax, D]; tokens >= L_b are zero."""
    if seq_lens is None:
        seq_lens = gen_seq_lens(w)
    if lmax is None:
        lmax = int(max(int(seq_lens.max()) if len(seq_lens) else 0, 0))
    shape = (w.batch, w.num_kv_heads, lmax, w.head_dim)
    k = np.zeros(shape, dtype=np.uint16)
    v = np.zeros(shape, dtype=np.uint16)
    # every (tensor, b, h) slice has its own stream, so the slices are drawn on
    # a thread pool (numpy's generators and ufuncs release the GIL) with
    # results identical to a serial loop
    jobs = [(t, b, h) for b in range(w.batch) for h in range(w.num_kv_heads) for t in ("k", "v")]

    def draw(job):
        t, b, h = job
        L = int(seq_lens[b])
        gen_kv_slice(w, t, b, h, L, out=(k if t == "k" else v)[b, h, :L])

    workers = max(1, min(len(jobs), len(os.sched_getaffinity(0)), 32))
    if workers == 1 or k.nbytes < (64 << 20):
        for j in jobs:
            draw(j)
    else:
        with ThreadPoolExecutor(workers) as pool:
            list(pool.map(draw, jobs))
    return k, v


def iter_groups(w: Workload) -> Iterator[tuple[int, int]]:
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            yield b, h
