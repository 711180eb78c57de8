"""Shared set-up for the GPU tests: build a paged cache from a seeded workload, run
the CUDA path through the C ABI, and run the fp64 oracle on the same inputs."""
from __future__ import annotations

import functools
import json
import os

import numpy as np
import torch

import decode_attention_host_b200 as dkv
import kvgen
import oracle

TOL = 2e-3   # max-abs error against the fp64 oracle for 16-bit K/V with fp32 accumulation


def oracle_dtype(w: kvgen.Workload) -> int:
    return oracle.KV_BF16 if w.kv_dtype == kvgen.BF16 else oracle.KV_F16


def lib_dtype(w: kvgen.Workload) -> int:
    return dkv.DKV_KV_BF16 if w.kv_dtype == kvgen.BF16 else dkv.DKV_KV_F16


def placement_code(w: kvgen.Workload) -> int:
    return dkv.DKV_PLACE_PREFIX_HOST if w.placement == "prefix_host" else dkv.DKV_PLACE_RANDOM


@functools.lru_cache(maxsize=None)
def attention(hq, hkv, d, s, dt, base, max_batch, max_blocks, host_ctas=0, scale=0.0) -> dkv.DecodeAttention:
    return dkv.DecodeAttention(hq, hkv, d, s, dt, base, max_batch, max_blocks, scale=scale, host_ctas=host_ctas)


def attention_for(w: kvgen.Workload, max_blocks: int | None = None, host_ctas: int = 0, max_batch=None):
    return attention(w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, lib_dtype(w), float(w.rope_base),
                     max_batch or w.batch, max_blocks or w.max_blocks_per_seq(), host_ctas)


class Case:
    """Inputs of one workload, its paged cache and the CUDA output."""

    def __init__(self, w: kvgen.Workload, lens=None, host_fraction=None, placement=None, shuffle=None,
                 plan_seed=None, stride=None, host_ctas=0, max_batch=None):
        self.w = w
        self.q = kvgen.gen_q(w)
        self.lens = kvgen.gen_seq_lens(w) if lens is None else np.asarray(lens, dtype=np.int32)
        self.k, self.v = kvgen.gen_kv(w, self.lens, lmax=max(1, int(self.lens.max(initial=0))))
        self.kv = dkv.PagedKV(self.k, self.v, self.lens, w.block_size,
                              placement_code(w) if placement is None else placement,
                              w.host_fraction if host_fraction is None else host_fraction,
                              w.shuffle if shuffle is None else shuffle,
                              w.seed if plan_seed is None else plan_seed, stride=stride)
        self.attn = attention_for(w, max_blocks=max(w.max_blocks_per_seq(), self.kv.stride), host_ctas=host_ctas,
                                  max_batch=max_batch)
        self.q_dev = torch.from_numpy(self.q).cuda()
        self.out = torch.full_like(self.q_dev, float("nan"))

    def run(self, stream=None) -> np.ndarray:
        self.attn(self.q_dev, self.kv, self.out, stream=stream)
        torch.cuda.synchronize()
        return self.out.cpu().numpy()

    def oracle(self, group_mask=None) -> np.ndarray:
        return oracle.decode(self.q, self.k, self.v, self.lens, oracle_dtype(self.w), self.w.rope_base,
                             group_mask=group_mask)

    def free(self):
        self.kv.free()


def max_err(got: np.ndarray, want: np.ndarray) -> float:
    assert got.shape == want.shape
    assert np.isfinite(got).all(), "non-finite output"
    return float(np.abs(got.astype(np.float64) - want).max())


def record(test: str, workload: str, err: float, groups: str = "all") -> None:
    """Append one measured parity error to the JSON-lines file named by DKV_PARITY_LOG, if set."""
    log = os.environ.get("DKV_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps({"test": test, "workload": workload, "max_abs_err": err, "groups": groups,
                                "tolerance": TOL}) + "\n")


def sampled_groups(w: kvgen.Workload, n: int, seed: int) -> np.ndarray:
    """uint8 [B, Hkv] mask of n (batch, kv head) groups drawn without replacement."""
    rng = np.random.default_rng(seed)
    mask = np.zeros((w.batch, w.num_kv_heads), dtype=np.uint8)
    for i in rng.choice(w.batch * w.num_kv_heads, size=min(n, w.batch * w.num_kv_heads), replace=False):
        mask.flat[i] = 1
    return mask


def sampled_err(w: kvgen.Workload, got: np.ndarray, want: np.ndarray, mask: np.ndarray) -> float:
    """Max abs error over the query-head rows of the masked groups."""
    rows = np.repeat(mask.astype(bool), w.group_size, axis=1)
    assert np.isfinite(got[rows]).all(), "non-finite output"
    return float(np.abs(got[rows].astype(np.float64) - want[rows]).max())
