"""Multi-token queries (speculative verification, chunked prefill) over the split cache (needs a B200).

Query i of a sequence with L cached tokens sits at position L + i and attends
to the tokens t < L + i, so it is single-token decode of the sequence cut at
L + i: the oracle checks each query token with its own decode at that length.
"""
import numpy as np
import pytest
import torch

import decode_attention_host_b200 as dkv
import kvgen
import oracle
from tests import gpu_cases as gc

pytestmark = pytest.mark.gpu


def _run(w: kvgen.Workload, tq: int, seed: int, lens=None, stride=None):
    lens = kvgen.gen_seq_lens(w) if lens is None else np.asarray(lens, dtype=np.int32)
    case = gc.Case(w, lens=lens + tq - 1, max_batch=w.batch * tq, stride=stride)
    q = np.random.default_rng(seed).standard_normal((w.batch, tq, w.num_q_heads, w.head_dim)).astype(np.float32)
    case.kv.seq_lens_dev.copy_(torch.from_numpy(lens))
    out = torch.full((w.batch, tq, w.num_q_heads, w.head_dim), float("nan"), device="cuda")
    case.attn.multi(torch.from_numpy(q).cuda(), case.kv, out)
    torch.cuda.synchronize()
    assert case.attn.status() == 0
    return case, lens, q, out.cpu().numpy()


def _check(case, lens, q, got):
    w = case.w
    odt = gc.oracle_dtype(w)
    for i in range(q.shape[1]):
        want = oracle.decode(q[:, i], case.k, case.v, lens + i, odt, w.rope_base)
        err = gc.max_err(got[:, i], want)
        assert err <= gc.TOL, f"query token {i}: max abs err {err:.3e}"


@pytest.mark.parametrize("tq", [1, 2, 4])
def test_gqa_speculative_queries(tq):
    w = kvgen.LLAMA3_8B.replace(name=f"multi_gqa_{tq}", batch=3, ctx=(200, 1500), seed=60 + tq)
    case, lens, q, got = _run(w, tq, 70 + tq)
    _check(case, lens, q, got)
    case.free()


@pytest.mark.parametrize("tq", [8, 16])
def test_mha_chunk_queries_fp16(tq):
    w = kvgen.OPT_6_7B.replace(name=f"multi_mha_{tq}", batch=2, num_q_heads=4, num_kv_heads=4, ctx=(50, 700),
                               seed=80 + tq)
    case, lens, q, got = _run(w, tq, 90 + tq)
    _check(case, lens, q, got)
    case.free()


def test_all_in_hbm_with_two_units_per_warp():
    """Every block in HBM and a table capacity of 4736 blocks of 16 tokens: the plan takes two units per warp
    of at least 1024 tokens (twice the splits of one unit per warp), so with sequences of 100-3000 tokens most
    units are empty and the rest hold the sequences' first blocks."""
    w = kvgen.LLAMA3_8B.replace(name="multi_refined", batch=4, ctx=(100, 3000), host_fraction=0.0, seed=97)
    case, lens, q, got = _run(w, 4, 98, stride=4736)
    warps = 8 * torch.cuda.get_device_properties(0).multi_processor_count
    per = w.batch * w.num_kv_heads
    one = -(-4736 // -(-4736 // max(1, warps // per)))
    nsplit, bps = case.attn.plan(w.batch, case.kv.stride)
    assert nsplit > one and bps * w.block_size >= 1024 and nsplit * bps >= 4736
    assert case.kv.host_split == 0 and case.attn.launches() == 2
    _check(case, lens, q, got)
    case.free()


def test_head_dim_64_and_empty_prefix():
    w = kvgen.TINY_GQA.replace(name="multi_d64", batch=3, num_q_heads=4, num_kv_heads=2, ctx=(0, 300), seed=95)
    case, lens, q, got = _run(w, 3, 96, lens=[0, 17, 300])
    _check(case, lens, q, got)
    assert not got[0, 0].any(), "the first query of an empty prefix sees no token"
    case.free()


def test_one_query_token_is_decode():
    w = kvgen.LLAMA3_8B.replace(name="multi_one", batch=2, ctx=(500, 2000), seed=97)
    case, lens, q, got = _run(w, 1, 98)
    case.q_dev.copy_(torch.from_numpy(q[:, 0]))
    out = torch.empty_like(case.q_dev)
    case.attn(case.q_dev, case.kv, out)
    torch.cuda.synchronize()
    assert np.abs(out.cpu().numpy() - got[:, 0]).max() <= 1e-5
    case.free()


def test_argument_limits():
    w = kvgen.LLAMA3_8B.replace(name="multi_args", batch=2, ctx=300, seed=99)
    case = gc.Case(w, max_batch=4)
    kv = case.kv
    q = torch.zeros(2, 5, w.num_q_heads, w.head_dim, device="cuda")
    out = torch.zeros_like(q)
    for tq, batch in ((5, 2), (2, 3), (0, 2)):   # 5*4 > 16 rows; 3*2 > max_batch 4; no query
        with pytest.raises(dkv.DkvError) as e:
            dkv.dkv_attn_decode_multi(case.attn.handle, tq, q, kv.k_host.ptr, kv.v_host.ptr, kv.k_dev, kv.v_dev,
                                      kv.table_dev, kv.seq_lens_dev, kv.host_split, out,
                                      torch.cuda.current_stream().cuda_stream, batch, kv.stride, kv.num_dev_blocks)
        assert e.value.code == dkv.DKV_ERR_INVALID_ARG
    case.free()
