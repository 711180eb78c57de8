"""CUDA path vs the fp64 oracle, element by element, through the C ABI (needs a B200)."""
import ctypes

import numpy as np
import pytest
import torch

import decode_attention_host_b200 as dkv
import kvgen
from tests import gpu_cases as gc
from tests.test_golden import load_golden

pytestmark = pytest.mark.gpu


def check(case: gc.Case, tol=gc.TOL, test: str = "parity"):
    got = case.run()
    want = case.oracle()
    err = gc.max_err(got, want)
    assert case.attn.status() == 0
    assert err <= tol, f"{case.w.name}: max abs err {err:.3e}"
    gc.record(test, case.w.name, err)
    return got, err


def test_tiny_gqa_matches_oracle_and_golden():
    case = gc.Case(kvgen.TINY_GQA)
    got, err = check(case, test="test_tiny_gqa_matches_oracle_and_golden")
    _, golden = load_golden()
    assert np.abs(got[0] - golden).max() <= gc.TOL
    # tokens 0..255 on the host, 256..511 in HBM: the pool lists, both split kernels and the merge ran
    assert case.kv.host_bytes == case.kv.dev_bytes == 256 * 2 * 64 * 2
    assert case.attn.launches() == 4
    case.free()


@pytest.mark.parametrize("name,kw", [
    ("llama3_8b", dict(batch=2, ctx=3000)),                           # ragged tail, random half on host
    ("long_ctx", dict(ctx=70000)),                                     # 64-token blocks, oldest 90% host
    ("opt_6_7b", dict(batch=4, ctx=(100, 3000))),                      # MHA, ragged, shuffled ids, 75% host
    ("opt_6_7b_norope", dict(batch=3, ctx=(20, 900), rope_base=0.0)),  # the same shape without rotation
])
def test_reduced_workloads(name, kw):
    base = kvgen.get(name.replace("_norope", ""))
    case = gc.Case(base.replace(**kw))
    check(case, test="test_reduced_workloads")
    case.free()


@pytest.mark.parametrize("f", kvgen.SWEEP_HOST_FRACTION)
def test_sweep_4k_cells_full_size(f):
    """The 4k-context cells of the sweep at their full size (B=4, outlier keys x8)."""
    cell = next(c for c in kvgen.sweep_cells() if c.max_ctx == 4096 and c.host_fraction == f)
    case = gc.Case(cell)
    check(case, test="test_sweep_4k_cells_full_size")
    if f == 0.0:
        assert case.kv.host_split == 0 and case.attn.launches() == 2
    if f == 1.0:
        assert case.kv.num_dev_blocks == 0 and case.attn.launches() == 2
    case.free()


@pytest.mark.parametrize("d,g,dt", [(64, 1, kvgen.F16), (64, 2, kvgen.BF16), (128, 1, kvgen.BF16),
                                    (128, 2, kvgen.F16), (64, 4, kvgen.BF16), (128, 4, kvgen.F16)])
def test_every_head_shape_and_dtype(d, g, dt):
    w = kvgen.LLAMA3_8B.replace(name=f"shape_d{d}_g{g}", batch=3, num_kv_heads=2, num_q_heads=2 * g, head_dim=d,
                                kv_dtype=dt, ctx=(1, 700), block_size=32, seed=40 + d + g)
    check(gc.Case(w), test="test_every_head_shape_and_dtype")


def test_edge_lengths_in_one_batch():
    """Empty, single-token, tile- and block-boundary and ragged sequences side by side."""
    lens = [0, 1, 15, 16, 17, 31, 32, 33, 64, 1000]
    w = kvgen.LLAMA3_8B.replace(name="edges", batch=len(lens), ctx=max(lens), seed=77)
    case = gc.Case(w, lens=lens)
    got, _ = check(case, test="test_edge_lengths_in_one_batch")
    assert not got[0].any(), "an empty sequence must give a zero row"
    case.free()


def test_result_independent_of_placement_and_block_order():
    w = kvgen.LLAMA3_8B.replace(name="placements", batch=2, ctx=2500, seed=91)
    outs = []
    for f, placement, shuffle in ((0.0, dkv.DKV_PLACE_RANDOM, False), (1.0, dkv.DKV_PLACE_RANDOM, False),
                                  (0.37, dkv.DKV_PLACE_RANDOM, True), (0.8, dkv.DKV_PLACE_PREFIX_HOST, True),
                                  (0.5, dkv.DKV_PLACE_RANDOM, True)):
        case = gc.Case(w, host_fraction=f, placement=placement, shuffle=shuffle, plan_seed=int(f * 100) + 1)
        outs.append(case.run())
        case.free()
    want = gc.Case(w, host_fraction=0.0).oracle()
    for o in outs:
        assert gc.max_err(o, want) <= gc.TOL
        assert np.abs(o - outs[0]).max() <= 2e-5   # only fp32 summation order differs


def test_batch_order_does_not_matter():
    w = kvgen.OPT_6_7B.replace(name="batch_order", batch=5, ctx=(50, 600), seed=5)
    case = gc.Case(w)
    a = case.run()
    perm = np.array([3, 0, 4, 1, 2])
    w2 = w
    case2 = gc.Case.__new__(gc.Case)
    case2.w, case2.q, case2.lens = w2, case.q[perm].copy(), case.lens[perm].copy()
    case2.k, case2.v = case.k[perm].copy(), case.v[perm].copy()
    case2.kv = dkv.PagedKV(case2.k, case2.v, case2.lens, w.block_size, dkv.DKV_PLACE_RANDOM, 0.75, True, 8)
    case2.attn = case.attn
    case2.q_dev = torch.from_numpy(case2.q).cuda()
    case2.out = torch.empty_like(case2.q_dev)
    b = case2.run()
    assert np.abs(b - a[perm]).max() <= 2e-5


def test_repeated_calls_are_bitwise_identical_and_graph_capturable():
    w = kvgen.LLAMA3_8B.replace(name="graph", batch=2, ctx=1500, seed=12)
    case = gc.Case(w)
    a = case.run()
    b = case.run()
    assert np.array_equal(a, b)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    case.out.fill_(float("nan"))
    with torch.cuda.graph(g, stream=s):
        case.attn(case.q_dev, case.kv, case.out, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(case.out.cpu().numpy(), a)
    case.free()


def test_bad_block_id_sets_status_and_poisons_only_its_sequence():
    w = kvgen.LLAMA3_8B.replace(name="bad_id", batch=3, ctx=600, seed=3)
    case = gc.Case(w)
    good = case.run()
    table = case.kv.table.copy()
    table[1, 7] = case.kv.host_split + case.kv.num_dev_blocks + 5
    case.kv.table_dev.copy_(torch.from_numpy(table))
    out = case.run()
    assert case.attn.status() == dkv.DKV_STATUS_BAD_BLOCK_ID
    assert np.isnan(out[1]).all()
    assert np.array_equal(out[[0, 2]], good[[0, 2]])
    assert case.attn.status() == 0   # reading the status clears it
    case.free()


def test_bad_seq_len_sets_status():
    w = kvgen.LLAMA3_8B.replace(name="bad_len", batch=2, ctx=300, seed=4)
    case = gc.Case(w)
    good = case.run()
    lens = case.lens.copy()
    lens[0] = case.kv.stride * w.block_size + 1
    case.kv.seq_lens_dev.copy_(torch.from_numpy(lens))
    out = case.run()
    assert case.attn.status() == dkv.DKV_STATUS_BAD_SEQ_LEN
    assert np.isnan(out[0]).all() and np.array_equal(out[1], good[1])
    case.free()


def test_host_side_argument_errors():
    w = kvgen.LLAMA3_8B.replace(name="args", batch=1, ctx=200, seed=6)
    case = gc.Case(w)
    kv, h = case.kv, case.attn.handle
    pageable = np.zeros(1 << 20, dtype=np.uint16)
    args = dict(q=case.q_dev, k_host=kv.k_host.ptr, v_host=kv.v_host.ptr, k_dev=kv.k_dev, v_dev=kv.v_dev,
                block_table=kv.table_dev, seq_lens=kv.seq_lens_dev, host_split=kv.host_split, out=case.out,
                stream=torch.cuda.current_stream().cuda_stream, batch=1, block_table_stride=kv.stride,
                num_dev_blocks=kv.num_dev_blocks)
    bad = [dict(k_host=pageable), dict(k_host=kv.k_dev.data_ptr()), dict(k_dev=kv.k_host.ptr), dict(batch=2),
           dict(block_table_stride=0), dict(host_split=-1), dict(q=None), dict(k_dev=None),
           dict(q=case.q_dev.data_ptr() + 4), dict(k_dev=kv.k_dev.data_ptr() + 2),
           dict(v_host=kv.v_host.ptr + 8)]
    for override in bad:
        a = dict(args, **override)
        with pytest.raises(dkv.DkvError) as e:
            dkv.dkv_attn_decode(h, **a)
        assert e.value.code == dkv.DKV_ERR_INVALID_ARG, override
    dkv.dkv_attn_decode(h, **args)   # the handle still works
    torch.cuda.synchronize()
    case.free()


def test_create_on_a_missing_device_fails_cleanly():
    cfg = dkv.DkvConfig(4, 1, 64, 16, dkv.DKV_KV_F16, 1e4, 0.0, 1, 32, torch.cuda.device_count() + 3, 0)
    hd = ctypes.c_void_p()
    assert dkv.lib.dkv_create(ctypes.byref(cfg), ctypes.byref(hd)) == dkv.DKV_ERR_INVALID_ARG


# ----------------------------------------------------------------------------- full sizes, bench launch config

@pytest.mark.parametrize("name,groups", [("llama3_8b", 6), ("opt_6_7b", 6), ("long_ctx", 3)])
def test_full_size_sampled_against_oracle(name, groups):
    """Full-size workloads, bench launch configuration; the oracle checks sampled (batch, kv head) groups."""
    w = kvgen.get(name)
    case = gc.Case(w)
    got = case.run()
    assert np.isfinite(got).all()
    assert case.attn.status() == 0
    mask = gc.sampled_groups(w, groups, 123)
    err = gc.sampled_err(w, got, case.oracle(group_mask=mask), mask)
    gc.record("test_full_size_sampled_against_oracle", name, err, f"{int(mask.sum())} of {mask.size}")
    assert err <= gc.TOL, f"{name}: {err:.3e}"
    case.free()


@pytest.mark.parametrize("name,groups", [("opt_6_7b", 6), ("llama3_8b", 6), ("long_ctx", 3)])
def test_full_size_all_in_hbm_sampled_against_oracle(name, groups):
    """The named workloads with every block in HBM: the HBM kernel alone, with the plan of two units per warp
    when the batch holds several sequences (opt_6_7b: 16 sequences of 1k-16k tokens, 4 splits of 256
    blocks) and one per warp for a single sequence (long_ctx).  Sampled groups against the oracle."""
    w = kvgen.get(name).replace(host_fraction=0.0)
    case = gc.Case(w)
    got = case.run()
    assert np.isfinite(got).all()
    assert case.attn.status() == 0 and case.kv.host_split == 0 and case.attn.launches() == 2
    if name == "opt_6_7b":
        # 1024 table blocks per sequence, 16 x 32 (sequence, kv head) pairs; one unit per warp of 2 CTAs x 4
        # warps per SM would give floor(8 SMs / 512) splits, two units per warp twice that
        warps = 8 * torch.cuda.get_device_properties(0).multi_processor_count
        one = max(1, warps // 512)
        nsplit, bps = case.attn.plan(w.batch, case.kv.stride)
        assert nsplit == -(-1024 // -(-1024 // (2 * one))) and bps * 16 >= 1024
    mask = gc.sampled_groups(w, groups, 321)
    err = gc.sampled_err(w, got, case.oracle(group_mask=mask), mask)
    gc.record("test_full_size_all_in_hbm_sampled_against_oracle", name + "_h0", err,
              f"{int(mask.sum())} of {mask.size}")
    assert err <= gc.TOL, f"{name}: {err:.3e}"
    case.free()


@pytest.mark.parametrize("host_fraction", [0.01, 0.03])
def test_small_host_share_full_size_sampled(host_fraction):
    """A placement near the offload planner's balance point: 1% (light host stream of 8 CTAs beside an HBM
    launch planned for the warps it leaves) and 3% (16 CTAs) of the 64k cell's blocks on the host."""
    w = kvgen.get("sweep_L65536_f0").replace(name=f"sweep_L65536_f{host_fraction:g}", host_fraction=host_fraction)
    case = gc.Case(w)
    got = case.run()
    assert np.isfinite(got).all()
    assert case.attn.status() == 0 and case.kv.host_split > 0 and case.attn.launches() == 4
    mask = gc.sampled_groups(w, 3, 77)
    err = gc.sampled_err(w, got, case.oracle(group_mask=mask), mask)
    gc.record("test_small_host_share_full_size_sampled", w.name, err, f"{int(mask.sum())} of {mask.size}")
    assert err <= gc.TOL, f"{w.name}: {err:.3e}"
    case.free()


@pytest.mark.parametrize("cell", [c.name for c in kvgen.sweep_cells()])
def test_every_sweep_cell_full_size_sampled(cell):
    """All 20 context x host-fraction cells at full size (B=4, 1% outlier keys x8), in the bench's launch
    configuration: three sampled (batch, kv head) groups of each against the oracle, element by element,
    and every output row finite."""
    w = kvgen.get(cell)
    case = gc.Case(w)
    got = case.run()
    assert np.isfinite(got).all()
    assert case.attn.status() == 0
    f = w.host_fraction
    if f == 0.0:
        assert case.kv.host_split == 0 and case.attn.launches() == 2
    elif f == 1.0:
        assert case.kv.num_dev_blocks == 0 and case.attn.launches() == 2
    else:
        assert case.kv.host_split > 0 and case.kv.num_dev_blocks > 0 and case.attn.launches() == 4
    mask = gc.sampled_groups(w, 3, w.seed)
    err = gc.sampled_err(w, got, case.oracle(group_mask=mask), mask)
    gc.record("test_every_sweep_cell_full_size_sampled", cell, err, f"{int(mask.sum())} of {mask.size}")
    assert err <= gc.TOL, f"{cell}: {err:.3e}"
    case.free()


@pytest.mark.parametrize("name,kw", [
    ("staged", dict(batch=2, ctx=2100, seed=31)),                            # random half on the host
    ("staged_ragged", dict(batch=5, ctx=(1, 3000), seed=32, host_fraction=0.8, shuffle=True)),
])
def test_staged_prefetch_comparator_matches_oracle(name, kw):
    """Copying the host pool into HBM first (the design the method argues against) gives the oracle's answer,
    and the zero-copy path's up to fp32 summation order."""
    w = kvgen.LLAMA3_8B.replace(name=name, **kw)
    case = gc.Case(w)
    zero_copy = case.run()
    want = case.oracle()
    blk = w.num_kv_heads * w.block_size * w.head_dim
    ks = torch.empty(case.kv.host_split * blk, dtype=torch.int16, device="cuda")
    vs = torch.empty_like(ks)
    out = torch.full_like(case.q_dev, float("nan"))
    case.attn.staged(case.q_dev, case.kv, out, ks, vs)
    torch.cuda.synchronize()
    assert case.attn.status() == 0
    staged = out.cpu().numpy()
    err = gc.max_err(staged, want)
    gc.record("test_staged_prefetch_comparator_matches_oracle", name, err)
    assert err <= gc.TOL, f"staged: {err:.3e}"
    # both launches of the staged path have the whole GPU, so its splits differ from the zero-copy
    # path's (whose host kernel has 16 CTAs): the two agree up to fp32 summation order
    assert np.abs(staged - zero_copy).max() <= 2e-5
    # the staging pool now holds a byte copy of the host pool
    assert np.array_equal(ks.cpu().numpy().view(np.uint16), case.kv.k_host.array[:ks.numel()])
    with pytest.raises(dkv.DkvError) as e:
        case.attn.staged(case.q_dev, case.kv, out, None, None)
    assert e.value.code == dkv.DKV_ERR_INVALID_ARG
    case.free()


@pytest.mark.parametrize("block_size,d,placement", [
    (256, 64, "prefix_host"),     # the tiny config with one 256-token block per side
    (512, 128, "random"),
    (1024, 128, "random"),        # the largest block: 64 tiles per block
    (1024, 64, "prefix_host"),
])
def test_large_blocks(block_size, d, placement):
    """Blocks of many tiles: every tile of a block is addressed from its own offset inside the block."""
    if d == 64 and placement == "prefix_host" and block_size == 256:
        w = kvgen.TINY_GQA.replace(name="tiny_s256", block_size=256)
    else:
        w = kvgen.LLAMA3_8B.replace(name=f"blocks_s{block_size}_d{d}", batch=3, head_dim=d, ctx=(700, 5000),
                                    block_size=block_size, placement=placement, host_fraction=0.5, seed=block_size + d)
    case = gc.Case(w)
    check(case, test="test_large_blocks")
    if w.name == "tiny_s256":
        assert case.kv.host_split == 1 and case.kv.num_dev_blocks == 1
    case.free()


def test_gqa_equals_mha_with_repeated_kv_heads():
    """G query heads sharing one KV head give what G copies of that KV head give to one query head each."""
    w = kvgen.LLAMA3_8B.replace(name="gqa", batch=2, num_q_heads=8, num_kv_heads=2, ctx=(300, 1400), seed=61)
    gqa = gc.Case(w)
    a = gqa.run()
    g = w.num_q_heads // w.num_kv_heads
    wm = w.replace(name="gqa_as_mha", num_kv_heads=w.num_q_heads)
    mha = gc.Case.__new__(gc.Case)
    mha.w, mha.q, mha.lens = wm, gqa.q.copy(), gqa.lens.copy()
    mha.k, mha.v = np.repeat(gqa.k, g, axis=1), np.repeat(gqa.v, g, axis=1)
    mha.kv = dkv.PagedKV(mha.k, mha.v, mha.lens, wm.block_size, gc.placement_code(wm), wm.host_fraction, wm.shuffle,
                         wm.seed)
    mha.attn = gc.attention_for(wm, max_blocks=max(wm.max_blocks_per_seq(), mha.kv.stride))
    mha.q_dev = torch.from_numpy(mha.q).cuda()
    mha.out = torch.empty_like(mha.q_dev)
    b = mha.run()
    assert mha.attn.status() == 0
    assert np.abs(a - b).max() <= 2e-5   # different kernel instances: only fp32 summation order differs
    assert gc.max_err(a, gqa.oracle()) <= gc.TOL
    gqa.free()
    mha.free()


def test_output_is_linear_in_v():
    """V doubled (exact in 16 bits) doubles the output bit for bit: the weights do not depend on V."""
    w = kvgen.LLAMA3_8B.replace(name="lin_v", batch=2, ctx=(200, 2100), seed=62)
    case = gc.Case(w)
    a = case.run()
    v2 = kvgen.to_bits(kvgen.bits_to_f32(case.v, w.kv_dtype) * 2.0, w.kv_dtype)
    twice = gc.Case.__new__(gc.Case)
    twice.w, twice.q, twice.lens, twice.k, twice.v = w, case.q, case.lens, case.k, v2
    twice.kv = dkv.PagedKV(case.k, v2, case.lens, w.block_size, gc.placement_code(w), w.host_fraction, w.shuffle,
                           w.seed)
    twice.attn, twice.q_dev = case.attn, case.q_dev
    twice.out = torch.empty_like(case.q_dev)
    b = twice.run()
    assert np.array_equal(b, 2.0 * a)
    case.free()
    twice.free()
