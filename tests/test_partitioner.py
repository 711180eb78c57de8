"""The host/device block partitioner and the KV packer (host code of libdkv, no GPU)."""
import numpy as np
import pytest

import decode_attention_host_b200 as dkv
import kvgen


def plan(lens, S, placement, f, shuffle=False, seed=0, stride=None):
    lens = np.asarray(lens, dtype=np.int32)
    stride = stride or max(1, int(-(-lens.max() // S)))
    table = np.zeros((len(lens), stride), dtype=np.int32)
    res = dkv.dkv_plan_blocks(dkv.DkvPlanParams(S, placement, f, int(shuffle), seed), lens, table)
    return table, res


def nblocks(lens, S):
    return [int(-(-L // S)) for L in lens]


@pytest.mark.parametrize("placement", [dkv.DKV_PLACE_PREFIX_HOST, dkv.DKV_PLACE_RANDOM])
@pytest.mark.parametrize("shuffle", [False, True])
def test_ids_are_a_bijection_onto_both_pools(placement, shuffle):
    lens = [0, 1, 15, 16, 17, 1000, 333]
    S = 16
    table, res = plan(lens, S, placement, 0.6, shuffle, seed=11)
    nb = nblocks(lens, S)
    used = np.concatenate([table[b, :n] for b, n in enumerate(nb)])
    assert sorted(used.tolist()) == list(range(sum(nb)))
    assert res.host_split + res.num_dev_blocks == sum(nb)
    for b, n in enumerate(nb):
        assert (table[b, n:] == -1).all()
        nh = int((table[b, :n] < res.host_split).sum())
        assert nh == int(np.floor(0.6 * n + 0.5)), (b, n, nh)
    if placement == dkv.DKV_PLACE_PREFIX_HOST:
        for b, n in enumerate(nb):
            host = table[b, :n] < res.host_split
            assert not (~host[:-1] & host[1:]).any(), "a host block follows a device block"


def test_token_counts():
    lens = [100, 37, 64]
    table, res = plan(lens, 32, dkv.DKV_PLACE_RANDOM, 0.5, seed=3)
    host_tok = dev_tok = 0
    for b, L in enumerate(lens):
        for j in range(-(-L // 32)):
            n = min(32, L - 32 * j)
            if table[b, j] < res.host_split:
                host_tok += n
            else:
                dev_tok += n
    assert (res.host_tokens, res.dev_tokens) == (host_tok, dev_tok)
    assert host_tok + dev_tok == sum(lens)


def test_long_context_placement_numbers():
    """1,048,576 tokens in 64-token blocks, 90% host: the oldest 14746 blocks host, newest 1638 HBM."""
    table, res = plan([1 << 20], 64, dkv.DKV_PLACE_PREFIX_HOST, 0.9)
    assert (res.host_split, res.num_dev_blocks) == (14746, 1638)
    assert (table[0, :14746] < res.host_split).all() and (table[0, 14746:] >= res.host_split).all()


def test_tiny_placement_tokens_0_255_on_host():
    table, res = plan([512], 16, dkv.DKV_PLACE_PREFIX_HOST, 0.5)
    assert res.host_tokens == 256 and res.dev_tokens == 256
    assert (table[0, :16] < res.host_split).all() and (table[0, 16:] >= res.host_split).all()


def test_extreme_fractions_and_determinism():
    lens = [500, 800]
    t0, r0 = plan(lens, 16, dkv.DKV_PLACE_RANDOM, 0.0, seed=5)
    assert r0.host_split == 0
    t1, r1 = plan(lens, 16, dkv.DKV_PLACE_RANDOM, 1.0, seed=5)
    assert r1.num_dev_blocks == 0
    a, _ = plan(lens, 16, dkv.DKV_PLACE_RANDOM, 0.5, True, seed=9)
    b, _ = plan(lens, 16, dkv.DKV_PLACE_RANDOM, 0.5, True, seed=9)
    c, _ = plan(lens, 16, dkv.DKV_PLACE_RANDOM, 0.5, True, seed=10)
    assert np.array_equal(a, b) and not np.array_equal(a, c)


def test_random_placement_is_roughly_uniform():
    n = 4096
    counts = np.zeros(n)
    for seed in range(40):
        table, res = plan([16 * n], 16, dkv.DKV_PLACE_RANDOM, 0.25, seed=seed)
        counts += table[0] < res.host_split
    # each block is on the host with probability 1/4: 40 draws -> mean 10, sd ~2.7
    assert abs(counts.mean() - 10) < 1e-9
    assert counts.std() < 4.0 and counts.min() >= 0 and (counts > 0).mean() > 0.95


def test_plan_rejects_bad_arguments():
    table = np.zeros((1, 2), dtype=np.int32)
    with pytest.raises(dkv.DkvError):
        dkv.dkv_plan_blocks(dkv.DkvPlanParams(16, 0, 1.5, 0, 0), np.array([10], np.int32), table)
    with pytest.raises(dkv.DkvError):
        dkv.dkv_plan_blocks(dkv.DkvPlanParams(16, 0, 0.5, 0, 0), np.array([100], np.int32), table)
    with pytest.raises(dkv.DkvError):
        dkv.dkv_plan_blocks(dkv.DkvPlanParams(16, 5, 0.5, 0, 0), np.array([10], np.int32), table)
    with pytest.raises(dkv.DkvError):
        dkv.dkv_plan_blocks(dkv.DkvPlanParams(16, 0, 0.5, 0, 0), np.array([-1], np.int32), table)


@pytest.mark.parametrize("S,f,shuffle", [(16, 0.5, False), (32, 0.75, True), (64, 0.0, True), (16, 1.0, False)])
def test_pack_places_every_token_where_the_table_says(S, f, shuffle):
    w = kvgen.OPT_6_7B.replace(batch=3, num_q_heads=4, num_kv_heads=2, ctx=(1, 150))
    lens = kvgen.gen_seq_lens(w)
    k, v = kvgen.gen_kv(w, lens)
    table, res = plan(lens, S, dkv.DKV_PLACE_RANDOM, f, shuffle, seed=2)
    Hkv, D = w.num_kv_heads, w.head_dim
    blk = Hkv * S * D
    kh = np.full(max(1, res.host_split * blk), 0xFFFF, np.uint16)
    vh = kh.copy()
    kd = np.full(max(1, res.num_dev_blocks * blk), 0xFFFF, np.uint16)
    vd = kd.copy()
    dkv.dkv_pack_kv(k, v, lens, Hkv, D, S, table, res.host_split, res.num_dev_blocks, kh, vh, kd, vd)
    for b, L in enumerate(lens):
        for j in range(-(-int(L) // S)):
            pid = int(table[b, j])
            kp, vp, idx = (kh, vh, pid) if pid < res.host_split else (kd, vd, pid - res.host_split)
            tile_k = kp[idx * blk:(idx + 1) * blk].reshape(Hkv, S, D)
            tile_v = vp[idx * blk:(idx + 1) * blk].reshape(Hkv, S, D)
            n = min(S, int(L) - j * S)
            assert np.array_equal(tile_k[:, :n], k[b, :, j * S:j * S + n])
            assert np.array_equal(tile_v[:, :n], v[b, :, j * S:j * S + n])
            assert not tile_k[:, n:].any() and not tile_v[:, n:].any()


# ----------------------------------------------------------------------------- offload-ratio planner

def test_offload_time_optimal_fraction_balances_the_two_sides():
    plan = dkv.dkv_plan_offload(1 << 30, 51.5, 6547.8)
    f = 51.5 / (51.5 + 6547.8)
    assert abs(plan.time_optimal_fraction - f) < 1e-15 and abs(plan.host_fraction - f) < 1e-15
    t_host = f * (1 << 30) / 51.5e9
    t_dev = (1 - f) * (1 << 30) / 6547.8e9
    assert abs(t_host - t_dev) < 1e-15 and abs(plan.step_seconds - t_host) < 1e-15
    assert abs(plan.hbm_bytes_freed - f * (1 << 30)) < 1e-3


def test_offload_budget_forces_more_onto_the_host():
    X = 4 * (1 << 30)
    plan = dkv.dkv_plan_offload(X, 51.5, 6547.8, hbm_budget_bytes=0.1 * X)   # long-context case: 10% fits
    assert abs(plan.host_fraction - 0.9) < 1e-12
    assert abs(plan.hbm_bytes_freed - 0.9 * X) < 1e-3
    assert abs(plan.step_seconds - 0.9 * X / 51.5e9) < 1e-12
    # a budget larger than the cache leaves the time-optimal split; a zero budget puts everything on the host
    assert abs(dkv.dkv_plan_offload(X, 51.5, 6547.8, 2 * X).host_fraction - plan.time_optimal_fraction) < 1e-15
    assert dkv.dkv_plan_offload(X, 51.5, 6547.8, 0.0).host_fraction == 1.0


def test_offload_step_time_is_minimal_at_the_plan():
    X, hb, db = 1e9, 50.0, 7000.0
    plan = dkv.dkv_plan_offload(X, hb, db)
    for f in np.linspace(0, 1, 101):
        t = max(f * X / (hb * 1e9), (1 - f) * X / (db * 1e9))
        assert t >= plan.step_seconds - 1e-15


def test_offload_all_hbm_when_the_kernel_alone_beats_the_concurrent_split():
    """At f = 0 the HBM kernel has the GPU to itself; when its alone rate is at least the two sides' concurrent
    rates together, keeping the whole cache in HBM is the fastest placement the budget allows."""
    X, hb, beside, alone = 4 * (1 << 30), 51.3, 4570.0, 5580.0
    plan = dkv.dkv_plan_offload(X, hb, beside, hbm_alone_gbs=alone)
    assert plan.host_fraction == 0.0 and plan.time_optimal_fraction == 0.0 and plan.hbm_bytes_freed == 0.0
    assert abs(plan.step_seconds - X / (alone * 1e9)) < 1e-15
    # an unlimited budget (< 0) and a budget of the whole cache both allow it
    assert dkv.dkv_plan_offload(X, hb, beside, float(X), alone).host_fraction == 0.0
    # a budget below the cache forces a concurrent split, planned from the side-by-side rates alone
    capped = dkv.dkv_plan_offload(X, hb, beside, 0.5 * X, alone)
    assert abs(capped.host_fraction - 0.5) < 1e-12 and capped.time_optimal_fraction == 0.0
    assert abs(capped.step_seconds - 0.5 * X / (hb * 1e9)) < 1e-12
    small = dkv.dkv_plan_offload(X, hb, beside, 0.999 * X, alone)   # the bound is below f*: the concurrent optimum
    assert abs(small.host_fraction - hb / (hb + beside)) < 1e-15


def test_offload_keeps_the_concurrent_split_when_it_is_faster():
    X, hb, beside = 1 << 30, 51.5, 6547.8
    f = hb / (hb + beside)
    for alone in (-1.0, 0.0, 6000.0, hb + beside - 1e-6):   # unknown, or slower than both sides together
        plan = dkv.dkv_plan_offload(X, hb, beside, hbm_alone_gbs=alone)
        assert abs(plan.host_fraction - f) < 1e-15 and abs(plan.time_optimal_fraction - f) < 1e-15
        assert abs(plan.step_seconds - X / ((hb + beside) * 1e9)) < 1e-15
    tie = dkv.dkv_plan_offload(X, hb, beside, hbm_alone_gbs=hb + beside)   # equal times: no host traffic
    assert tie.host_fraction == 0.0


@pytest.mark.parametrize("alone", [3000.0, 6000.0, 7000.0, 9000.0])
@pytest.mark.parametrize("budget_frac", [-1.0, 1.0, 0.7, 0.2])
def test_offload_plan_is_minimal_over_the_placements_the_budget_allows(alone, budget_frac):
    """Brute force over f on a fine grid, with T(0) = X / alone and T(f > 0) = max(f X / hb, (1 - f) X / hbm)."""
    X, hb, beside = 1e9, 50.0, 6500.0
    budget = budget_frac * X if budget_frac >= 0 else -1.0
    plan = dkv.dkv_plan_offload(X, hb, beside, budget, alone)
    f_min = 0.0 if budget < 0 else max(0.0, 1.0 - budget / X)
    best = None
    for f in np.concatenate([[0.0], np.linspace(1e-6, 1.0, 200001)]):
        if f < f_min - 1e-12:
            continue
        t = X / (alone * 1e9) if f == 0.0 else max(f * X / (hb * 1e9), (1 - f) * X / (beside * 1e9))
        best = t if best is None else min(best, t)
    assert plan.step_seconds <= best * (1 + 1e-9)
    assert plan.host_fraction >= f_min - 1e-12
    t_plan = X / (alone * 1e9) if plan.host_fraction == 0.0 else max(
        plan.host_fraction * X / (hb * 1e9), (1 - plan.host_fraction) * X / (beside * 1e9))
    assert abs(t_plan - plan.step_seconds) < 1e-15


@pytest.mark.parametrize("args", [(0, 50, 7000, -1), (1e9, 0, 7000, -1), (1e9, 50, -1, -1), (float("inf"), 50, 7000, -1),
                                  (1e9, 50, 7000, float("nan")), (1e9, 50, 7000, -1, float("nan")),
                                  (1e9, 50, 7000, -1, float("inf"))])
def test_offload_rejects_bad_inputs(args):
    with pytest.raises(dkv.DkvError):
        dkv.dkv_plan_offload(*args)
