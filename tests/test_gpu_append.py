"""The write side of the cache: K/V projection of the new token and its store (needs a B200).

The kernel accumulates in fp32 and rounds to the 16-bit storage type, so each
stored value must be the nearest-even rounding of the exact product.  The one
exception is a product within the fp32 accumulation error of a rounding
midpoint, where either neighbour is correct.
"""
import numpy as np
import pytest
import torch

import decode_attention_host_b200 as dkv
import kvgen
import oracle
from tests import gpu_cases as gc

pytestmark = pytest.mark.gpu


def w_batch(kw) -> int:
    return kw["batch"]


def _exact_round(y: np.ndarray, kv_dtype: str) -> np.ndarray:
    """fp64 -> value of the nearest 16-bit number (ties to even), computed exactly."""
    bits = 8 if kv_dtype == kvgen.BF16 else 11
    m, e = np.frexp(y)
    return np.rint(m * 2.0 ** bits) * 2.0 ** (e.astype(np.float64) - bits)


def _check_rounding(got_bits, y, bound, kv_dtype):
    got = kvgen.bits_to_f32(got_bits, kv_dtype).astype(np.float64)
    want = _exact_round(y, kv_dtype)
    diff = got != want
    if diff.any():
        # accepted only next to a rounding midpoint, within the fp32 accumulation error
        mid = 0.5 * (got[diff] + want[diff])
        assert np.all(np.abs(y[diff] - mid) <= bound[diff]), "rounding differs away from a midpoint"
        ulp = np.abs(want[diff]) * 2.0 ** (-7 if kv_dtype == kvgen.BF16 else -10)
        assert np.all(np.abs(got[diff] - want[diff]) <= ulp * 1.01), "more than one step apart"
    return int(diff.sum())


def _setup(w: kvgen.Workload, hidden: int, seed: int):
    """A cache whose table already covers position L_b of every sequence (lengths L_b + 1)."""
    rng = np.random.default_rng(seed)
    lens = kvgen.gen_seq_lens(w)
    case = gc.Case(w, lens=lens + 1)
    R = w.num_kv_heads * w.head_dim
    x = rng.standard_normal((w.batch, hidden)).astype(np.float32)
    wk = kvgen.to_bits(rng.standard_normal((R, hidden)).astype(np.float32) / np.sqrt(hidden), w.kv_dtype)
    wv = kvgen.to_bits(rng.standard_normal((R, hidden)).astype(np.float32) / np.sqrt(hidden), w.kv_dtype)
    return case, lens, x, wk, wv


def _append(case, lens, x, wk, wv):
    case.kv.seq_lens_dev.copy_(torch.from_numpy(lens))
    xd = torch.from_numpy(x).cuda()
    wkd = torch.from_numpy(wk.view(np.int16)).cuda()
    wvd = torch.from_numpy(wv.view(np.int16)).cuda()
    case.attn.append(xd, wkd, wvd, case.kv)
    torch.cuda.synchronize()


def _stored(case, w, b, pos, which):
    """Stored bits of token `pos` of sequence b, all kv heads: uint16 [Hkv, D]."""
    kv = case.kv
    S, Hkv, D = w.block_size, w.num_kv_heads, w.head_dim
    pid = int(kv.table[b, pos // S])
    blk = Hkv * S * D
    if pid < kv.host_split:
        pool = (kv.k_host if which == "k" else kv.v_host).array
        tile = pool[pid * blk:(pid + 1) * blk]
    else:
        pool = kv.k_dev if which == "k" else kv.v_dev
        tile = pool[(pid - kv.host_split) * blk:(pid - kv.host_split + 1) * blk].cpu().numpy().view(np.uint16)
    return tile.reshape(Hkv, S, D)[:, pos % S, :].copy()


@pytest.mark.parametrize("name,kw,hidden", [
    ("llama3_8b", dict(batch=5, ctx=(40, 700), block_size=16), 512),
    ("opt_6_7b", dict(batch=3, ctx=(1, 300)), 256),
    # 16 sequences per pass over the weights: one full pass, then a pass of 4 more; a hidden size that is
    # not a multiple of the 256 columns a CTA covers per step
    ("llama3_8b", dict(batch=20, ctx=(10, 200), block_size=16), 4104),
    ("tiny_gqa", dict(batch=12, ctx=(1, 100)), 264),
])
def test_projection_is_stored_rounded_at_its_position(name, kw, hidden):
    w = kvgen.get(name).replace(name=f"append_{name}_{w_batch(kw)}", **kw)
    case, lens, x, wk, wv = _setup(w, hidden, 50)
    before_k = [_stored(case, w, b, int(lens[b]) - 1, "k") for b in range(w.batch) if lens[b] > 0]
    _append(case, lens, x, wk, wv)
    assert case.attn.status() == 0
    odt = gc.oracle_dtype(w)
    yk = oracle.project(x, wk, odt)
    yv = oracle.project(x, wv, odt)
    gamma = hidden * 2.0 ** -24
    bk = gamma * oracle.project(np.abs(x), wk & 0x7FFF, odt)
    bv = gamma * oracle.project(np.abs(x), wv & 0x7FFF, odt)
    near_ties = 0
    Hkv, D = w.num_kv_heads, w.head_dim
    for b in range(w.batch):
        pos = int(lens[b])
        near_ties += _check_rounding(_stored(case, w, b, pos, "k").reshape(-1), yk[b], bk[b], w.kv_dtype)
        near_ties += _check_rounding(_stored(case, w, b, pos, "v").reshape(-1), yv[b], bv[b], w.kv_dtype)
    assert near_ties <= 0.01 * 2 * w.batch * Hkv * D
    # the previous token of every sequence is untouched
    after_k = [_stored(case, w, b, int(lens[b]) - 1, "k") for b in range(w.batch) if lens[b] > 0]
    assert all(np.array_equal(a, c) for a, c in zip(before_k, after_k))
    case.free()


def test_decode_after_append_attends_to_the_new_token():
    w = kvgen.LLAMA3_8B.replace(name="append_decode", batch=3, ctx=(100, 900), seed=51)
    hidden = 256
    case, lens, x, wk, wv = _setup(w, hidden, 52)
    _append(case, lens, x, wk, wv)
    new_lens = lens + 1
    case.kv.seq_lens_dev.copy_(torch.from_numpy(new_lens))
    got = case.run()
    assert case.attn.status() == 0
    # oracle: logical K/V with token L_b replaced by the oracle's own rounded projection
    odt = gc.oracle_dtype(w)
    k, v = case.k.copy(), case.v.copy()
    yk = _exact_round(oracle.project(x, wk, odt), w.kv_dtype).astype(np.float32)
    yv = _exact_round(oracle.project(x, wv, odt), w.kv_dtype).astype(np.float32)
    for b in range(w.batch):
        L = int(lens[b])
        k[b, :, L, :] = kvgen.to_bits(yk[b].reshape(w.num_kv_heads, w.head_dim), w.kv_dtype)
        v[b, :, L, :] = kvgen.to_bits(yv[b].reshape(w.num_kv_heads, w.head_dim), w.kv_dtype)
    want = oracle.decode(case.q, k, v, new_lens, odt, w.rope_base)
    assert gc.max_err(got, want) <= gc.TOL
    case.free()


def test_append_outside_the_table_sets_status_and_skips():
    w = kvgen.LLAMA3_8B.replace(name="append_bad", batch=2, ctx=200, seed=53)
    case, lens, x, wk, wv = _setup(w, 64, 54)
    bad = lens.copy()
    bad[1] = case.kv.stride * w.block_size   # one past the table
    snapshot = [_stored(case, w, 1, int(lens[1]), "k")]
    _append(case, bad, x, wk, wv)
    assert case.attn.status() & dkv.DKV_STATUS_BAD_SEQ_LEN
    assert np.array_equal(_stored(case, w, 1, int(lens[1]), "k"), snapshot[0])
    table = case.kv.table.copy()
    table[0, int(lens[0]) // w.block_size] = case.kv.host_split + case.kv.num_dev_blocks + 3
    case.kv.table_dev.copy_(torch.from_numpy(table))
    _append(case, lens, x, wk, wv)
    assert case.attn.status() & dkv.DKV_STATUS_BAD_BLOCK_ID
    with pytest.raises(dkv.DkvError):
        dkv.dkv_append_kv(case.attn.handle, torch.zeros(2, 60, device="cuda"), torch.zeros(1, device="cuda"),
                          torch.zeros(1, device="cuda"), 60, case.kv.table_dev, case.kv.seq_lens_dev, 0, None, None,
                          None, None, None, 2, case.kv.stride, 0)
    case.free()
