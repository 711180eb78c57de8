"""Failure detection on the host side (needs a B200): allocation failures injected by a test hook
or requested from the driver, never a GPU fault.

dkv_create makes 7 device allocations.  The hook dkv_debug_fail_alloc makes one of them fail as an
out-of-memory would; every such create must return DKV_ERR_NO_MEMORY with no handle, give back what
it had allocated, and leave the device usable for the next create.  A pinned host pool larger than
any machine's memory must fail with DKV_ERR_NO_MEMORY too.
"""
import ctypes

import numpy as np
import pytest
import torch

import decode_attention_host_b200 as dkv
import kvgen
from tests import gpu_cases as gc

pytestmark = pytest.mark.gpu

N_ALLOCS = 7


def _cfg():
    return dkv.DkvConfig(32, 8, 128, 16, dkv.DKV_KV_BF16, 5e5, 0.0, 8, 2048, 0, 0)


def test_create_reports_each_failed_allocation_and_frees_the_rest():
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for n in range(1, N_ALLOCS + 1):
        dkv.dkv_debug_fail_alloc(n)
        h = ctypes.c_void_p()
        rc = dkv.lib.dkv_create(ctypes.byref(_cfg()), ctypes.byref(h))
        assert rc == dkv.DKV_ERR_NO_MEMORY, (n, rc)
        assert h.value is None
        assert "allocation" in dkv.dkv_last_error_string()
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    assert abs(free1 - free0) <= (4 << 20), f"failed creates kept {(free0 - free1) / 2**20:.1f} MiB"
    # a hook past the last allocation does not fire, and is cleared by that create
    dkv.dkv_debug_fail_alloc(N_ALLOCS + 1)
    h = dkv.dkv_create(_cfg())
    dkv.dkv_destroy(h)
    h = dkv.dkv_create(_cfg())
    dkv.dkv_destroy(h)


def test_device_stays_usable_after_failed_creates():
    dkv.dkv_debug_fail_alloc(1)
    with pytest.raises(dkv.DkvError) as e:
        dkv.dkv_create(_cfg())
    assert e.value.code == dkv.DKV_ERR_NO_MEMORY
    w = kvgen.LLAMA3_8B.replace(name="after_oom", batch=2, ctx=900, seed=71)
    q = kvgen.gen_q(w)
    lens = kvgen.gen_seq_lens(w)
    k, v = kvgen.gen_kv(w, lens)
    kv = dkv.PagedKV(k, v, lens, w.block_size, dkv.DKV_PLACE_RANDOM, 0.5, False, 3)
    attn = dkv.DecodeAttention(w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, dkv.DKV_KV_BF16,
                               w.rope_base, w.batch, kv.stride)
    q_dev = torch.from_numpy(q).cuda()
    out = torch.empty_like(q_dev)
    attn(q_dev, kv, out)
    torch.cuda.synchronize()
    import oracle
    err = gc.max_err(out.cpu().numpy(), oracle.decode(q, k, v, lens, oracle.KV_BF16, w.rope_base))
    assert attn.status() == 0 and err <= gc.TOL
    attn.close()
    kv.free()


def test_pinned_pool_beyond_memory_is_reported():
    with pytest.raises(dkv.DkvError) as e:
        dkv.dkv_host_pool_alloc(1 << 50)   # 1 PiB of page-locked host memory
    assert e.value.code == dkv.DKV_ERR_NO_MEMORY
    p = dkv.dkv_host_pool_alloc(1 << 20)   # an ordinary pool still works
    dkv.dkv_host_pool_free(p)


def test_hook_rejects_negative_counts():
    with pytest.raises(dkv.DkvError) as e:
        dkv.dkv_debug_fail_alloc(-1)
    assert e.value.code == dkv.DKV_ERR_INVALID_ARG
    dkv.dkv_debug_fail_alloc(0)


def test_a_copy_that_never_completes_times_out_and_is_reported():
    """The HBM kernel's waits on its tile copies are bounded: a copy that never lands (the test hook arms a
    barrier and issues nothing) ends that warp's wait after about 2 s with DKV_STATUS_COPY_TIMEOUT and NaN
    rows for the units it held; the other rows are exact and the next call is clean."""
    import time
    import oracle
    # blocks in both pools: the HBM kernel runs beside the host kernel and moves its tiles by tensor copies
    w = kvgen.LLAMA3_8B.replace(name="stall", batch=2, ctx=3000, seed=72, host_fraction=0.5)
    case = gc.Case(w)
    want = case.oracle()
    dkv.dkv_debug_stall_copy(True)
    t0 = time.monotonic()
    got = case.run()
    elapsed = time.monotonic() - t0
    assert case.attn.status() == dkv.DKV_STATUS_COPY_TIMEOUT
    assert elapsed < 30
    bad = np.isnan(got).any(axis=2)
    assert bad.any() and not bad.all()
    assert np.abs(got[~bad] - want[~bad]).max() <= gc.TOL
    again = case.run()   # hook cleared: a clean call on the same handle and device
    assert case.attn.status() == 0 and gc.max_err(again, want) <= gc.TOL
    case.free()
