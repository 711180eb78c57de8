"""The allocation-free decode entry point against the fp64 oracle and the handle-based one (needs a B200).

dkv_attn_decode_noalloc is for callers that cannot allocate device memory or
keep a handle.  Examples: an engine that gives all GPU memory to its own
allocator at start-up, a latency-critical loop in which cudaMalloc may
synchronise the device, or a plain-C plugin that only sees raw pointers.  Its
scratch is one fixed array inside the library, shared by every call, so this
file runs calls back to back on different workloads.  Each call must give the
oracle's answer (and dkv_attn_decode's) even though the previous call left its
partials in the array.  The file is named to be collected last.
"""
import numpy as np
import pytest
import torch

import decode_attention_host_b200 as dkv
import kvgen
from tests import gpu_cases as gc

pytestmark = pytest.mark.gpu


def _noalloc(case: gc.Case) -> tuple[np.ndarray, int]:
    kv = case.kv
    out = torch.full_like(case.q_dev, float("nan"))
    status = torch.full((1,), -1, dtype=torch.int32, device=case.q_dev.device)
    dkv.dkv_attn_decode_noalloc(case.attn.cfg, case.q_dev, kv.k_host.ptr or None, kv.v_host.ptr or None,
                                kv.k_dev if kv.num_dev_blocks else None, kv.v_dev if kv.num_dev_blocks else None,
                                kv.table_dev, kv.seq_lens_dev, kv.host_split, out, status,
                                torch.cuda.current_stream().cuda_stream, kv.batch, kv.stride, kv.num_dev_blocks)
    torch.cuda.synchronize()
    return out.cpu().numpy(), int(status.item())


def test_noalloc_matches_oracle_and_handle_path_on_calls_in_a_row():
    cases = [gc.Case(kvgen.LLAMA3_8B.replace(name="noalloc_a", batch=3, ctx=2900, seed=21)),
             gc.Case(kvgen.OPT_6_7B.replace(name="noalloc_b", batch=5, ctx=(40, 1700), seed=22))]
    refs = [c.run() for c in cases]
    wants = [c.oracle() for c in cases]
    for c in cases:
        assert c.attn.status() == 0
    # two calls in a row on different workloads, then the first workload again
    for i in (0, 1, 0):
        got, status = _noalloc(cases[i])
        assert status == 0
        err = gc.max_err(got, wants[i])   # against the fp64 oracle (also checks every value is finite)
        gc.record("test_noalloc_matches_oracle_and_handle_path_on_calls_in_a_row", cases[i].w.name, err)
        assert err <= gc.TOL, f"call on workload {i}: max abs err {err:.3e} against the oracle"
        diff = float(np.abs(got - refs[i]).max())
        assert diff <= gc.TOL, f"call on workload {i}: max abs diff {diff:.3e} against dkv_attn_decode"
    for c in cases:
        c.free()


def test_noalloc_reports_device_status_per_call():
    case = gc.Case(kvgen.LLAMA3_8B.replace(name="noalloc_bad", batch=2, ctx=500, seed=23))
    table = case.kv.table.copy()
    table[0, 3] = case.kv.host_split + case.kv.num_dev_blocks + 1
    case.kv.table_dev.copy_(torch.from_numpy(table))
    got, status = _noalloc(case)
    assert status == dkv.DKV_STATUS_BAD_BLOCK_ID and np.isnan(got[0]).all() and np.isfinite(got[1]).all()
    case.kv.table_dev.copy_(torch.from_numpy(case.kv.table))
    got, status = _noalloc(case)   # the next call starts from a cleared status word
    assert status == 0 and np.isfinite(got).all()
    case.free()


def test_noalloc_rejects_a_batch_beyond_the_fixed_scratch():
    cfg = dkv.DkvConfig(32, 8, 128, 16, dkv.DKV_KV_BF16, 5e5, 0.0, 1, 64, 0, 0)
    # all blocks in HBM: one split of partials per (sequence, query head), 4 * (D + 1) bytes each
    batch = 2 + (16 << 20) // (32 * 129 * 4)
    fake = 1 << 20   # never dereferenced: the size check comes before any launch
    with pytest.raises(dkv.DkvError) as e:
        dkv.dkv_attn_decode_noalloc(cfg, fake, None, None, fake, fake, fake, fake, 0, fake, None, None, batch, 4, 8)
    assert e.value.code == dkv.DKV_ERR_INVALID_ARG and "scratch" in str(e.value)
