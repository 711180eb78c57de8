"""Per-kernel attribution on the GPU: the events the library records around each kernel, the per-call timeline
(which shows the host-stream and HBM kernels overlapping) and the launch counts."""
import pytest

import decode_attention_host_b200 as dkv
import kvgen
from tests import gpu_cases as gc

pytestmark = pytest.mark.gpu


def test_timeline_shows_the_host_and_hbm_kernels_overlapping():
    w = kvgen.LLAMA3_8B.replace(name="timeline", batch=2, ctx=60000, seed=81)
    case = gc.Case(w)
    case.run()
    calls = 3
    dkv.dkv_profile_begin(case.attn.handle, calls)
    for _ in range(calls):
        case.run()
    t = dkv.dkv_profile_timeline(case.attn.handle, calls - 1)
    ms, counts = dkv.dkv_profile_end(case.attn.handle)
    assert counts == [calls, calls, calls]
    assert all(m > 0 for m in ms)
    host0, host1, hbm0, hbm1, merge0, merge1 = t
    assert min(host0, hbm0) == 0.0 and host1 > host0 and hbm1 > hbm0
    # the HBM kernel runs inside the host-stream kernel's interval, and the merge follows both
    assert hbm0 < host1 and hbm1 <= host1
    assert merge0 >= max(host1, hbm1) - 1e-3 and merge1 > merge0
    assert case.attn.launches() == 4 and case.attn.status() == 0
    case.free()


def test_timeline_of_a_single_pool_call_and_bad_arguments():
    w = kvgen.LLAMA3_8B.replace(name="timeline_hbm", batch=2, ctx=4000, seed=82, host_fraction=0.0)
    case = gc.Case(w)
    dkv.dkv_profile_begin(case.attn.handle, 1)
    case.run()
    host0, host1, hbm0, hbm1, merge0, merge1 = dkv.dkv_profile_timeline(case.attn.handle, 0)
    assert host0 == host1 == -1.0 and hbm0 == 0.0 and hbm1 > 0 and merge0 >= hbm1 - 1e-3
    with pytest.raises(dkv.DkvError) as e:
        dkv.dkv_profile_timeline(case.attn.handle, 5)   # no such recorded call
    assert e.value.code == dkv.DKV_ERR_INVALID_ARG
    ms, counts = dkv.dkv_profile_end(case.attn.handle)
    assert counts == [0, 1, 1] and case.attn.launches() == 2
    case.free()
