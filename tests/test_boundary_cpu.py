"""The C-ABI library on the CPU: it loads, exports what include/dkv.h declares, its structs
match the header's layout, and host-side argument checks answer without a GPU."""
import ctypes
import os
import re
import subprocess
from pathlib import Path

import pytest

import decode_attention_host_b200 as dkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dkv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:DKV_API\s+)?(?:int|const char\*)\s+(dkv_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(dkv.EXPORTED)


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", str(dkv.LIB_PATH)], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, missing
    # nothing else with the dkv_ prefix leaks out
    assert {s for s in exported if s.startswith("dkv_")} == set(declared_functions())


def test_struct_layout_matches_header(tmp_path):
    src = tmp_path / "layout.c"
    fields = {"dkv_config": [f for f, _ in dkv.DkvConfig._fields_],
              "dkv_plan_params": [f for f, _ in dkv.DkvPlanParams._fields_],
              "dkv_plan_result": [f for f, _ in dkv.DkvPlanResult._fields_],
              "dkv_offload_plan": [f for f, _ in dkv.DkvOffloadPlan._fields_]}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "dkv.h"', "int main(void) {"]
    for st, fs in fields.items():
        lines.append(f'printf("{st} size %zu\\n", sizeof({st}));')
        for f in fs:
            lines.append(f'printf("{st} {f} %zu\\n", offsetof({st}, {f}));')
    lines.append("return 0; }")
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", f"-I{ROOT}/include", "-o", str(exe), str(src)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines():
        *key, val = line.split()
        got[tuple(key)] = int(val)
    for st, cls in (("dkv_config", dkv.DkvConfig), ("dkv_plan_params", dkv.DkvPlanParams),
                    ("dkv_plan_result", dkv.DkvPlanResult), ("dkv_offload_plan", dkv.DkvOffloadPlan)):
        assert got[(st, "size")] == ctypes.sizeof(cls)
        for f, _ in cls._fields_:
            assert got[(st, f)] == getattr(cls, f).offset, (st, f)


def _cfg(**kw):
    base = dict(num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16, kv_dtype=dkv.DKV_KV_BF16,
                rope_base=5e5, scale=0.0, max_batch=8, max_blocks_per_seq=2048, device=0, host_ctas=0)
    base.update(kw)
    return dkv.DkvConfig(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(num_q_heads=30), dkv.DKV_ERR_INVALID_ARG),
    (dict(num_kv_heads=0), dkv.DKV_ERR_INVALID_ARG),
    (dict(block_size=24), dkv.DKV_ERR_INVALID_ARG),
    (dict(block_size=0), dkv.DKV_ERR_INVALID_ARG),
    (dict(kv_dtype=7), dkv.DKV_ERR_INVALID_ARG),
    (dict(rope_base=-1.0), dkv.DKV_ERR_INVALID_ARG),
    (dict(rope_base=float("nan")), dkv.DKV_ERR_INVALID_ARG),
    (dict(scale=-0.1), dkv.DKV_ERR_INVALID_ARG),
    (dict(max_batch=0), dkv.DKV_ERR_INVALID_ARG),
    (dict(max_blocks_per_seq=1 << 27, block_size=16), dkv.DKV_ERR_INVALID_ARG),
    (dict(host_ctas=-3), dkv.DKV_ERR_INVALID_ARG),
    (dict(head_dim=96), dkv.DKV_ERR_UNSUPPORTED),
    (dict(num_q_heads=64, num_kv_heads=8), dkv.DKV_ERR_UNSUPPORTED),
])
def test_create_rejects_bad_config_before_any_cuda_call(kw, code):
    h = ctypes.c_void_p()
    rc = dkv.lib.dkv_create(ctypes.byref(_cfg(**kw)), ctypes.byref(h))
    assert rc == code and h.value is None
    assert dkv.dkv_last_error_string()


def test_null_arguments_are_rejected():
    assert dkv.lib.dkv_create(None, None) == dkv.DKV_ERR_INVALID_ARG
    assert dkv.lib.dkv_attn_decode(None, None, None, None, None, None, None, None, 0, None, None, 1, 1, 0) \
        == dkv.DKV_ERR_INVALID_ARG
    assert dkv.lib.dkv_get_status(None, None) == dkv.DKV_ERR_INVALID_ARG
    assert dkv.lib.dkv_query_plan(None, 1, 1, None, None) == dkv.DKV_ERR_INVALID_ARG
    assert dkv.lib.dkv_last_launch_count(None, None) == dkv.DKV_ERR_INVALID_ARG
    assert dkv.lib.dkv_host_pool_alloc(0, None) == dkv.DKV_ERR_INVALID_ARG
    assert dkv.lib.dkv_destroy(None) == dkv.DKV_OK
    assert dkv.lib.dkv_host_pool_free(None) == dkv.DKV_OK


def test_a_c_program_links_and_calls_the_host_entry_points(tmp_path):
    """A plain C11 program built against include/dkv.h and linked to libdkv.so: the host-only entry points
    answer through their declared prototypes (no GPU needed)."""
    src = tmp_path / "consumer.c"
    src.write_text(r"""
#include <math.h>
#include <stdio.h>
#include "dkv.h"
int main(void) {
  dkv_offload_plan plan;
  /* 4 GiB, 51 GB/s host, 4500 GB/s beside the host stream, unlimited budget, 5600 GB/s alone */
  if (dkv_plan_offload(4294967296.0, 51.0, 4500.0, -1.0, 5600.0, &plan) != DKV_OK) return 1;
  if (plan.host_fraction != 0.0) return 2;
  if (fabs(plan.step_seconds - 4294967296.0 / 5600e9) > 1e-15) return 3;
  if (dkv_plan_offload(4294967296.0, 51.0, 4500.0, 0.5 * 4294967296.0, 5600.0, &plan) != DKV_OK) return 4;
  if (fabs(plan.host_fraction - 0.5) > 1e-12) return 5;
  if (dkv_plan_offload(0.0, 51.0, 4500.0, -1.0, -1.0, &plan) != DKV_ERR_INVALID_ARG) return 6;
  if (dkv_last_error_string()[0] == '\0') return 7;
  if (dkv_create(NULL, NULL) != DKV_ERR_INVALID_ARG) return 8;
  printf("ok\n");
  return 0;
}
""")
    exe = tmp_path / "consumer"
    lib = Path(dkv.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", f"-I{ROOT}/include", "-o", str(exe), str(src), str(lib),
                    f"-Wl,-rpath,{lib.parent}", "-lm"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
