"""bench.py host logic on the CPU: max-over-ranks timing with world size 2 (gloo),
per-rank replica seeds, and the reference arm (the oracle) end to end."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r, w = bench.dist_init("gloo")
    got = bench.max_over_ranks(1.5 + 10 * rank)
    bench.barrier()
    seed = bench.workload_for_rank("llama3_8b", r).seed
    q.put((r, w, got, seed))
    dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[2] for r in res] == [11.5, 11.5]
    assert [r[1] for r in res] == [2, 2]
    assert res[0][3] != res[1][3], "replicas must draw different inputs"


def test_single_process_max_is_identity():
    assert bench.max_over_ranks(3.25) == 3.25


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny_gqa", "--steps", "2", "--warmup", "1"], capture_output=True, text=True,
                         timeout=300, cwd=ROOT, env=dict(os.environ, OMP_NUM_THREADS="2"))
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "GB/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] == 2
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["config"]["workload"] == "tiny_gqa"


def test_reduced_context_keeps_the_shape_and_renames_the_workload():
    w = bench.workload_for_rank("long_ctx", 0, 262144)
    base = bench.workload_for_rank("long_ctx", 0)
    assert w.name == "long_ctx_ctx262144" and w.ctx == 262144
    assert (w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.placement, w.host_fraction) == \
        (base.batch, base.num_q_heads, base.num_kv_heads, base.head_dim, base.block_size, base.placement,
         base.host_fraction)
    assert bench.workload_for_rank("long_ctx", 2, 4096).seed == base.seed + 2000


def test_default_workload_is_the_largest_single_gpu_config():
    args = bench.parse_args([])
    assert args.workload == "long_ctx" and args.mode == "zero_copy" and args.gpus == 1
    import kvgen
    sizes = {n: kvgen.get(n).batch * kvgen.get(n).max_ctx for n in ("tiny_gqa", "llama3_8b", "long_ctx", "opt_6_7b")}
    assert max(sizes, key=sizes.get) == "long_ctx"


def test_host_fraction_override_names_the_placement():
    import bench
    w = bench.workload_for_rank("opt_6_7b", 0, 0, 0.0)
    assert w.host_fraction == 0.0 and w.name == "opt_6_7b_h0"
    assert bench.workload_for_rank("opt_6_7b", 0).host_fraction == 0.75
    assert bench.workload_for_rank("long_ctx", 1, 4096, 0.5).name == "long_ctx_ctx4096_h0.5"
    with pytest.raises(SystemExit):
        bench.parse_args(["--host-fraction", "1.5"])


def _planner_model(alone_gbs, beside_far=2300.0, beside_near=4500.0, host_gbs=51.0):
    """A modelled GPU: the host stream at host_gbs; the HBM kernel at alone_gbs with no host blocks, beside the
    host stream slower, and slowest when the host stream dominates the step (f >= 0.5)."""
    def measure(x, f):
        hbm = alone_gbs if f == 0 else (beside_far if f >= 0.5 else beside_near)
        t = x / (hbm * 1e9) if f == 0 else max(f * x / (host_gbs * 1e9), (1 - f) * x / (hbm * 1e9))
        return {"ms": t * 1e3, "host": host_gbs if f > 0 else None, "hbm": hbm}
    return measure


def _plan(x, budget, f0, alone):
    import decode_attention_host_b200 as dkv
    model = _planner_model(alone)
    seen = []

    def measure_at(f):
        seen.append(f)
        return model(x, f)
    rates = lambda m: (m["host"] if m["host"] is not None else 51.0 * 0.92, m["hbm"])  # noqa: E731
    planner, meas = bench.plan_placement(dkv.dkv_plan_offload, measure_at, rates, x, budget, f0, model(x, f0))
    return planner, meas, seen


def test_planner_keeps_the_cache_in_hbm_when_the_kernel_alone_is_fastest():
    x = 4.0 * (1 << 30)
    planner, meas, seen = _plan(x, -1.0, 0.9, alone=5600.0)
    # the whole cache in HBM, two side-by-side splits (from the far and then the near rates), then back
    assert seen[0] == 0.0 and 0 < seen[1] < 0.05 and 0 < seen[2] < seen[1] and seen[-1] == 0.0
    assert planner["host_fraction"] == 0.0 and planner["time_optimal_fraction"] == 0.0
    assert planner["hbm_alone_gbs"] == 5600.0
    assert abs(planner["predicted_over_measured"] - 1.0) < 1e-9
    assert abs(meas["ms"] - x / 5600e9 * 1e3) < 1e-9


def test_planner_splits_when_the_side_by_side_rate_wins():
    x = 4.0 * (1 << 30)
    planner, meas, seen = _plan(x, -1.0, 0.9, alone=3000.0)   # alone slower than 51 + 4500 side by side
    f = planner["host_fraction"]
    assert seen[0] == 0.0 and 0 < f < 0.05 and seen[-1] == f
    assert abs(f - 51.0 / (51.0 + 4500.0)) < 1e-12           # settled on the near-point side-by-side rates
    assert planner["rounds"][-1]["host_fraction"] == f
    assert abs(planner["predicted_over_measured"] - 1.0) < 1e-9


def test_planner_with_a_budget_never_measures_the_all_hbm_placement():
    x = 4.0 * (1 << 30)
    planner, meas, seen = _plan(x, 0.5 * x, 0.9, alone=5600.0)
    assert seen == [0.5] and planner["hbm_alone_gbs"] is None
    assert abs(planner["host_fraction"] - 0.5) < 1e-12
    assert abs(planner["predicted_over_measured"] - 1.0) < 1e-9   # the model is exact at f >= 0.5


def test_planner_on_a_workload_already_in_hbm():
    """The workload's own placement is all-HBM: its measurement gives the alone rate; the side-by-side splits
    are measured, lose to it, and the cache is rebuilt in HBM."""
    x = 1.0 * (1 << 30)
    planner, meas, seen = _plan(x, -1.0, 0.0, alone=5600.0)
    assert planner["hbm_alone_gbs"] == 5600.0 and planner["host_fraction"] == 0.0
    assert len(seen) == 3 and all(0 < f < 0.05 for f in seen[:2]) and seen[-1] == 0.0
    assert abs(meas["ms"] - x / 5600e9 * 1e3) < 1e-9


def test_append_bytes_count_weights_states_and_stores():
    import kvgen
    w = kvgen.get("llama3_8b")             # Hkv*D = 1024 rows, 8 sequences
    hbm, host = bench.append_bytes(w, 4096, dev_stores=5, host_stores=3)
    assert hbm == 2 * 1024 * 4096 * 2 + 8 * 4096 * 4 + 5 * 2 * 1024 * 2
    assert host == 3 * 2 * 1024 * 2
    assert bench.parse_args(["--mode", "append"]).mode == "append"
