"""Host-side pieces of bench.py that need no GPU: the multi-rank timing
aggregation over a world-size-2 gloo group, and the JSON contract of the
reference arm (the fp64 oracle) on a small sample."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as tmp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    elapsed = 10.0 + 5.0 * rank                 # the slowest rank decides
    worst = bench.max_over_ranks(elapsed)
    seed = bench.replica_seed(20263, rank)
    q.put((rank, worst, seed, bench.throughput(world, 20, worst)))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_replicas_with_gloo():
    world, port = 2, 29533
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    assert [o[1] for o in out] == [15.0, 15.0]
    assert out[0][2] != out[1][2]                                   # independent replicas
    assert out[0][3] == pytest.approx(2 * 20 / 15e-3)              # whole-job steps/s


def test_reference_arm_json_contract():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "c2",
                        "--n", "2048", "--layers", "2", "--steps", "1", "--warmup", "1"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("{")][-1]
    j = json.loads(line)
    assert j["impl"] == "reference" and j["unit"] == "steps/s" and j["value"] > 0
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["cores"] >= 1
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["d2h_bytes_per_step"] == 0
    for k in ("metric", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling", "config"):
        assert k in j
    # steps x ms_per_step is the sampled work that ran; the full-step figure is labelled
    ex = j["extrapolation"]
    assert j["steps"] == 1 and ex["units_per_timed_step"] == j["cpu_baseline"]["cores"]
    assert ex["full_step_ms"] == pytest.approx(j["ms_per_step"] * ex["units_per_full_step"] / ex["units_per_timed_step"])
    assert j["value"] == pytest.approx(1e3 / ex["full_step_ms"])
    assert j["cpu_baseline"]["cpu_model"]


def test_percentile_and_flags():
    sys.path.insert(0, ROOT)
    import bench
    xs = [5.0, 1.0, 4.0, 2.0, 3.0]
    assert bench.pct(xs, 0) == 1.0 and bench.pct(xs, 50) == 3.0 and bench.pct(xs, 100) == 5.0
    assert bench.pct([7.0], 90) == 7.0
    a = bench.parse_args(["--latency-form", "--route-dim", "32", "--budget", "4"])
    assert a.latency_form and a.route_dim == 32 and a.budget == 4
    assert not bench.parse_args([]).latency_form and bench.parse_args([]).route_dim == 0


def test_eq17_memory_model_arithmetic():
    """Eq. (17) from realised counts on a fake cache: hand-computed byte counts"""
    from types import SimpleNamespace
    sys.path.insert(0, ROOT)
    import bench
    B, L, Hq, Hkv, n, d, a_cap, m_cap = 1, 2, 4, 2, 1000, 8, 64, 64
    z = lambda *sh, dt=torch.bfloat16: torch.zeros(*sh, dtype=dt)
    c = SimpleNamespace(B=B, L=L, Hq=Hq, Hkv=Hkv, n=n, d=d, a_cap=a_cap, m_cap=m_cap, dr=0, dtype_name="bf16",
                        a_count=torch.tensor([40], dtype=torch.int32), m_count=torch.tensor([30], dtype=torch.int32),
                        Ka=z(B, L, Hkv, a_cap, d), Va=z(B, L, Hkv, a_cap, d), kbar=z(B, L, Hkv, m_cap, d),
                        vbar=z(B, L, Hkv, m_cap, d), inv_norm=z(B, L, Hkv, m_cap, dt=torch.float32),
                        logS=z(B, m_cap, dt=torch.float32), anchor_pos=z(B, a_cap, dt=torch.int32),
                        span_beg=z(B, m_cap, dt=torch.int32), span_end=z(B, m_cap, dt=torch.int32),
                        blk_off=z(B, m_cap + 1, dt=torch.int64), kbar_r=None, home=z(B, L, 512))
    r = bench.memory_model(c, cold=True)
    assert r["anchors_bytes"] == 2 * 2 * 2 * 8 * 40 * 2
    assert r["eq17_bytes"] == 2 * 2 * 2 * 8 * 40 * 2 + 2 * 2 * 2 * 8 * 30 * 2 + 2 * 2 * 30 * 4 + 30 * 4
    assert r["full_kv_bytes"] == 2 * 2 * 2 * 1000 * 8 * 2
    assert r["allocated_bytes"] == (2 * 2 * 2 * 64 * 8 * 2 + 2 * 2 * 2 * 64 * 8 * 2 + 2 * 2 * 64 * 4 + 64 * 4
                                    + 64 * 4 * 3 + 65 * 8)
    c.dr, c.kbar_r = 32, z(B, L, Hq, m_cap, 32)
    r2 = bench.memory_model(c, cold=False)
    assert r2["eq17_bytes"] - r["eq17_bytes"] == 2 * 4 * 32 * 30 * 2
    assert r2["allocated_bytes"] - r["allocated_bytes"] == 2 * 4 * 64 * 32 * 2 + 2 * 512 * 2
