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


def test_percentile_and_flags():
    sys.path.insert(0, ROOT)
    import bench
    xs = [5.0, 1.0, 4.0, 2.0, 3.0]
    assert bench.pct(xs, 0) == 1.0 and bench.pct(xs, 50) == 3.0 and bench.pct(xs, 100) == 5.0
    assert bench.pct([7.0], 90) == 7.0
    a = bench.parse_args(["--latency-form", "--route-dim", "32", "--budget", "4"])
    assert a.latency_form and a.route_dim == 32 and a.budget == 4
    assert not bench.parse_args([]).latency_form and bench.parse_args([]).route_dim == 0
