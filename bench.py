#!/usr/bin/env python
"""Benchmark of the SeKV span-cache hot path on B200.

Default workload (c3): Llama-3-8B-shaped decode at 128K context, batch 1, bf16
K/V, 32 layers x 32 query / 8 KV heads, head_dim 128, rank-16 bases held cold in
pinned host memory, thresholds calibrated for ~2% zoom. One step is one decode
token over all 32 layers: ROUTE (routing + zoom mask), fetch of the zoomed
spans' bases (cudaMemcpyAsync on a side stream), ATTEND (one shared softmax over
anchors, log|S|-corrected summaries and low-rank reconstructed tokens). The
prefill build (boundary scan, summaries, Jacobi bases) of the same cache is
timed too and reported under "prefill_build".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c3|c2|c4|c5]
    python bench.py --impl reference ...   # the fp64 CPU oracle as the reference arm

Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import multiprocessing as mp
import os
import statistics
import subprocess
import sys
import tempfile
import time
from datetime import timedelta

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SeKV decode attn µs/step & steps/s at 128K ctx; HBM GB/s vs B200 peak"
_BLAS_ENV = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")
FALLBACK_HBM_GBS = 6650.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="sekv", choices=["sekv", "reference"])
    ap.add_argument("--workload", default="c3", choices=["c2", "c3", "c4", "c5"])
    ap.add_argument("--n", type=int, default=0, help="override the context length (profiling runs)")
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cache", action="store_true",
                    help="cold workloads: keep fetched bases resident in a device cache across steps "
                         "(the configs fetch every step)")
    ap.add_argument("--route-dim", type=int, default=0, choices=[0, 32, 64],
                    help="learned-form routing with a seeded d'-dimensional projection (0: identity form)")
    ap.add_argument("--latency-form", action="store_true",
                    help="also time the step as per-layer decode calls replayed from one CUDA graph")
    ap.add_argument("--budget", type=int, default=0,
                    help="zoom budget per (layer, query head), keeping the largest routing logits; 0 = none "
                         "(the configs run without one)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "decode_kernel_attend_c3_4layers.txt")


def profiled_traffic(workload: str):
    """DRAM bytes (read + write) per ATTEND launch from the committed ncu summary, or
    None when the summary covers another workload or the decode source has changed
    since the counters were taken."""
    import hashlib
    try:
        with open(PROFILE_SUMMARY) as f:
            text = f.read()
        with open(os.path.join(ROOT, "hierarchical_kv_cache_span_b200", "csrc", "sekv_decode.cu"), "rb") as f:
            h16 = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    if f"decode source sha256[:16] = {h16}" not in text:
        return None
    key = f"traffic_per_launch_bytes {workload} = "
    for line in text.splitlines():
        if line.startswith(key):
            return int(line[len(key):].strip())
    return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy read+write)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (earlier measurement on this pool)"


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms during a region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.dev), "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
def max_over_ranks(value: float, device=None) -> float:
    """The largest value over all ranks (timing is reported as the slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(base_seed: int, rank: int) -> int:
    """Each rank runs an independent replica of the workload (its own sequences)."""
    return base_seed + 1000 * rank


def throughput(world: int, steps: int, elapsed_ms: float) -> float:
    """Whole-job steps/s: every rank completes `steps` steps in the slowest rank's time."""
    return world * steps / (elapsed_ms * 1e-3)


def calibrate_theta(cache, q, quantile, P, torch):
    """Per (layer, query head): theta at the target quantile of the routing logits
    of a calibration query (the learned per-head thresholds are not available)."""
    rl = torch.full((cache.B, cache.L, cache.Hq, cache.m_cap), float("nan"), device="cuda")
    zm = cache.new_zmask()
    th0 = torch.zeros(cache.L, cache.Hq, device="cuda")
    cache.decode(q, th0, phase=P.SEKV_ROUTE, zmask=zm, route_logits=rl)
    torch.cuda.synchronize()
    m = cache.m_count.cpu()
    theta = torch.zeros(cache.L, cache.Hq)
    rl = rl.cpu()
    for l in range(cache.L):
        for h in range(cache.Hq):
            x = torch.cat([rl[b, l, h, :int(m[b])] for b in range(cache.B)])
            x, _ = torch.sort(x)
            if x.numel() < 2:
                theta[l, h] = 0.0
                continue
            k = min(int(quantile * x.numel()), x.numel() - 1)     # (1 - quantile) of spans above
            theta[l, h] = 0.5 * (x[k - 1] + x[k]) if k >= 1 else x[0] - 1.0
    return theta.cuda()


def attend_bytes(cache, zmask_host, P):
    """Algorithmic bytes of one ATTEND/FUSED call: per (b, l, kv head) the anchor
    K/V rows, kbar/vbar rows, 1/||kbar|| and log|S|, the bases of every span any
    of its G query heads zooms, the G queries and the G outputs + lse."""
    import numpy as np
    c = cache
    s = 2 if c.dtype_name == "bf16" else 4
    G = c.Hq // c.Hkv
    a = c.a_count.cpu().numpy()
    m = c.m_count.cpu().numpy()
    span_len = (c.span_end - c.span_beg).cpu().numpy()
    z = np.ascontiguousarray(zmask_host).view(np.uint32).reshape(c.B, c.L, c.Hkv, G, -1)
    unions = np.bitwise_or.reduce(z, axis=3)                     # [B][L][Hkv][mw]
    total = 0
    zoom_units = 0
    for b in range(c.B):
        mb = int(m[b])
        blk = np.array([P.sekv.sekv_block_elems(int(x), c.d, c.rank) for x in span_len[b, :mb]], dtype=np.int64) * s
        bits = np.unpackbits(unions[b].view(np.uint8), axis=-1, bitorder="little")[..., :mb].astype(bool)
        base = 2 * int(a[b]) * c.d * s + 2 * mb * c.d * s + 8 * mb + G * c.d * s + G * (c.d + 1) * 4
        total += base * c.L * c.Hkv + int((bits * blk[None, None, :]).sum())
        zoom_units += int(bits.sum())
    return total, zoom_units


FP32_LANES_PER_SM = 128      # B200: 4 SM sub-partitions x 32 fp32 FMA lanes


def basis_work(cache, layers, P):
    """Operation counts of the basis build (BASES step) from the realised span
    lengths, per the algorithm the kernel runs (one problem per span, kv head, layer
    and side K / V; X is |S| x d, N = min(|S|, d), rS = min(r, |S|, d)):
    Gram 2 N^2 max(|S|, d) (tensor cores); Householder tridiagonalisation 4/3 N^3;
    back-transformation of rS vectors 2 rS N^2; factors 2 rS |S| d (fp32). The
    eigenvalue / eigenvector steps on the tridiagonal are O(rS N) and left out.
    Also the bytes the step must move: K, V read once, factors written."""
    import numpy as np
    c = cache
    s = 2 if c.dtype_name == "bf16" else 4
    ln = (c.span_end - c.span_beg).cpu().numpy().astype(np.float64)
    m = c.m_count.cpu().numpy()
    gram = f32 = 0.0
    wbytes = 0
    for b in range(c.B):
        L_ = ln[b, :int(m[b])]
        N = np.minimum(L_, c.d)
        rS = np.minimum(np.minimum(L_, c.d), c.rank)
        gram += float(np.sum(2 * N ** 2 * np.maximum(L_, c.d)))
        f32 += float(np.sum(4.0 / 3.0 * N ** 3 + 2 * rS * N ** 2 + 2 * rS * L_ * c.d))
        wbytes += int(sum(c.Hkv * P.sekv.sekv_block_elems(int(x), c.d, c.rank) for x in L_)) * s
    per = 2 * layers * c.Hkv                 # K and V, every layer and kv head
    return {"tensor_flops": gram * per, "fp32_flops": f32 * per,
            "bytes": int(2 * c.B * layers * c.Hkv * c.n * c.d * s + wbytes * layers)}


def route_bytes(cache, learned):
    """Algorithmic bytes of one ROUTE call without a budget. Identity form: per
    (b, l, kv head) the kbar rows, 1/||kbar|| and log|S| once, the G queries and the
    G mask rows. Learned form: per (b, l, query head) its dr-wide routing summaries,
    log|S|, its query and d' x d projection, and its mask row."""
    c = cache
    s = 2 if c.dtype_name == "bf16" else 4
    G = c.Hq // c.Hkv
    mw = c.m_cap // 32
    tot = 0
    for b in range(c.B):
        m = int(c.m_count[b])
        if learned:
            tot += c.L * c.Hq * (m * c.dr * s + m * 4 + c.d * s + c.dr * c.d * s + mw * 4)
        else:
            tot += c.L * c.Hkv * (m * c.d * s + 8 * m + G * c.d * s + G * mw * 4)
    return tot


def zoom_rate(cache, zmask_host):
    import numpy as np
    c = cache
    z = np.ascontiguousarray(zmask_host).view(np.uint32).reshape(c.B, c.L, c.Hq, -1)
    m = c.m_count.cpu().numpy()
    tot = sum(int(np.unpackbits(z[b].view(np.uint8), axis=-1, bitorder="little")[..., :int(m[b])].sum())
              for b in range(c.B))
    return tot / max(1, int(m.sum()) * c.L * c.Hq)


# ---------------------------------------------------------------------------
# CPU oracle timing (bounded sample, spawn pool)
def _oracle_unit_task(args):
    import numpy as np
    import oracle as O
    kv_path, H, alpha, window, wmode, rank, dtype, q, theta, quantile, scale, reps, budget, W = args
    with np.load(kv_path) as f:
        K, V = f["K"].astype(np.float64), f["V"].astype(np.float64)
    seg = O.segment(H, alpha, window)
    t0 = time.perf_counter()
    u = O.build_unit(K, V, H, seg, wmode, rank, dtype, W=W)
    t_build = time.perf_counter() - t0

    def route(g):
        if W is not None:
            return O.learned_routing_logits(q[g], u.W[g], u.kbar_r[g], u.logS)
        return O.routing_logits(q[g], u.kbar, u.inv_norm, u.logS, scale)

    if theta is None:             # calibrate on the oracle's own routing logits
        theta = []
        for g in range(q.shape[0]):
            x = np.sort(route(g))
            k = int(round(quantile * (x.size - 1)))
            theta.append(0.5 * (x[min(k, x.size - 1)] + x[min(k + 1, x.size - 1)]))
    times = []
    for _ in range(reps):
        t0 = time.perf_counter()
        z = np.stack([O.zoom_decisions(route(g), theta[g], budget=budget or None) for g in range(q.shape[0])])
        O.decode_unit(q, u.Ka, u.Va, u.kbar, u.vbar, u.logS, z, u.bases, scale)
        times.append(time.perf_counter() - t0)
    return t_build, times


def oracle_sample(wl, H, KV_units, q, theta, reps, workers, quantile=None, budget=0, W=None):
    """Time the oracle on the sampled (layer, kv head) units (one per process of a
    spawn pool). K/V of each unit go through a temporary .npz file (float32 holds
    the bf16 values exactly). Returns per-unit build seconds and decode seconds."""
    import numpy as np
    scale = 1.0 / math.sqrt(wl.d)
    G = wl.Hq // wl.Hkv
    tmp = tempfile.mkdtemp(prefix="sekv_oracle_")
    tasks = []
    try:
        for i, ((l, h), (K, V)) in enumerate(KV_units.items()):
            path = os.path.join(tmp, f"u{i}.npz")
            np.savez(path, K=K, V=V)
            th = None if theta is None else theta[l, h * G:(h + 1) * G]
            Wu = None if W is None else W[l, h * G:(h + 1) * G]
            tasks.append((path, H, wl.alpha, wl.window, wl.wmode, wl.rank, wl.dtype,
                          q[l, h * G:(h + 1) * G], th, quantile, scale, reps, budget, Wu))
        ctx = mp.get_context("spawn")
        saved = {k: os.environ.get(k) for k in _BLAS_ENV}
        os.environ.update({k: "1" for k in _BLAS_ENV})      # one BLAS thread per worker process
        try:
            with ctx.Pool(processes=workers) as pool:
                res = pool.map(_oracle_unit_task, tasks)
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
    finally:
        for fn in os.listdir(tmp):
            os.unlink(os.path.join(tmp, fn))
        os.rmdir(tmp)
    return [r[0] for r in res], [r[1] for r in res]


# ---------------------------------------------------------------------------
def build_workload(args):
    from sekv_synth import WORKLOADS
    wl = WORKLOADS[args.workload]
    over = {}
    if args.n:
        over["n"] = args.n
    if args.layers:
        over["L"] = args.layers
    return wl.scaled(**over) if over else wl


def caps_for(wl):
    a_cap = ((wl.n // 32 + wl.window + 256 + 31) // 32) * 32
    m_cap = ((wl.n // 32 + 256 + 31) // 32) * 32
    return a_cap, m_cap


def run_sekv(args, rank, world, local_rank):
    import numpy as np
    import torch
    import hierarchical_kv_cache_span_b200 as P
    from sekv_synth import gen

    torch.cuda.set_device(local_rank)
    wl = build_workload(args)
    wl = wl.scaled(seed=replica_seed(wl.seed, rank))     # independent replica per rank
    G = wl.Hq // wl.Hkv
    cold = wl.basis_home == "host"
    a_cap, m_cap = caps_for(wl)
    dev = torch.device("cuda", local_rank)

    # ---- synthetic inputs (seeded generators), on the device
    H, spikes = gen.surprisal(wl, device=dev)
    K, V = gen.keys_values(wl, spikes, device=dev)
    cache = P.SpanCache(wl.B, wl.L, wl.Hq, wl.Hkv, wl.n, wl.d, wl.dtype, a_cap, m_cap, wl.rank,
                        home=None, device=dev)
    learned = args.route_dim > 0
    if learned:
        cache.set_routing(gen.route_projection(wl, args.route_dim, device=dev))
    # ---- prefill build, timed by step
    ev = lambda: torch.cuda.Event(enable_timing=True)
    seg_e = [ev(), ev()]
    seg_e[0].record()
    cache.build(H, None, None, wl.alpha, wl.window, wl.wmode, steps=P.SEKV_BUILD_SCAN | P.SEKV_BUILD_LAYOUT)
    seg_e[1].record()
    torch.cuda.synchronize()
    P.check(cache.read_status(), "segmentation")
    region = cache.exact_region()
    cache.alloc_home("host" if cold else "device", region)
    sum_e = [ev(), ev()]
    bas_e = [ev(), ev()]
    sum_e[0].record()
    cache.build(H, K, V, wl.alpha, wl.window, wl.wmode, steps=P.SEKV_BUILD_SUMMARY)
    sum_e[1].record()
    bas_e[0].record()
    cache.build(H, K, V, wl.alpha, wl.window, wl.wmode, steps=P.SEKV_BUILD_BASES)
    bas_e[1].record()
    torch.cuda.synchronize()
    st = cache.read_status()
    if st not in (0, P.sekv.SEKV_WARN_NOT_CONVERGED):
        raise RuntimeError(f"build status {P.sekv.sekv_status_str(st)}")
    cache.clear_status()
    kv_bytes = 2 * K.numel() * K.element_size()
    build = {
        "segment_ms": seg_e[0].elapsed_time(seg_e[1]),
        "summary_ms": sum_e[0].elapsed_time(sum_e[1]),
        "bases_ms": bas_e[0].elapsed_time(bas_e[1]),
        "bases_home": "pinned host" if cold else "device",
        "summary_kv_read_GBps": kv_bytes / (sum_e[0].elapsed_time(sum_e[1]) * 1e-3) / 1e9,
        "not_converged_warning": st == P.sekv.SEKV_WARN_NOT_CONVERGED,
    }
    build["total_ms"] = build["segment_ms"] + build["summary_ms"] + build["bases_ms"]
    try:
        bw = basis_work(cache, wl.L, P)
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        sec = build["bases_ms"] * 1e-3
        build["bases_work"] = {
            "fp32_tflop": bw["fp32_flops"] / 1e12, "tensor_tflop": bw["tensor_flops"] / 1e12,
            "fp32_TFLOPs": bw["fp32_flops"] / sec / 1e12, "tensor_TFLOPs": bw["tensor_flops"] / sec / 1e12,
            "GBps": bw["bytes"] / sec / 1e9,
            "fp32_peak_TFLOPs": sms * FP32_LANES_PER_SM * 2 * 1.965e9 / 1e12,
            "note": "counts from the realised span lengths (Gram on tensor cores; tridiagonalisation, "
                    "back-transformation and factors in fp32); fp32 peak = SMs x 128 lanes x 2 x 1965 MHz "
                    "(nominal, from unit counts and the maximum clock)"}
        build["bases_work"]["fp32_frac"] = build["bases_work"]["fp32_TFLOPs"] / build["bases_work"]["fp32_peak_TFLOPs"]
    except Exception as e:                            # context only; never fatal to the line
        build["bases_work"] = {"error": f"{type(e).__name__}: {e}"}

    # sample units for the CPU oracle before K/V are freed
    cpu_units = {}
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    workers = max(1, min(8, (os.cpu_count() or 2) - 1))
    if want_cpu:
        for i in range(workers):
            l, h = (i * 7) % wl.L, i % wl.Hkv
            cpu_units[(l, h)] = (K[0, l, h].float().cpu().numpy(), V[0, l, h].float().cpu().numpy())
        H0 = H[0].double().cpu().numpy()
    del K, V, spikes
    torch.cuda.empty_cache()

    # ---- queries: a pool of device-resident inputs, thresholds
    steps, warm = args.steps, args.warmup
    qpool = [gen.queries(wl, step=s_, device=dev) for s_ in range(warm + steps)]
    if wl.tau_kind == "quantile":
        theta = calibrate_theta(cache, gen.queries(wl, step=10 ** 6, device=dev), wl.tau_a, P, torch)
    else:
        theta = P.tau_to_theta(gen.taus(wl)).to(dev)
    O, lse = cache.new_outputs()
    zm = cache.new_zmask()
    comp = torch.cuda.current_stream()
    # zoom_hint: zoomed spans per (b, l, kv head), the union over the group's query
    # heads, from one routing pass with a query outside the timed pool (a previous
    # step's count, as a serving loop would pass it)
    cache.decode(gen.queries(wl, step=10 ** 6 + 1, device=dev), theta, phase=P.SEKV_ROUTE, zmask=zm,
                 budget=args.budget)
    zw_ = zm.view(torch.int32).cpu().numpy().view(np.uint32).reshape(wl.B, wl.L, wl.Hkv, wl.Hq // wl.Hkv, -1)
    union = np.bitwise_or.reduce(zw_, axis=3)
    zoom_hint = int(np.unpackbits(union.view(np.uint8), axis=-1).sum() // max(1, wl.B * wl.L * wl.Hkv))
    zm.zero_()

    fetcher = None
    if cold:
        # size the arena from a calibration step: 3x its zoomed bytes
        cache.decode(qpool[0], theta, phase=P.SEKV_ROUTE, zmask=zm, budget=args.budget)
        probe = P.ColdFetcher(cache, arena_elems=64)
        try:
            probe.fetch(zm)
            need = probe.stats[0].item()
        except P.SekvError:
            need = int(probe.stats[0].item())
        es = 2 if wl.dtype == "bf16" else 4
        del probe
        fetcher = P.ColdFetcher(cache, arena_elems=max(1 << 20, 3 * need // es), keep=args.cache)

    # descriptors are built once; each step copies its query into q_buf and calls the C ABI
    q_buf = torch.empty_like(qpool[0])
    sid = comp.cuda_stream
    bud = args.budget
    if cold:
        d_route = cache.decode_desc(q_buf, theta, phase=P.SEKV_ROUTE, zmask=zm, budget=bud, static_ready=True)
        d_attn = cache.decode_desc(q_buf, theta, phase=P.SEKV_ATTEND, O=O, lse=lse, slot=fetcher.slot_dev,
                                   arena=fetcher.arena, zmask=zm, budget=bud, zoom_hint=zoom_hint,
                                   static_ready=True)
    else:
        d_attn = cache.decode_desc(q_buf, theta, phase=P.SEKV_FUSED, O=O, lse=lse, zmask=zm, budget=bud,
                                   zoom_hint=zoom_hint, static_ready=True)

    def one_step(q, rec=None):
        if q is not None:
            q_buf.copy_(q, non_blocking=True)
        if cold:
            if rec: rec[0].record()
            P.check(P.sekv.sekv_decode_attn(d_route, sid), "route")
            if rec: rec[1].record()
            info = fetcher.fetch(zm)
            comp.wait_event(fetcher.done)
            if rec: rec[2].record()
            P.check(P.sekv.sekv_decode_attn(d_attn, sid), "attend")
            if rec: rec[3].record()
            return info
        if rec: rec[0].record(); rec[1].record(); rec[2].record()
        P.check(P.sekv.sekv_decode_attn(d_attn, sid), "fused")
        if rec: rec[3].record()
        return None

    for s_ in range(warm):
        one_step(qpool[s_])
    torch.cuda.synchronize()
    if cache.read_status() != 0:
        raise RuntimeError(f"decode status {P.sekv.sekv_status_str(cache.read_status())}")

    # ---- timed region: device-resident inputs
    import torch.distributed as dist
    recs = [[ev() for _ in range(4)] for _ in range(steps)]
    zhost, fetched = [], []
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = ev(), ev()
    t0.record()
    for i in range(steps):
        info = one_step(qpool[warm + i], recs[i])
        if cold:
            fetched.append(info)
            zhost.append(fetcher.zmask_host.numpy().copy())
    t1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    elapsed_ms = t0.elapsed_time(t1)
    if not cold:
        zhost.append(zm.cpu().numpy())
    elapsed_ms = max_over_ranks(elapsed_ms, dev)
    if cache.read_status() != 0:
        raise RuntimeError(f"decode status {P.sekv.sekv_status_str(cache.read_status())}")
    route_ms = [r[0].elapsed_time(r[1]) for r in recs]
    fetch_ms = [r[1].elapsed_time(r[2]) for r in recs]
    attn_ms = [r[2].elapsed_time(r[3]) for r in recs]
    by = [attend_bytes(cache, zh, P) for zh in (zhost if cold else zhost * steps)]
    alg_bytes = statistics.mean(b[0] for b in by)
    attn_avg = statistics.mean(attn_ms)
    peak, peak_src = measured_peaks()
    achieved = alg_bytes / (attn_avg * 1e-3) / 1e9
    zr = statistics.mean(zoom_rate(cache, zh) for zh in zhost)
    ms_per_step = elapsed_ms / steps
    value = throughput(world, steps, elapsed_ms)

    # ---- e2e through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        q_host = [q.cpu().pin_memory() for q in qpool[warm:warm + steps]]
        qd = q_buf
        O_h = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
        l_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = ev(), ev()
        e0.record()
        h2d_extra = 0
        for i in range(steps):
            qd.copy_(q_host[i], non_blocking=True)
            info = one_step(None)
            if info:
                h2d_extra += info["bytes"] + cache.B * cache.L * cache.m_cap * 8
            O_h.copy_(O, non_blocking=True)
            l_h.copy_(lse, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        qb = qpool[0].numel() * qpool[0].element_size()
        e2e = {"value": throughput(world, steps, e_ms), "unit": "steps/s",
               "h2d_bytes_per_step": int(qb + h2d_extra / steps),
               "d2h_bytes_per_step": int(O.numel() * 4 + lse.numel() * 4),
               "note": "per step: q H2D from pinned host, ROUTE, fetch (zmask D2H, bases + slot table H2D), "
                       "ATTEND, O and lse D2H; h2d counts q + fetched bases + slot table"}

    # ---- CPU oracle baseline (rank 0, N = 1)
    cpu = None
    if want_cpu:
        qs = qpool[warm].double().cpu().numpy()[0]
        th = theta.double().cpu().numpy()
        Wn = cache.route_W.double().cpu().numpy() if learned else None
        t_build, t_dec = oracle_sample(wl, H0, cpu_units, qs, th, reps=2, workers=workers, budget=args.budget,
                                       W=Wn)
        per_unit = statistics.mean(min(t) for t in t_dec)
        units_total = wl.B * wl.L * wl.Hkv
        oracle_step_s = per_unit * units_total / workers
        cpu = {"value": 1.0 / oracle_step_s, "unit": "steps/s", "cores": workers, "kind": "oracle",
               "cpu_model": cpu_model(),
               "sample": f"{workers} (layer, kv-head) units of one decode step, one unit per process "
                         f"(spawn pool, 1 BLAS thread each); per-unit decode time x {units_total} units / "
                         f"{workers} cores. Oracle build of those units: mean {statistics.mean(t_build):.2f} s/unit",
               "oracle_build_s_per_unit": statistics.mean(t_build)}

    # ROUTE + ATTEND (cold) or FUSED (hot), each one decode_kernel launch (the split-K
    # merge runs in its last CTA per unit); a budget adds the cap kernel, and on the
    # hot path the routing pass before the capped FUSED pass (learned routing: its own
    # routing kernel before the attention pass)
    if cold or learned:
        launches_per_step = 2 + (1 if args.budget else 0)
    else:
        launches_per_step = 1 + (2 if args.budget else 0)
    rb = route_bytes(cache, learned)
    route_avg = statistics.mean(route_ms)
    from sekv_synth import WORKLOADS as _WL
    full_size = (wl.L, wl.n) == (_WL[wl.name].L, _WL[wl.name].n)
    kv_total = kv_bytes
    out = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": steps, "warmup": warm,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic (seeded generators standing in for the pages' 128K workloads)",
        "config": {"workload": f"{wl.name}: {'cold' if cold else 'hot'} bases, {wl.n // 1024}K ctx, batch {wl.B}, "
                               f"{wl.L} layers, {wl.Hq}q/{wl.Hkv}kv heads, d={wl.d}, rank {wl.rank}, "
                               f"{wl.dtype} K/V, tau {wl.tau_kind} {wl.tau_a}",
                   "B": wl.B, "n": wl.n, "L": wl.L, "Hq": wl.Hq, "Hkv": wl.Hkv, "d": wl.d, "rank": wl.rank,
                   "anchors": int(cache.a_count.sum()), "spans": int(cache.m_count.sum()),
                   "l2": f"inputs larger than L2 ({alg_bytes / 1e6:.0f} MB read per ATTEND)",
                   "parallelism": f"replicas x{world} (no collective)",
                   **({"budget": args.budget} if args.budget else {}),
                   **({"routing": f"learned form, d'={args.route_dim} (seeded projection)"} if learned else {})},
        "decode_attn": {"us_per_step": attn_avg * 1e3, "steps_per_s": 1e3 / attn_avg,
                        "alg_bytes_per_step": int(alg_bytes), "GBps": achieved,
                        "us_p10_median_p90": [pct(attn_ms, 10) * 1e3, pct(attn_ms, 50) * 1e3,
                                              pct(attn_ms, 90) * 1e3]},
        "route_us": route_avg * 1e3,
        **({"route": {"form": "learned" if learned else "identity", "alg_bytes": rb,
                      "GBps": rb / (route_avg * 1e-3) / 1e9, "frac": rb / (route_avg * 1e-3) / 1e9 / peak,
                      "note": "the ROUTE call of the cold path (no budget): summaries, log|S|, queries, "
                              "projections and mask words"}} if cold and route_avg > 0 else {}),
        "zoom_rate": zr,
        "zoom_hint": zoom_hint,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": profiled_traffic(wl.name) if full_size else None,
                     "traffic_unit": "DRAM bytes read + written per ATTEND launch (ncu, profiles/)",
                     "kernel": "sekv_decode_attn ATTEND call (one decode_kernel launch; the split-K merge runs in its last CTA per unit)",
                     "peak_source": peak_src, "frac_of_8TBps_nominal": achieved / 8000.0},
        "prefill_build": build,
        "gpu_launches": launches_per_step * steps,
        "clocks": clk,
    }
    if cold:
        fb = statistics.mean(f["bytes"] for f in fetched)
        out["fetch"] = {"ms": statistics.mean(fetch_ms), "bytes_per_step": int(fb),
                        "GBps": fb / (statistics.mean(fetch_ms) * 1e-3) / 1e9,
                        "copies_per_step": statistics.mean(f["copies"] for f in fetched),
                        "note": "includes the zmask read-back and the host wait for the routing result"}
        if args.cache:
            out["fetch"]["cache"] = "device cache across steps (resident spans not copied again)"
            out["fetch"]["resident_spans_per_step"] = statistics.mean(f["resident"] for f in fetched)
            out["fetch"]["copied_spans_per_step"] = statistics.mean(f["spans"] for f in fetched)
            out["config"]["fetch"] = "cached across steps"
    try:
        out["memory"] = memory_model(cache, cold)
    except Exception as e:                            # context only; never fatal to the line
        out["memory"] = {"error": f"{type(e).__name__}: {e}"}
    if cold:
        try:
            pk = h2d_peak(torch, dev)
            out["fetch"]["h2d_peak_GBps"] = pk
            out["fetch"]["frac_of_h2d_peak"] = out["fetch"]["GBps"] / pk
        except Exception as e:                        # context only; never fatal to the line
            out["fetch"]["h2d_peak_GBps"] = None
            out["fetch"]["h2d_peak_error"] = f"{type(e).__name__}: {e}"
    if e2e:
        out["e2e"] = e2e
    if cpu:
        out["cpu_baseline"] = cpu
    if args.latency_form:
        out["latency_form"] = latency_form(P, torch, cache, wl, q_buf, qpool[warm], theta, O, lse, zm, fetcher,
                                           cold, learned, bud, zoom_hint, steps)
        if cold and args.cache:
            out["latency_form"]["prefetch_pipeline"] = prefetch_pipeline(
                P, torch, cache, wl, q_buf, qpool, theta, O, lse, zm, fetcher.arena.numel(), bud, zoom_hint,
                steps, warm)
    return out


def memory_model(cache, cold: bool):
    """SeKV blog §2.3 Eq. (17): GPU-resident bytes 2·L·H_kv·d·(a+w)·b (anchors, the
    window included in a) + 2·L·H·d'·m·b (span summaries), from the realised anchor
    and span counts, beside the buffers the cache actually holds on the device and
    the full KV cache of the same context. The summaries here are kbar and vbar per
    kv head (d' = d, H = H_kv) plus, with learned routing, the d'-wide routing
    summaries per query head; bases count only when they live on the device."""
    c = cache
    s = 2 if c.dtype_name == "bf16" else 4
    a = int(c.a_count.clamp(max=c.a_cap).sum())
    m = int(c.m_count.clamp(max=c.m_cap).sum())
    anchors = 2 * c.L * c.Hkv * c.d * a * s
    summaries = 2 * c.L * c.Hkv * c.d * m * s
    routing = c.L * c.Hq * c.dr * m * s if c.kbar_r is not None else 0
    meta = c.L * c.Hkv * m * 4 + m * 4            # 1/||kbar|| and log|S|
    bufs = [c.Ka, c.Va, c.kbar, c.vbar, c.inv_norm, c.logS, c.anchor_pos, c.span_beg, c.span_end, c.blk_off]
    if c.kbar_r is not None:
        bufs.append(c.kbar_r)
    allocated = sum(t.numel() * t.element_size() for t in bufs)
    home = c.home.numel() * c.home.element_size() if c.home is not None else 0
    full_kv = 2 * c.B * c.L * c.Hkv * c.n * c.d * s
    eq17 = anchors + summaries + routing + meta
    return {"eq17_bytes": eq17, "anchors_bytes": anchors, "summaries_bytes": summaries + routing + meta,
            "allocated_bytes": allocated + (0 if cold else home),
            "bases_bytes": home, "bases_on": "pinned host" if cold else "device",
            "full_kv_bytes": full_kv, "eq17_over_full_kv": eq17 / full_kv,
            "note": "allocated = the cache's device buffers at their capacities (a_cap, m_cap)"
                    + ("" if cold else " plus the device-resident bases")}


def pct(xs, p):
    """p-th percentile (nearest rank) of a list of timings"""
    ys = sorted(xs)
    return ys[min(len(ys) - 1, max(0, int(round(p / 100.0 * (len(ys) - 1)))))]


def h2d_peak(torch, dev, nbytes=512 << 20):
    """pinned host -> device copy rate of one large copy (the ceiling the fetch is held to)"""
    src = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    for _ in range(2):
        dst.copy_(src, non_blocking=True)
    best = None
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dst.copy_(src, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1)
        best = t if best is None else min(best, t)
    return nbytes / (best * 1e-3) / 1e9


def latency_form(P, torch, cache, wl, q_buf, q, theta, O, lse, zm, fetcher, cold, learned, bud, zoom_hint, steps):
    """The step as L per-layer decode calls (l0 = l, l1 = l + 1) replayed from one CUDA
    graph. Cold bases: the graph holds the per-layer ATTEND calls after one ROUTE +
    fetch outside it (the fetch waits on the host and cannot be captured)."""
    try:
        q_buf.copy_(q)
        if cold:
            dr_ = cache.decode_desc(q_buf, theta, phase=P.SEKV_ROUTE, zmask=zm, budget=bud, static_ready=True)
            P.check(P.sekv.sekv_decode_attn(dr_, torch.cuda.current_stream().cuda_stream), "route")
            fetcher.fetch(zm)
            torch.cuda.current_stream().wait_event(fetcher.done)
        descs = []
        for l in range(wl.L):
            if cold:
                descs.append(cache.decode_desc(q_buf, theta, phase=P.SEKV_ATTEND, O=O, lse=lse,
                                               slot=fetcher.slot_dev, arena=fetcher.arena, zmask=zm, budget=bud,
                                               zoom_hint=zoom_hint, l0=l, l1=l + 1, static_ready=True))
            else:
                descs.append(cache.decode_desc(q_buf, theta, phase=P.SEKV_FUSED, O=O, lse=lse, zmask=zm,
                                               budget=bud, zoom_hint=zoom_hint, l0=l, l1=l + 1, static_ready=True))
        torch.cuda.synchronize()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):                 # one eager pass (first-use setup outside the capture)
            for d_ in descs:
                P.check(P.sekv.sekv_decode_attn(d_, side.cuda_stream), "per-layer decode")
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="relaxed"):
            sid = torch.cuda.current_stream().cuda_stream
            for d_ in descs:
                P.check(P.sekv.sekv_decode_attn(d_, sid), "per-layer decode (capture)")
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(max(steps, 5)):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        st = cache.read_status()
        del g
        return {"us_per_step": statistics.median(ts) * 1e3, "us_p10": pct(ts, 10) * 1e3, "us_p90": pct(ts, 90) * 1e3,
                "calls_per_step": wl.L, "status": st,
                "note": ("per-layer ATTEND calls" if cold else "per-layer FUSED calls") +
                        " captured in one CUDA graph; L2 is not flushed between replays (each replay reads "
                        "the whole step, far above L2)"}
    except Exception as e:                            # reported, never fatal to the main line
        return {"error": f"{type(e).__name__}: {e}"}


def prefetch_pipeline(P, torch, cache, wl, q_buf, qpool, theta, O, lse, zm, arena_elems, bud, zoom_hint, steps,
                      warm):
    """The serving loop's cold step, layer by layer, with the fetch overlapped: layer
    l + 1 is routed before layer l attends, and its zoomed bases are fetched on the
    copy stream (after that routing event, into the keep-mode device cache) while
    layer l attends. The host takes part in every layer (the fetch reads the routing
    result), so the step is timed with events around the whole loop, not replayed
    from a graph."""
    try:
        fetcher = P.ColdFetcher(cache, arena_elems=arena_elems, keep=True)
        comp = torch.cuda.current_stream()
        sid = comp.cuda_stream
        route = [cache.decode_desc(q_buf, theta, phase=P.SEKV_ROUTE, zmask=zm, budget=bud, l0=l, l1=l + 1,
                                   static_ready=True) for l in range(wl.L)]
        attend = [cache.decode_desc(q_buf, theta, phase=P.SEKV_ATTEND, O=O, lse=lse, slot=fetcher.slot_dev,
                                    arena=fetcher.arena, zmask=zm, budget=bud, zoom_hint=zoom_hint, l0=l, l1=l + 1,
                                    static_ready=True) for l in range(wl.L)]
        evs = [torch.cuda.Event() for _ in range(wl.L)]
        stats = {"bytes": 0, "copies": 0, "resident": 0, "spans": 0, "evicted": 0}

        def step(t, q, count):
            q_buf.copy_(q, non_blocking=True)
            P.check(P.sekv.sekv_decode_attn(route[0], sid), "route")
            evs[0].record(comp)
            infos = [fetcher.fetch(zm, l0=0, l1=1, step=t, route_done=evs[0])]
            for l in range(wl.L):
                if l + 1 < wl.L:
                    P.check(P.sekv.sekv_decode_attn(route[l + 1], sid), "route")
                    evs[l + 1].record(comp)
                comp.wait_event(fetcher.done)
                P.check(P.sekv.sekv_decode_attn(attend[l], sid), "attend")
                if l + 1 < wl.L:
                    infos.append(fetcher.fetch(zm, l0=l + 1, l1=l + 2, step=t, route_done=evs[l + 1]))
            if count:
                for i in infos:
                    for k in stats:
                        stats[k] += i[k]

        for t in range(warm):
            step(t, qpool[t], False)
        torch.cuda.synchronize()
        ts = []
        for i in range(steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(comp)
            step(warm + i, qpool[warm + i], True)
            e1.record(comp)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        st = cache.read_status()
        return {"us_per_step": statistics.median(ts) * 1e3, "us_p10": pct(ts, 10) * 1e3,
                "us_p90": pct(ts, 90) * 1e3, "steps_per_s": 1e3 / statistics.median(ts), "status": st,
                "fetch_bytes_per_step": stats["bytes"] / steps, "copies_per_step": stats["copies"] / steps,
                "resident_spans_per_step": stats["resident"] / steps,
                "copied_spans_per_step": stats["spans"] / steps, "evicted_per_step": stats["evicted"] / steps,
                "note": "per layer: ROUTE(l+1), ATTEND(l), fetch(l+1) on the copy stream after ROUTE(l+1) "
                        "(keep-mode cache, arena as the main line's); i.i.d. queries"}
    except Exception as e:                            # reported, never fatal to the main line
        return {"error": f"{type(e).__name__}: {e}"}


def run_reference(args):
    """The fp64 oracle as the reference arm, on the host cores. Each step is a
    bounded sample of the workload's decode step: one (layer, kv head) unit per
    worker process, decoded once per step (W warm-up steps, then K timed steps).
    `ms_per_step` and `steps` describe that sample as it ran; `value` scales the
    sample to the whole step (units_total / units per sample), which the
    `extrapolation` field states."""
    import numpy as np
    import torch
    from sekv_synth import gen
    wl = build_workload(args)
    workers = max(1, min(8, (os.cpu_count() or 2) - 1))
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    H, spikes = gen.surprisal(wl, device=dev)
    units = {}
    for i in range(workers):
        l, h = (i * 7) % wl.L, i % wl.Hkv
        K, V = gen.keys_values(wl, spikes, device=dev, layers=range(l, l + 1))
        units[(l, h)] = (K[0, 0, h].float().cpu().numpy(), V[0, 0, h].float().cpu().numpy())
        del K, V
    H0 = H[0].double().cpu().numpy()
    q = gen.queries(wl, step=0).double().numpy()[0]
    # thresholds: fixed / drawn taus, or the oracle's own quantile calibration
    import oracle as O
    taus = gen.taus(wl)
    theta = O.tau_to_theta(taus.numpy()) if taus is not None else None
    W = gen.route_projection(wl, args.route_dim).double().numpy() if args.route_dim else None
    steps, warm = max(1, args.steps), max(0, args.warmup)
    t_build, t_dec = oracle_sample(wl, H0, units, q, theta, reps=warm + steps, workers=workers,
                                   quantile=wl.tau_a, budget=args.budget, W=W)
    # a sampled step runs the workers' units side by side: its time is the slowest unit's
    sample_ms = [1e3 * max(t[warm + i] for t in t_dec) for i in range(steps)]
    ms = statistics.mean(sample_ms)
    units_total = wl.B * wl.L * wl.Hkv
    scale_up = units_total / workers
    v = 1.0 / (ms * 1e-3 * scale_up)
    sample = (f"{workers} (layer, kv-head) units of one decode step per timed step, one unit per process on "
              f"{workers} host cores (spawn pool, 1 BLAS thread each); oracle build of the units outside the "
              f"timed steps (mean {statistics.mean(t_build):.2f} s per unit)")
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "steps/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": warm, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{wl.name}: {wl.n // 1024}K ctx, {wl.L} layers, {wl.Hq}q/{wl.Hkv}kv, "
                                   f"d={wl.d}, rank {wl.rank} (fp64 oracle)",
                       **({"budget": args.budget} if args.budget else {}),
                       **({"routing": f"learned form, d'={args.route_dim} (seeded projection)"}
                          if args.route_dim else {})},
            "extrapolation": {"units_per_timed_step": workers, "units_per_full_step": units_total,
                              "full_step_ms": ms * scale_up,
                              "note": "ms_per_step and steps are the sampled steps that ran; value = 1 / "
                                      "full_step_ms, the sample scaled to every (layer, kv head) unit"},
            "cpu_baseline": {"value": v, "unit": "steps/s", "cores": workers, "kind": "oracle", "sample": sample,
                             "cpu_model": cpu_model()},
            "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    args = parse_args(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0
    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        out = run_sekv(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
