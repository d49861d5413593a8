"""Cold-basis fetch with a device cache across steps (keep mode): spans that are
resident are not copied again, misses are appended, a full arena is flushed and
refilled. Every step must equal the hot FUSED decode exactly (same kernels, the
same factor bytes, only their addresses differ)."""
import math

import numpy as np
import pytest
import torch

from sekv_synth import WORKLOADS, gen
from tests import helpers as T

pytestmark = pytest.mark.gpu


def _lib():
    import hierarchical_kv_cache_span_b200 as P
    return P


def _caches(wl):
    P = _lib()
    H, K, V = T.make_inputs(wl)
    segs = T.oracle_segments(H, wl)
    units = T.oracle_units(K, V, H, segs, wl)
    ac, mc = T.caps(wl)
    hot = P.SpanCache(wl.B, wl.L, wl.Hq, wl.Hkv, wl.n, wl.d, wl.dtype, ac, mc, wl.rank)
    cold = P.SpanCache(wl.B, wl.L, wl.Hq, wl.Hkv, wl.n, wl.d, wl.dtype, ac, mc, wl.rank, home="host")
    T.upload_oracle_cache(hot, segs, units)
    T.upload_oracle_cache(cold, segs, units)
    return hot, cold, units, segs


def _step(P, hot, cold, fetch, q, th):
    zm_f = hot.new_zmask()
    O_f, lse_f = hot.decode(q, th, zmask=zm_f)
    zm = cold.new_zmask()
    cold.decode(q, th, phase=P.SEKV_ROUTE, zmask=zm)
    info = fetch.fetch(zm)
    torch.cuda.current_stream().wait_event(fetch.done)
    O_a, lse_a = cold.decode(q, th, phase=P.SEKV_ATTEND, slot=fetch.slot_dev, arena=fetch.arena)
    torch.cuda.synchronize()
    assert hot.read_status() == 0 and cold.read_status() == 0
    assert torch.equal(zm, zm_f)
    assert torch.equal(O_a, O_f) and torch.equal(lse_a, lse_f)
    return info


def test_keep_mode_reuses_resident_spans():
    P = _lib()
    wl = WORKLOADS["c3"].scaled(n=8192, L=2)
    hot, cold, units, segs = _caches(wl)
    scale = 1.0 / math.sqrt(wl.d)
    q0 = gen.queries(wl, step=0)
    theta, _ = T.thetas_with_margin(q0, units, segs, wl, scale, wl.G, quantile=0.9)
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    fetch = P.ColdFetcher(cold, arena_elems=cold.region * wl.L, keep=True)
    infos = [_step(P, hot, cold, fetch, gen.queries(wl, step=s).cuda(), th) for s in range(4)]
    assert infos[0]["resident"] == 0 and infos[0]["bytes"] > 0
    # with log|S| dominating the routing logits, later steps zoom mostly the same spans
    assert all(i["resident"] > 0 for i in infos[1:])
    assert sum(i["bytes"] for i in infos[1:]) < 3 * infos[0]["bytes"]
    # a repeated query copies nothing
    again = _step(P, hot, cold, fetch, gen.queries(wl, step=3).cuda(), th)
    assert again["bytes"] == 0 and again["copies"] == 0 and again["spans"] == 0 and again["resident"] > 0


def test_keep_mode_flushes_a_full_arena():
    P = _lib()
    wl = WORKLOADS["c3"].scaled(n=8192, L=2)
    hot, cold, units, segs = _caches(wl)
    scale = 1.0 / math.sqrt(wl.d)
    theta, _ = T.thetas_with_margin(gen.queries(wl, step=0), units, segs, wl, scale, wl.G, quantile=0.9)
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    # size the arena at the largest single step's need: every step fits alone, the
    # accumulated misses do not, so the cache must flush along the way
    probe = P.ColdFetcher(cold, arena_elems=cold.region * wl.L)
    steps = [gen.queries(wl, step=10 + s).cuda() for s in range(6)]
    need = 0
    for q in steps:
        zm = cold.new_zmask()
        cold.decode(q, th, phase=P.SEKV_ROUTE, zmask=zm)
        need = max(need, probe.fetch(zm)["bytes"] // 2)
        torch.cuda.synchronize()
    fetch = P.ColdFetcher(cold, arena_elems=need, keep=True)
    used = []
    for q in steps:
        _step(P, hot, cold, fetch, q, th)
        used.append(int(fetch.arena_used[0]))
    assert all(0 < u <= fetch.arena.numel() for u in used)
    assert any(b < a for a, b in zip(used, used[1:])), "expected at least one flush"


def test_keep_mode_capacity_error_empties_the_cache():
    P = _lib()
    wl = WORKLOADS["c3"].scaled(n=8192, L=1)
    hot, cold, units, segs = _caches(wl)
    scale = 1.0 / math.sqrt(wl.d)
    theta, _ = T.thetas_with_margin(gen.queries(wl, step=0), units, segs, wl, scale, wl.G, quantile=0.9)
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    fetch = P.ColdFetcher(cold, arena_elems=64, keep=True)
    zm = cold.new_zmask()
    cold.decode(gen.queries(wl, step=0).cuda(), th, phase=P.SEKV_ROUTE, zmask=zm)
    with pytest.raises(P.SekvError) as ei:
        fetch.fetch(zm)
    assert ei.value.status == P.sekv.SEKV_ERR_CAPACITY
    assert int(fetch.arena_used[0]) == 0
    assert (fetch.slot_host == -1).all()
