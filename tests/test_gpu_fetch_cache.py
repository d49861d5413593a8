"""Cold-basis fetch with a device cache across steps (keep mode): spans that are
resident are not copied again, misses go to free space, and the least recently
used spans that the current and previous step do not need are evicted when the
arena is full. Every step must equal the hot FUSED decode exactly (same kernels,
the same factor bytes, only their addresses differ). The per-layer pipeline
(route layer l + 1 and fetch its bases while layer l attends) is checked against
the oracle over several steps of temporally correlated queries."""
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


def _step(P, hot, cold, fetch, q, th, step=0):
    zm_f = hot.new_zmask()
    O_f, lse_f = hot.decode(q, th, zmask=zm_f)
    zm = cold.new_zmask()
    cold.decode(q, th, phase=P.SEKV_ROUTE, zmask=zm)
    info = fetch.fetch(zm, step=step)
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
    infos = [_step(P, hot, cold, fetch, gen.queries(wl, step=s).cuda(), th, step=s) for s in range(4)]
    assert infos[0]["resident"] == 0 and infos[0]["bytes"] > 0
    # with log|S| dominating the routing logits, later steps zoom mostly the same spans
    assert all(i["resident"] > 0 for i in infos[1:])
    assert sum(i["bytes"] for i in infos[1:]) < 3 * infos[0]["bytes"]
    # a repeated query copies nothing
    again = _step(P, hot, cold, fetch, gen.queries(wl, step=3).cuda(), th, step=4)
    assert again["bytes"] == 0 and again["copies"] == 0 and again["spans"] == 0 and again["resident"] > 0


def _zoomed_sets(P, cold, qs, th):
    """per step: {(b, l, S)} zoomed by any head of (b, l), from the library's ROUTE"""
    out = []
    for q in qs:
        zm = cold.new_zmask()
        cold.decode(q, th, phase=P.SEKV_ROUTE, zmask=zm)
        torch.cuda.synchronize()
        z = zm.cpu().numpy().view(np.uint32)
        sets = set()
        for b in range(cold.B):
            m = int(cold.m_count[b])
            for l in range(cold.L):
                u = np.bitwise_or.reduce(z[b, l], axis=0)
                bits = np.unpackbits(u.view(np.uint8), bitorder="little")[:m]
                sets |= {(b, l, int(S)) for S in np.flatnonzero(bits)}
        out.append(sets)
    return out


def _targeted_queries(cache, steps, gain=50.0):
    """Step t: query head h of layer l points at one span's mean key (a different span
    per step, head and layer), so that a high threshold zooms mostly those spans and
    the zoomed sets of different steps are nearly disjoint."""
    G = cache.Hq // cache.Hkv
    m = int(cache.m_count[0])
    kb = cache.kbar.float()
    out = []
    for t in range(steps):
        q = torch.zeros(cache.B, cache.L, cache.Hq, cache.d, device="cuda")
        for l in range(cache.L):
            for h in range(cache.Hq):
                S = (t * 97 + h * 13 + l * 5) % m
                v = kb[0, l, h // G, S]
                q[0, l, h] = gain * v / v.norm().clamp_min(1e-6)
        out.append(q.to(cache.dt))
    return out


def test_keep_mode_evicts_least_recently_used():
    P = _lib()
    wl = WORKLOADS["c3"].scaled(n=8192, L=2)
    hot, cold, units, segs = _caches(wl)
    th = torch.full((wl.L, wl.Hq), 7.0, dtype=torch.float32, device="cuda")
    steps = _targeted_queries(cold, 8)
    sets = _zoomed_sets(P, cold, steps, th)
    assert all(len(x) > 0 for x in sets)
    bo = cold.blk_off.cpu().numpy()
    size = lambda e: int(bo[e[0], e[2] + 1] - bo[e[0], e[2]])
    pair = max(sum(size(e) for e in (a | b)) for a, b in zip(sets, sets[1:]))
    total = sum(size(e) for e in set().union(*sets))
    arena = int(1.25 * pair) + 64
    # room for any two consecutive steps (never evicted), not for every span of the run
    assert arena < total
    fetch = P.ColdFetcher(cold, arena_elems=arena, keep=True)
    evicted = 0
    for t, q in enumerate(steps):
        slot0, last0 = fetch.slot_host.clone(), fetch.last_use.clone()
        info = _step(P, hot, cold, fetch, q, th, step=t)
        evicted += info["evicted"]
        slot1 = fetch.slot_host
        gone = (slot0 >= 0) & (slot1 < 0)
        kept_idle = (slot0 >= 0) & (slot1 >= 0) & (fetch.last_use < t)     # resident, not needed now
        assert int(gone.sum()) == info["evicted"]
        if info["evicted"]:
            # least recently used first: nothing evicted was used later than anything kept idle
            if kept_idle.any():
                assert int(last0[gone].max()) <= int(last0[kept_idle].min())
            assert int(last0[gone].max()) < t - 1
        # every span this step needs is resident and stamped
        for (b, l, S) in sets[t]:
            assert int(slot1[b, l, S]) >= 0 and int(fetch.last_use[b, l, S]) == t
        assert 0 < int(fetch.arena_used[0]) <= fetch.arena.numel()
    assert evicted > 0, "expected evictions"


def test_keep_mode_capacity_error_leaves_the_cache_as_it_was():
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
    assert (fetch.slot_host == -1).all() and (fetch.last_use == -1).all()
    assert (fetch.slot_dev == -1).all()


def _ar1_queries(wl, units, segs, theta, scale, steps, rho=0.9, delta=1e-3):
    """q_t = rho q_{t-1} + sqrt(1 - rho^2) e_t (a query model with temporal locality),
    e_t redrawn (seeded) until every routing logit of the units keeps `delta` from
    theta (the fp32 routing logit differs from the fp64 one by < 1e-5 here)"""
    G = wl.G
    g = torch.Generator().manual_seed(gen.unit_seed(wl.seed, 31))
    q = gen.queries(wl, step=0).float()
    out = []
    for t in range(steps):
        for attempt in range(200):
            e = torch.randn(q.shape, generator=g)
            cand = (rho * q + math.sqrt(1 - rho * rho) * e) if t else (q if attempt == 0 else e)
            qb = cand.to(torch.bfloat16)
            qn = T.f64(qb)
            ok = all(T.margin(T.unit_route(qn[b, l, kvh * G + h], u, h, scale), theta[l, kvh * G + h]) > delta
                     for (b, l, kvh), u in units.items() for h in range(G))
            if ok:
                break
        else:
            raise AssertionError("no AR(1) query with margins")
        q = cand
        out.append(qb)
    return out


def test_per_layer_prefetch_pipeline_matches_the_oracle():
    """Layer l + 1 is routed before layer l attends and its bases are fetched on the
    copy stream (after the routing event) while layer l attends; the keep-mode cache
    carries spans across steps. Per step: masks bit-exact and O / lse within the bf16
    tolerance of the oracle, and equal to per-layer hot FUSED calls."""
    P = _lib()
    wl = WORKLOADS["c3"].scaled(n=8192, L=3, Hq=8, Hkv=2)
    hot, cold, units, segs = _caches(wl)
    scale = 1.0 / math.sqrt(wl.d)
    theta, _ = T.thetas_with_margin(gen.queries(wl, step=0), units, segs, wl, scale, wl.G, quantile=0.9)
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    qs = _ar1_queries(wl, units, segs, theta, scale, steps=4)
    fetch = P.ColdFetcher(cold, arena_elems=cold.region * wl.L, keep=True)
    comp = torch.cuda.current_stream()
    hits = 0
    for t, q in enumerate(qs):
        qd = q.cuda()
        zm = cold.new_zmask()
        O, lse = cold.new_outputs()
        ev = torch.cuda.Event()
        cold.decode(qd, th, phase=P.SEKV_ROUTE, zmask=zm, l0=0, l1=1)
        ev.record(comp)
        info = fetch.fetch(zm, l0=0, l1=1, step=t, route_done=ev)
        hits += info["resident"]
        for l in range(wl.L):
            nxt = None
            if l + 1 < wl.L:
                cold.decode(qd, th, phase=P.SEKV_ROUTE, zmask=zm, l0=l + 1, l1=l + 2)
                nxt = torch.cuda.Event()
                nxt.record(comp)
            comp.wait_event(fetch.done)
            cold.decode(qd, th, phase=P.SEKV_ATTEND, O=O, lse=lse, slot=fetch.slot_dev, arena=fetch.arena, zmask=zm,
                        l0=l, l1=l + 1)
            if nxt is not None:
                hits += fetch.fetch(zm, l0=l + 1, l1=l + 2, step=t, route_done=nxt)["resident"]
        zm_f = hot.new_zmask()
        O_f, lse_f = hot.new_outputs()
        for l in range(wl.L):
            hot.decode(qd, th, O=O_f, lse=lse_f, zmask=zm_f, l0=l, l1=l + 1)
        torch.cuda.synchronize()
        assert cold.read_status() == 0 and hot.read_status() == 0
        assert torch.equal(zm, zm_f)
        Oo, lo, zooms = T.oracle_decode(q, units, segs, theta, scale, wl.G)
        for (b, l, h), z in zooms.items():
            np.testing.assert_array_equal(T.zmask_bits(zm, b, l, h, len(segs[b].spans)), z)
        assert np.abs(T.f64(O) - Oo).max() <= 2e-2
        assert np.abs(T.f64(lse) - lo).max() <= 2e-2
        assert (O - O_f).abs().max().item() <= 2e-3 and (lse - lse_f).abs().max().item() <= 2e-3
    assert hits > 0, "correlated queries should find resident spans"
