"""GPU parity of the decode attention against the fp64 oracle.

Kernel level: the oracle's own stored-dtype cache is uploaded, so both sides see
identical inputs; zoom masks must be bit-exact (routing logits kept DELTA_L away
from theta) and O / lse within 1e-4 (fp32) or 2e-2 (bf16 inputs, fp32
accumulation) max-abs. End to end: the library builds the cache itself.
Invariants: singleton spans and all-zoom full-rank reduce to dense attention; the
split count does not change the result; ROUTE + fetch + ATTEND equals FUSED.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from sekv_synth import WORKLOADS, gen
from tests import helpers as T
from tests.textbook import dense_attention

pytestmark = pytest.mark.gpu


def _lib():
    import hierarchical_kv_cache_span_b200 as P
    return P


def _tol(wl):
    return 1e-4 if wl.dtype == "f32" else 2e-2


def _cache(wl, home="device", a_cap=None, m_cap=None):
    P = _lib()
    ac, mc = T.caps(wl)
    return P.SpanCache(wl.B, wl.L, wl.Hq, wl.Hkv, wl.n, wl.d, wl.dtype, a_cap or ac, m_cap or mc,
                       wl.rank, home=home)


def _setup(wl, quantile=None, with_bases=True):
    """inputs + oracle cache + thresholds with margin"""
    H, K, V = T.make_inputs(wl)
    segs = T.oracle_segments(H, wl)
    units = T.oracle_units(K, V, H, segs, wl, with_bases=with_bases)
    q = gen.queries(wl)
    scale = 1.0 / math.sqrt(wl.d)
    taus = gen.taus(wl)
    if quantile is None and taus is None:
        quantile = wl.tau_a
    theta, q = T.thetas_with_margin(q, units, segs, wl, scale, wl.G, taus=taus, quantile=quantile)
    return H, K, V, segs, units, q, theta, scale


def _compare(wl, c, q, theta, scale, segs, units, O_gpu, lse_gpu, zmask):
    Oo, lseo, zooms = T.oracle_decode(q, units, segs, theta, scale, wl.G)
    for (b, l, h), z in zooms.items():
        np.testing.assert_array_equal(T.zmask_bits(zmask, b, l, h, len(z)), z, err_msg=str((b, l, h)))
    err = np.abs(T.f64(O_gpu) - Oo).max()
    lerr = np.abs(T.f64(lse_gpu) - lseo).max()
    assert err <= _tol(wl), err
    assert lerr <= _tol(wl), lerr
    return err, lerr, sum(int(z.sum()) for z in zooms.values())


KERNEL_CASES = [
    ("c1", dict()),                                         # fp32 tiny config, tau = 0.5
    ("c1", dict(n=777, window=40)),                         # ragged tail, window
    ("c2", dict(n=4096, L=2)),                              # Llama shape, bf16, ~2% zoom
    ("c4", dict(n=2048, L=2, B=3)),                         # batch, tau ~ U(0.3, 0.9)
    ("c5", dict(n=4096, L=1, Hq=8, Hkv=2)),                 # rank 32, 25% zoom
    ("c2", dict(n=2048, L=1, d=64, Hq=16, Hkv=2, rank=8)),  # G = 8, d = 64
    ("c2", dict(n=2048, L=1, Hq=16, Hkv=8)),                # G = 2
    ("c5", dict(n=2048, L=1, Hq=8, Hkv=2, rank=48)),        # d = 128, r = 48: two B / D pieces per span
    ("c5", dict(n=2048, L=1, Hq=8, Hkv=2, rank=20)),        # r8 = 24: odd count of 8-row basis blocks
    ("c5", dict(n=2048, L=1, d=64, Hq=4, Hkv=1, rank=64)),  # d = 64, r = 64
]


@pytest.mark.parametrize("name,over", KERNEL_CASES)
def test_decode_kernel_level(name, over):
    P = _lib()
    wl = WORKLOADS[name].scaled(**over)
    H, K, V, segs, units, q, theta, scale = _setup(wl)
    c = _cache(wl)
    T.upload_oracle_cache(c, segs, units)
    zmask = c.new_zmask()
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    O_gpu, lse_gpu = c.decode(q.cuda(), th, zmask=zmask)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    err, lerr, nz = _compare(wl, c, q, theta, scale, segs, units, O_gpu, lse_gpu, zmask)
    print(f"{name} {over}: max|dO|={err:.2e} max|dlse|={lerr:.2e} zoomed={nz}")


@pytest.mark.parametrize("name,over", KERNEL_CASES)
def test_attend_with_mask_matches_oracle(name, over):
    """ROUTE -> fetch -> ATTEND with ROUTE's mask as input, for every kernel-level
    shape: all layers in one call at two split counts, and one call per layer (a
    one-wave grid: the tensor-core path deals each unit's zoomed token units over
    its splits, cutting spans between them); every result against the oracle"""
    P = _lib()
    wl = WORKLOADS[name].scaled(**over)
    H, K, V, segs, units, q, theta, scale = _setup(wl)
    c = _cache(wl, home="host")
    T.upload_oracle_cache(c, segs, units)
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    qd = q.cuda()
    zm = c.new_zmask()
    c.decode(qd, th, phase=P.SEKV_ROUTE, zmask=zm)
    fetch = P.ColdFetcher(c, arena_elems=c.region * wl.L)
    fetch.fetch(zm)
    torch.cuda.current_stream().wait_event(fetch.done)
    kw = dict(phase=P.SEKV_ATTEND, slot=fetch.slot_dev, arena=fetch.arena, zmask=zm)
    results = []
    for ns in (0, 5):
        results.append(c.decode(qd, th, nsplit=ns, **kw))
    O_p, lse_p = c.new_outputs()
    for l in range(wl.L):
        c.decode(qd, th, O=O_p, lse=lse_p, l0=l, l1=l + 1, **kw)
    results.append((O_p, lse_p))
    torch.cuda.synchronize()
    assert c.read_status() == 0
    for O_gpu, lse_gpu in results:
        _compare(wl, c, q, theta, scale, segs, units, O_gpu, lse_gpu, zm)


@pytest.mark.parametrize("name,over", [
    ("c2", dict(n=2048, L=1, Hq=8, Hkv=2)),                 # r = 16
    ("c5", dict(n=1536, L=1, Hq=8, Hkv=2, rank=40)),        # r8 = 40: two B / D pieces, odd blocks
    ("c2", dict(n=1024, L=1, d=64, Hq=8, Hkv=1, rank=12)),  # d = 64, G = 8, r8 = 16 with rS = 12
])
def test_decode_all_zoom_matches_oracle(name, over):
    """theta = -inf: every span of every length is attended token by token through
    its bases (short spans with r_S = |S| < r included)."""
    wl = WORKLOADS[name].scaled(**over)
    H, K, V, segs, units, q, _, scale = _setup(wl)
    theta = np.full((wl.L, wl.Hq), -np.inf)
    c = _cache(wl)
    T.upload_oracle_cache(c, segs, units)
    zmask = c.new_zmask()
    th = torch.full((wl.L, wl.Hq), -math.inf, dtype=torch.float32, device="cuda")
    O_gpu, lse_gpu = c.decode(q.cuda(), th, zmask=zmask)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    err, lerr, nz = _compare(wl, c, q, theta, scale, segs, units, O_gpu, lse_gpu, zmask)
    assert nz == wl.L * wl.Hq * sum(len(s.spans) for s in segs)
    print(f"all-zoom {name} {over}: max|dO|={err:.2e} max|dlse|={lerr:.2e} zoomed={nz}")


@pytest.mark.parametrize("name,over", [("c1", dict()), ("c2", dict(n=4096, L=2)), ("c5", dict(n=2048, L=1))])
def test_decode_end_to_end(name, over):
    """library build (scan, summaries, bases) + decode vs oracle build + decode"""
    wl = WORKLOADS[name].scaled(**over)
    H, K, V, segs, units, q, theta, scale = _setup(wl)
    c = _cache(wl)
    c.build(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode)
    zmask = c.new_zmask()
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    O_gpu, lse_gpu = c.decode(q.cuda(), th, zmask=zmask)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    err, lerr, nz = _compare(wl, c, q, theta, scale, segs, units, O_gpu, lse_gpu, zmask)
    print(f"e2e {name}: max|dO|={err:.2e} max|dlse|={lerr:.2e} zoomed={nz}")


def test_split_count_does_not_change_result():
    """split-K + log-sum-exp merge equals a single pass, up to the rounding of the
    bf16 probabilities fed to the tensor-core p.V product (2^-9 relative)"""
    wl = WORKLOADS["c2"].scaled(n=4096, L=1)
    H, K, V, segs, units, q, theta, scale = _setup(wl)
    c = _cache(wl)
    T.upload_oracle_cache(c, segs, units)
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    ref = None
    for ns in (1, 2, 3, 7, 0):
        O_gpu, lse_gpu = c.decode(q.cuda(), th, nsplit=ns)
        torch.cuda.synchronize()
        if ref is None:
            ref = (O_gpu.clone(), lse_gpu.clone())
        else:
            assert (O_gpu - ref[0]).abs().max().item() < 1e-3
            assert (lse_gpu - ref[1]).abs().max().item() < 2e-5


@pytest.mark.parametrize("name,over,phase", [("c2", dict(n=4096, L=2), "fused"),
                                             ("c1", dict(), "fused"),
                                             ("c3", dict(n=8192, L=2), "attend")])
def test_in_kernel_merge_equals_merge_kernel(name, over, phase):
    """with arrival counters the last CTA of each (b, l, kv head) merges the split-K
    partials; on the tensor-core path the result has the same bits as the separate
    merge kernel (arrive = NULL), for several split counts and for per-layer calls,
    and the counters are zero again after every call"""
    P = _lib()
    S = P.sekv
    wl = WORKLOADS[name].scaled(**over)
    H, K, V, segs, units, q, theta, scale = _setup(wl, quantile=0.9 if phase == "attend" else None)
    c = _cache(wl, home="device" if phase == "fused" else "host")
    T.upload_oracle_cache(c, segs, units)
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    qd = q.cuda()
    kw = {}
    if phase == "attend":
        zr = c.new_zmask()
        c.decode(qd, th, phase=S.SEKV_ROUTE, zmask=zr)
        fetch = P.ColdFetcher(c, arena_elems=c.region * wl.L)
        info = fetch.fetch(zr)
        torch.cuda.current_stream().wait_event(fetch.done)
        assert info["spans"] > 0
        kw = dict(phase=S.SEKV_ATTEND, slot=fetch.slot_dev, arena=fetch.arena)
    stream = torch.cuda.current_stream().cuda_stream
    refs = []
    for ns in (1, 3, 0):
        for lr in ((0, wl.L),) + tuple((l, l + 1) for l in range(wl.L)):
            outs = []
            for with_counters in (True, False):
                O_g, lse_g = c.new_outputs()
                O_g.fill_(float("nan"))
                zm = c.new_zmask() if phase == "fused" else zr      # ATTEND reads ROUTE's mask
                d = c.decode_desc(qd, th, O=O_g, lse=lse_g, zmask=zm, nsplit=ns, l0=lr[0], l1=lr[1], **kw)
                assert d.arrive
                if not with_counters:
                    d.arrive = None
                S.check(S.sekv_decode_attn(d, stream), "decode")
                torch.cuda.synchronize()
                outs.append((O_g[:, lr[0]:lr[1]].clone(), lse_g[:, lr[0]:lr[1]].clone(), zm))
            assert c.read_status() == 0
            assert int(c._arrive.abs().sum()) == 0
            if wl.dtype == "bf16":
                assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1]), (ns, lr)
            else:
                # the fp32 path hands zoomed spans to its warps in arrival order, so the
                # CTA's sum order (and the last bits) vary from call to call
                assert (outs[0][0] - outs[1][0]).abs().max().item() <= 1e-6, (ns, lr)
                assert (outs[0][1] - outs[1][1]).abs().max().item() <= 1e-6, (ns, lr)
            if lr == (0, wl.L):
                refs.append(outs[0])
    # every split count against the oracle (with a mask given, ATTEND deals the zoomed
    # token units of a unit over its splits, cutting spans between them)
    for O_r, lse_r, zm_r in refs:
        _compare(wl, c, q, theta, scale, segs, units, O_r, lse_r, zm_r)


def test_layer_range_calls_equal_one_call():
    """per-layer calls (l0 = l, l1 = l + 1, each with its own split plan) write the
    same masks and, up to split-K summation order, the same O / lse as one call
    over all layers"""
    wl = WORKLOADS["c2"].scaled(n=2048, L=3)
    H, K, V, segs, units, q, theta, scale = _setup(wl)
    c = _cache(wl)
    T.upload_oracle_cache(c, segs, units)
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    qd = q.cuda()
    zm_f = c.new_zmask()
    O_f, lse_f = c.decode(qd, th, zmask=zm_f)
    zm_p = c.new_zmask()
    O_p, lse_p = c.new_outputs()
    for l in range(wl.L):
        c.decode(qd, th, O=O_p, lse=lse_p, zmask=zm_p, l0=l, l1=l + 1)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    assert torch.equal(zm_p, zm_f)
    assert (O_p - O_f).abs().max().item() < 1e-3
    assert (lse_p - lse_f).abs().max().item() < 2e-5
    _compare(wl, c, q, theta, scale, segs, units, O_p, lse_p, zm_p)


@pytest.mark.parametrize("name,over", [("c2", dict(n=4096, L=3)), ("c4", dict(B=2, n=2048, L=2))])
def test_static_ready_calls_give_the_same_bits(name, over):
    """with static_ready the kernels read the counts and their first anchor / summary
    tiles before the programmatic-launch wait; once the cache is settled (stream
    synchronised after the upload) back-to-back calls give the same bits as without:
    FUSED per layer and over all layers (device bases), ROUTE per layer, then fetch
    and ATTEND per layer with the routed mask (bases in host memory)"""
    P = _lib()
    S = P.sekv
    wl = WORKLOADS[name].scaled(**over)
    H, K, V, segs, units, q, theta, scale = _setup(wl)
    hot = _cache(wl)
    T.upload_oracle_cache(hot, segs, units)
    cold = _cache(wl, home="host")
    T.upload_oracle_cache(cold, segs, units)
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    qd = q.cuda()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    runs = {}
    for ready in (False, True):
        zm_f = hot.new_zmask()
        O_f, lse_f = hot.new_outputs()
        O_f.fill_(float("nan"))
        # calls enqueued back to back: each one's early reads overlap the previous kernel
        for l in range(wl.L):
            d = hot.decode_desc(qd, th, phase=S.SEKV_FUSED, O=O_f, lse=lse_f, zmask=zm_f, l0=l, l1=l + 1,
                                static_ready=ready)
            S.check(S.sekv_decode_attn(d, stream), "fused")
        O_1, lse_1 = hot.new_outputs()
        zm_1 = hot.new_zmask()
        d = hot.decode_desc(qd, th, phase=S.SEKV_FUSED, O=O_1, lse=lse_1, zmask=zm_1, static_ready=ready)
        S.check(S.sekv_decode_attn(d, stream), "fused, all layers")
        zm_r = cold.new_zmask()
        for l in range(wl.L):
            d = cold.decode_desc(qd, th, phase=S.SEKV_ROUTE, zmask=zm_r, l0=l, l1=l + 1, static_ready=ready)
            S.check(S.sekv_decode_attn(d, stream), "route")
        fetch = P.ColdFetcher(cold, arena_elems=cold.region * wl.L)
        fetch.fetch(zm_r)
        torch.cuda.current_stream().wait_event(fetch.done)
        O_a, lse_a = cold.new_outputs()
        O_a.fill_(float("nan"))
        for l in range(wl.L):
            d = cold.decode_desc(qd, th, phase=S.SEKV_ATTEND, O=O_a, lse=lse_a, zmask=zm_r, slot=fetch.slot_dev,
                                 arena=fetch.arena, l0=l, l1=l + 1, static_ready=ready)
            S.check(S.sekv_decode_attn(d, stream), "attend")
        torch.cuda.synchronize()
        assert hot.read_status() == 0 and cold.read_status() == 0
        runs[ready] = (zm_f, O_f, lse_f, zm_1, O_1, lse_1, zm_r, O_a, lse_a)
    for a, b in zip(runs[False], runs[True]):
        assert torch.equal(a, b)
    zm_f, O_f, lse_f, zm_1, O_1, lse_1, zm_r, O_a, lse_a = runs[True]
    assert torch.equal(zm_r, zm_f) and torch.equal(zm_1, zm_f)
    _compare(wl, hot, q, theta, scale, segs, units, O_f, lse_f, zm_f)
    _compare(wl, hot, q, theta, scale, segs, units, O_1, lse_1, zm_1)
    _compare(wl, cold, q, theta, scale, segs, units, O_a, lse_a, zm_r)


def test_route_fetch_attend_equals_fused():
    """cold bases in pinned host memory: ROUTE, fetch zoomed bases, ATTEND"""
    P = _lib()
    wl = WORKLOADS["c3"].scaled(n=8192, L=2)
    H, K, V, segs, units, q, theta, scale = _setup(wl, quantile=0.9)
    hot = _cache(wl)
    T.upload_oracle_cache(hot, segs, units)
    cold = _cache(wl, home="host")
    T.upload_oracle_cache(cold, segs, units)
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    qd = q.cuda()
    zm_f = hot.new_zmask()
    O_f, lse_f = hot.decode(qd, th, zmask=zm_f)
    fetch = P.ColdFetcher(cold, arena_elems=cold.region * wl.L)
    for step in range(2):                                   # the arena is reused across steps
        zm = cold.new_zmask()
        cold.decode(qd, th, phase=P.SEKV_ROUTE, zmask=zm)
        info = fetch.fetch(zm)
        torch.cuda.current_stream().wait_event(fetch.done)
        O_a, lse_a = cold.decode(qd, th, phase=P.SEKV_ATTEND, slot=fetch.slot_dev, arena=fetch.arena)
        torch.cuda.synchronize()
        assert cold.read_status() == 0
        assert torch.equal(zm, zm_f)
        assert info["spans"] > 0 and info["bytes"] > 0
        assert (O_a - O_f).abs().max().item() <= 1e-6
        assert (lse_a - lse_f).abs().max().item() <= 1e-6
    _compare(wl, hot, q, theta, scale, segs, units, O_f, lse_f, zm_f)


def test_attend_without_fetch_reports_cold_span():
    P = _lib()
    wl = WORKLOADS["c2"].scaled(n=4096, L=1)
    H, K, V, segs, units, q, theta, scale = _setup(wl, quantile=0.5)
    c = _cache(wl, home="host")
    T.upload_oracle_cache(c, segs, units)
    slot = torch.full((wl.B, wl.L, c.m_cap), -1, dtype=torch.int64, device="cuda")
    arena = torch.zeros(1024, dtype=c.dt, device="cuda")
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    c.decode(q.cuda(), th, phase=P.SEKV_ATTEND, slot=slot, arena=arena)
    torch.cuda.synchronize()
    assert c.read_status() == P.sekv.SEKV_ERR_COLD_SPAN


def test_fetch_capacity_error_copies_nothing():
    P = _lib()
    wl = WORKLOADS["c2"].scaled(n=4096, L=1)
    H, K, V, segs, units, q, theta, scale = _setup(wl, quantile=0.5)
    c = _cache(wl, home="host")
    T.upload_oracle_cache(c, segs, units)
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    zm = c.new_zmask()
    c.decode(q.cuda(), th, phase=P.SEKV_ROUTE, zmask=zm)
    fetch = P.ColdFetcher(c, arena_elems=64)
    with pytest.raises(P.SekvError) as ei:
        fetch.fetch(zm)
    assert ei.value.status == P.sekv.SEKV_ERR_CAPACITY
    assert (fetch.slot_dev == -1).all()


def _dense_unit_check(wl, c, q, K, V, scale, tol):
    O_gpu, lse_gpu = c.last
    for b in range(wl.B):
        for l in range(wl.L):
            for h in range(wl.Hq):
                o, ls = dense_attention(T.f64(q[b, l, h]), T.f64(K[b, l, h // wl.G]), T.f64(V[b, l, h // wl.G]), scale)
                assert np.abs(T.f64(O_gpu[b, l, h]) - o).max() <= tol
                assert abs(float(lse_gpu[b, l, h]) - ls) <= tol


def test_singleton_spans_give_dense_attention():
    """caller-supplied segmentation: every non-anchor token its own span"""
    P = _lib()
    wl = WORKLOADS["c1"].scaled(n=300)
    H, K, V = T.make_inputs(wl)
    c = _cache(wl, a_cap=320, m_cap=320)
    rng = np.random.default_rng(0)
    anchor = rng.random(wl.n) < 0.3
    ap = np.flatnonzero(anchor)
    sp = np.flatnonzero(~anchor)
    c.a_count[0] = len(ap)
    c.m_count[0] = len(sp)
    c.anchor_pos[0, :len(ap)] = torch.tensor(ap, dtype=torch.int32)
    c.span_beg[0, :len(sp)] = torch.tensor(sp, dtype=torch.int32)
    c.span_end[0, :len(sp)] = torch.tensor(sp + 1, dtype=torch.int32)
    c.build(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode,
            steps=P.SEKV_BUILD_LAYOUT | P.SEKV_BUILD_SUMMARY | P.SEKV_BUILD_BASES)
    q = gen.queries(wl)
    scale = 1.0 / math.sqrt(wl.d)
    for theta in (math.inf, -math.inf):         # nothing zoomed / everything zoomed
        th = torch.full((wl.L, wl.Hq), theta, dtype=torch.float32, device="cuda")
        c.last = c.decode(q.cuda(), th)
        torch.cuda.synchronize()
        assert c.read_status() == 0
        _dense_unit_check(wl, c, q, K, V, scale, 1e-4)


def test_all_zoom_full_rank_gives_dense_attention():
    wl = WORKLOADS["c1"].scaled(n=700, rank=64)                 # r = d: exact bases
    H, K, V = T.make_inputs(wl)
    c = _cache(wl)
    c.build(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode, max_sweeps=40)
    q = gen.queries(wl)
    th = torch.full((wl.L, wl.Hq), -math.inf, dtype=torch.float32, device="cuda")
    c.last = c.decode(q.cuda(), th)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    _dense_unit_check(wl, c, q, K, V, 1.0 / math.sqrt(wl.d), 1e-4)


def test_all_zoom_full_rank_bf16_gives_dense_attention():
    """bf16, r = d = 64, every span zoomed: K_S = A B and V_S = C D hold up to the
    bf16 rounding of the stored factors (relative 2^-9 per factor), which moves
    logits by ~1e-3 here, inside the bf16 tolerance."""
    wl = WORKLOADS["c2"].scaled(n=1200, L=1, d=64, Hq=4, Hkv=2, rank=64)
    H, K, V = T.make_inputs(wl)
    c = _cache(wl)
    c.build(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode, max_sweeps=40)
    q = gen.queries(wl)
    th = torch.full((wl.L, wl.Hq), -math.inf, dtype=torch.float32, device="cuda")
    c.last = c.decode(q.cuda(), th)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    _dense_unit_check(wl, c, q, K, V, 1.0 / math.sqrt(wl.d), 2e-2)


def test_empty_cache_rows():
    """a sequence with no spans and one with no anchors"""
    P = _lib()
    wl = WORKLOADS["c1"].scaled(n=64, B=2, window=0)
    H = torch.ones(2, 64)
    H[1, 5] = 50.0
    K = torch.randn(2, 1, wl.Hkv, 64, wl.d)
    V = torch.randn_like(K)
    c = _cache(wl)
    c.build(H.cuda(), K.cuda(), V.cuda(), 1.0, 64, "uniform")   # window covers all: no spans
    q = gen.queries(wl)
    th = torch.zeros(wl.L, wl.Hq, device="cuda")
    O1, l1 = c.decode(q.cuda(), th)
    torch.cuda.synchronize()
    assert int(c.m_count[0]) == 0 and int(c.a_count[0]) == 64
    c.last = (O1, l1)
    _dense_unit_check(wl, c, q, K, V, 1.0 / math.sqrt(wl.d), 1e-4)
    c2 = _cache(wl)
    c2.build(H.cuda(), K.cuda(), V.cuda(), 100.0, 0, "uniform")  # no boundary: one span, no anchors
    th = torch.full((wl.L, wl.Hq), math.inf, device="cuda")
    O2, l2 = c2.decode(q.cuda(), th)
    torch.cuda.synchronize()
    assert int(c2.a_count[0]) == 0 and int(c2.m_count[0]) == 1
    for h in range(wl.Hq):
        kb = T.f64(K[0, 0, h // wl.G]).mean(0)
        vb = T.f64(V[0, 0, h // wl.G]).mean(0)
        np.testing.assert_allclose(T.f64(O2[0, 0, h]), vb, atol=1e-5)   # one entry: softmax weight 1
        lo = float(T.f64(q[0, 0, h]) @ kb / math.sqrt(wl.d) + math.log(64))
        assert float(l2[0, 0, h]) == pytest.approx(lo, abs=1e-4)


def test_whole_span_variant_matches_oracle():
    """zoom_hint >= 64 selects the decode variant that hands small zoomed spans whole
    to one warp (taken per CTA when it holds >= 64 zoomed spans). Every span zoomed,
    one split, ~240 spans per CTA: both variants must match the oracle."""
    wl = WORKLOADS["c2"].scaled(n=16384, L=1, Hq=8, Hkv=2)
    H, K, V, segs, units, q, _, scale = _setup(wl)
    theta = np.full((wl.L, wl.Hq), -np.inf)
    c = _cache(wl)
    T.upload_oracle_cache(c, segs, units)
    th = torch.full((wl.L, wl.Hq), -math.inf, dtype=torch.float32, device="cuda")
    assert min(len(s.spans) for s in segs) >= 64
    outs = []
    for hint in (0, 10 ** 6):
        zmask = c.new_zmask()
        O_gpu, lse_gpu = c.decode(q.cuda(), th, zmask=zmask, nsplit=1, zoom_hint=hint)
        torch.cuda.synchronize()
        assert c.read_status() == 0
        err, lerr, nz = _compare(wl, c, q, theta, scale, segs, units, O_gpu, lse_gpu, zmask)
        outs.append(O_gpu)
        print(f"zoom_hint={hint}: max|dO|={err:.2e} max|dlse|={lerr:.2e} zoomed={nz}")
    assert (outs[0] - outs[1]).abs().max().item() <= 2e-2
