"""Zoom budget cap (SeKV blog 2.3, the paragraph under Eq. (9)): when more spans
pass a head's threshold than the budget allows, the spans are kept in descending
alpha~ order (the routing logit), equal logits lower span index first.

Parity against the oracle uses a budget at which every capped head's k-th and
(k+1)-th passing logits are at least DELTA_L apart, so the fp32 kernel and the
fp64 oracle select the same spans; masks must then be bit-exact. The selection
itself is checked exactly against the kernel's own fp32 logits, ties included.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from sekv_synth import WORKLOADS, gen
from tests import helpers as T

pytestmark = pytest.mark.gpu


def _lib():
    import hierarchical_kv_cache_span_b200 as P
    return P


def _cache(wl, home="device", a_cap=None, m_cap=None):
    P = _lib()
    ac, mc = T.caps(wl)
    return P.SpanCache(wl.B, wl.L, wl.Hq, wl.Hkv, wl.n, wl.d, wl.dtype, a_cap or ac, m_cap or mc,
                       wl.rank, home=home)


def _setup_budget(wl, quantile):
    H, K, V = T.make_inputs(wl)
    segs = T.oracle_segments(H, wl)
    units = T.oracle_units(K, V, H, segs, wl)
    scale = 1.0 / math.sqrt(wl.d)
    for attempt in range(8):
        q = gen.queries(wl, step=attempt)
        theta, q = T.thetas_with_margin(q, units, segs, wl, scale, wl.G, quantile=quantile)
        k = T.budget_with_margin(q, units, segs, theta, scale, wl.G)
        if k is not None:
            return segs, units, q, theta, scale, k
    pytest.fail("no budget with a DELTA_L margin for any of the queries tried")


def _check(wl, q, theta, scale, segs, units, k, O_gpu, lse_gpu, zm):
    Oo, lseo, zooms = T.oracle_decode(q, units, segs, theta, scale, wl.G, budget=k)
    capped = 0
    for (b, l, h), z in zooms.items():
        np.testing.assert_array_equal(T.zmask_bits(zm, b, l, h, len(z)), z, err_msg=str((b, l, h)))
        capped += int(z.sum() == k)
    assert capped > 0
    tol = 1e-4 if wl.dtype == "f32" else 2e-2
    assert np.abs(T.f64(O_gpu) - Oo).max() <= tol
    assert np.abs(T.f64(lse_gpu) - lseo).max() <= tol


@pytest.mark.parametrize("name,over,quantile", [
    ("c2", dict(n=4096, L=1, Hq=8, Hkv=2), 0.6),
    ("c5", dict(n=2048, L=1, Hq=8, Hkv=2), 0.5),
    ("c1", dict(n=1500), 0.4),
])
def test_fused_budget_matches_oracle(name, over, quantile):
    wl = WORKLOADS[name].scaled(**over)
    segs, units, q, theta, scale, k = _setup_budget(wl, quantile)
    c = _cache(wl)
    T.upload_oracle_cache(c, segs, units)
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    zm = c.new_zmask()
    O_gpu, lse_gpu = c.decode(q.cuda(), th, zmask=zm, budget=k)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    _check(wl, q, theta, scale, segs, units, k, O_gpu, lse_gpu, zm)


def test_route_fetch_attend_with_budget_equals_fused():
    P = _lib()
    wl = WORKLOADS["c3"].scaled(n=8192, L=2)
    segs, units, q, theta, scale, k = _setup_budget(wl, 0.9)
    hot = _cache(wl)
    T.upload_oracle_cache(hot, segs, units)
    cold = _cache(wl, home="host")
    T.upload_oracle_cache(cold, segs, units)
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    qd = q.cuda()
    zm_f = hot.new_zmask()
    O_f, lse_f = hot.decode(qd, th, zmask=zm_f, budget=k)
    zm = cold.new_zmask()
    cold.decode(qd, th, phase=P.SEKV_ROUTE, zmask=zm, budget=k)
    fetch = P.ColdFetcher(cold, arena_elems=cold.region * wl.L)
    info = fetch.fetch(zm)
    torch.cuda.current_stream().wait_event(fetch.done)
    O_a, lse_a = cold.decode(qd, th, phase=P.SEKV_ATTEND, slot=fetch.slot_dev, arena=fetch.arena, zmask=zm,
                             budget=k)
    torch.cuda.synchronize()
    assert cold.read_status() == 0 and hot.read_status() == 0
    assert torch.equal(zm, zm_f)
    assert info["spans"] > 0
    assert (O_a - O_f).abs().max().item() <= 1e-6
    assert (lse_a - lse_f).abs().max().item() <= 1e-6
    _check(wl, q, theta, scale, segs, units, k, O_f, lse_f, zm_f)


@pytest.mark.parametrize("n", [300, 600])      # ~270 zoomed spans per head: direct ranking; ~540: radix select
def test_cap_selection_is_exact_on_the_kernel_logits_with_ties(n):
    """Singleton spans whose key rows come in identical pairs: equal logits in every
    head. With theta = -inf and a budget, each head must keep exactly `budget` spans,
    no dropped span may outrank a kept one, and of equal logits the lower index wins
    (checked on the kernel's own fp32 logits)."""
    P = _lib()
    wl = WORKLOADS["c2"].scaled(n=n, L=1, Hq=8, Hkv=2, rank=4)
    H, K, V = T.make_inputs(wl)
    rng = np.random.default_rng(1)
    anchor = np.zeros(wl.n, dtype=bool)
    anchor[rng.choice(wl.n, n // 10, replace=False)] = True
    sp = np.flatnonzero(~anchor)
    # duplicate key rows pairwise along the span order
    for i in range(0, len(sp) - 1, 2):
        K[:, :, :, sp[i + 1]] = K[:, :, :, sp[i]]
    ap = np.flatnonzero(anchor)
    c = _cache(wl, a_cap=64, m_cap=((len(sp) + 31) // 32) * 32)
    c.a_count[0], c.m_count[0] = len(ap), len(sp)
    c.anchor_pos[0, :len(ap)] = torch.tensor(ap, dtype=torch.int32)
    c.span_beg[0, :len(sp)] = torch.tensor(sp, dtype=torch.int32)
    c.span_end[0, :len(sp)] = torch.tensor(sp + 1, dtype=torch.int32)
    c.build(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode,
            steps=P.SEKV_BUILD_LAYOUT | P.SEKV_BUILD_SUMMARY | P.SEKV_BUILD_BASES)
    q = gen.queries(wl).cuda()
    th = torch.full((wl.L, wl.Hq), -math.inf, dtype=torch.float32, device="cuda")
    m = len(sp)
    for k in (1, 7, 64, m - 1):
        zm = c.new_zmask()
        logits = torch.full((wl.B, wl.L, wl.Hq, c.m_cap), float("nan"), device="cuda")
        O_, lse_ = c.new_outputs()
        c.decode(q, th, O=O_, lse=lse_, zmask=zm, route_logits=logits, budget=k)
        torch.cuda.synchronize()
        assert c.read_status() == 0
        for h in range(wl.Hq):
            lg = logits[0, 0, h, :m].double().cpu().numpy()
            keep = T.zmask_bits(zm, 0, 0, h, m)
            assert keep.sum() == k
            kept, dropped = np.flatnonzero(keep), np.flatnonzero(~keep)
            lo_kept = lg[kept].min()
            assert (lg[dropped] <= lo_kept).all()
            ties = dropped[lg[dropped] == lo_kept]
            assert (ties > kept[lg[kept] == lo_kept].max()).all()
        assert torch.isfinite(O_).all()


def test_budget_validation_errors():
    P = _lib()
    S = P.sekv
    wl = WORKLOADS["c2"].scaled(n=1024, L=1, Hq=8, Hkv=2)
    c = _cache(wl)
    q = torch.zeros(wl.B, wl.L, wl.Hq, wl.d, dtype=torch.bfloat16, device="cuda")
    th = torch.zeros(wl.L, wl.Hq, device="cuda")
    O_, lse_ = c.new_outputs()
    d = c.decode_desc(q, th, O=O_, lse=lse_, budget=3)       # no zmask
    assert S.sekv_decode_attn(d, 0) == S.SEKV_ERR_INVALID_ARG
    assert "zmask" in S.sekv_last_error()
    d = c.decode_desc(q, th, O=O_, lse=lse_, zmask=c.new_zmask())
    d.budget = -1
    assert S.sekv_decode_attn(d, 0) == S.SEKV_ERR_INVALID_ARG
