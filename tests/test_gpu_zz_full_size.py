"""Full-size parity in the benchmark's launch configuration.

The default benchmark workload (one 128K-token sequence, 32 layers, 32 query / 8
kv heads, d = 128, bf16, rank 16, bases in pinned host memory) is built by the
library and decoded as the benchmark does it: ROUTE, fetch of the zoomed bases,
ATTEND with the automatic split plan and the zoom hint. The oracle cannot redo the
whole step, so it builds and decodes three sampled (layer, kv head) units from
the same device-generated inputs; for those units the zoom masks must be
bit-exact (their heads' thresholds sit >= DELTA_L from every routing logit) and
O / lse within the bf16 tolerance of the end-to-end tests.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from sekv_synth import WORKLOADS, gen
from tests import helpers as T

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SAMPLED = [(0, 0), (13, 5), (31, 7)]      # (layer, kv head)


def test_full_size_cold_step_on_sampled_units():
    import bench
    import hierarchical_kv_cache_span_b200 as P
    wl = WORKLOADS["c3"]
    dev = torch.device("cuda")
    G = wl.Hq // wl.Hkv
    scale = 1.0 / math.sqrt(wl.d)
    H, spikes = gen.surprisal(wl, device=dev)
    K, V = gen.keys_values(wl, spikes, device=dev)
    a_cap, m_cap = bench.caps_for(wl)
    c = P.SpanCache(wl.B, wl.L, wl.Hq, wl.Hkv, wl.n, wl.d, wl.dtype, a_cap, m_cap, wl.rank, home=None,
                    device=dev)
    c.build(H, None, None, wl.alpha, wl.window, wl.wmode, steps=P.SEKV_BUILD_SCAN | P.SEKV_BUILD_LAYOUT)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    c.alloc_home("host", c.exact_region())
    c.build(H, K, V, wl.alpha, wl.window, wl.wmode, steps=P.SEKV_BUILD_SUMMARY | P.SEKV_BUILD_BASES)
    torch.cuda.synchronize()
    assert c.read_status() == 0, P.sekv.sekv_status_str(c.read_status())

    # the oracle's own build of the sampled units, from the same inputs
    Hn = T.f64(H[0])
    seg = O.segment(Hn, wl.alpha, wl.window)
    assert T.h_margin_ok(Hn, seg)
    assert int(c.a_count[0]) == len(seg.anchor_pos) and int(c.m_count[0]) == len(seg.spans)
    units = {(0, l, kvh): O.build_unit(T.f64(K[0, l, kvh]), T.f64(V[0, l, kvh]), Hn, seg, wl.wmode, wl.rank,
                                       wl.dtype)
             for (l, kvh) in SAMPLED}
    del K, V, spikes
    torch.cuda.empty_cache()

    q = gen.queries(wl, step=0, device=dev)
    qn = T.f64(q)
    # thresholds: the benchmark's calibration; the sampled heads' thresholds are
    # moved into a gap of the oracle's logits near the same quantile
    theta = bench.calibrate_theta(c, gen.queries(wl, step=10 ** 6, device=dev), wl.tau_a, P, torch)
    theta = theta.double().cpu().numpy()
    for (b, l, kvh), u in units.items():
        for g in range(G):
            ell = T.unit_route(qn[b, l, kvh * G + g], u, g, scale)
            for qt in (wl.tau_a, wl.tau_a - 0.005, wl.tau_a + 0.005, wl.tau_a - 0.01, wl.tau_a + 0.01):
                th = T.calibrate_theta(ell, qt)
                if T.margin(ell, th) > T.DELTA_L:
                    break
            assert T.margin(ell, th) > T.DELTA_L
            theta[l, kvh * G + g] = th
    th_d = torch.tensor(theta, dtype=torch.float32, device=dev)

    # the benchmark's cold step: zoom hint from a routing pass with another query,
    # then ROUTE -> fetch -> ATTEND
    zm = c.new_zmask()
    c.decode(gen.queries(wl, step=10 ** 6 + 1, device=dev), th_d, phase=P.SEKV_ROUTE, zmask=zm)
    zw = zm.cpu().numpy().view(np.uint32).reshape(wl.B, wl.L, wl.Hkv, G, -1)
    zoom_hint = int(np.unpackbits(np.bitwise_or.reduce(zw, axis=3).view(np.uint8), axis=-1).sum()
                    // (wl.B * wl.L * wl.Hkv))
    zm.zero_()
    c.decode(q, th_d, phase=P.SEKV_ROUTE, zmask=zm)
    fetch = P.ColdFetcher(c, arena_elems=c.region * wl.L)
    info = fetch.fetch(zm)
    torch.cuda.current_stream().wait_event(fetch.done)
    O_g, lse_g = c.decode(q, th_d, phase=P.SEKV_ATTEND, slot=fetch.slot_dev, arena=fetch.arena,
                          zoom_hint=zoom_hint)
    torch.cuda.synchronize()
    assert c.read_status() == 0, P.sekv.sekv_status_str(c.read_status())
    assert info["spans"] > 0

    m = len(seg.spans)
    zoomed = 0
    for (b, l, kvh), u in units.items():
        qg = qn[b, l, kvh * G:(kvh + 1) * G]
        z = np.stack([O.zoom_decisions(T.unit_route(qg[g], u, g, scale), theta[l, kvh * G + g])
                      for g in range(G)])
        for g in range(G):
            np.testing.assert_array_equal(T.zmask_bits(zm, b, l, kvh * G + g, m), z[g], err_msg=str((l, kvh, g)))
        zoomed += int(z.sum())
        o, ls = O.decode_unit(qg, u.Ka, u.Va, u.kbar, u.vbar, u.logS, z, u.bases, scale)
        err = np.abs(T.f64(O_g[b, l, kvh * G:(kvh + 1) * G]) - o).max()
        lerr = np.abs(T.f64(lse_g[b, l, kvh * G:(kvh + 1) * G]) - ls).max()
        assert err <= 2e-2, (l, kvh, err)
        assert lerr <= 2e-2, (l, kvh, lerr)
    assert zoomed > 0
