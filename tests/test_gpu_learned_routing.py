"""GPU parity of the learned-form routing and the rank gate against the fp64 oracle.

SeKV blog 2.2 Eq. (3): per (layer, query head) routing summaries in a d'-dimensional
space, y = sum_t w_t W K_t normalised; 2.3 Eq. (5): l_S = (W q) . Kbar_S / sqrt(d')
+ log|S|; 2.2 Eq. (6): the rank gate m_{S,i} scales component i of each span's
truncated SVD. W and the gates are seeded stand-ins for trained weights.

Summaries: within one storage ulp of the oracle (plus fp32 accumulation).
Decode: zoom masks bit-exact (routing logits kept DELTA_L away from theta), O / lse
within the decode tolerance; ROUTE + fetch + ATTEND equals FUSED; with a budget the
capped masks equal the oracle's. Gated bases: products within the basis tolerance.
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


def _tol(wl):
    return 1e-4 if wl.dtype == "f32" else 2e-2


def _cache(wl, W=None, home="device"):
    P = _lib()
    ac, mc = T.caps(wl)
    c = P.SpanCache(wl.B, wl.L, wl.Hq, wl.Hkv, wl.n, wl.d, wl.dtype, ac, mc, wl.rank, home=home)
    if W is not None:
        c.set_routing(W.cuda())
    return c


SUMMARY_CASES = [
    ("c1", dict(n=1500, Hq=8, Hkv=2), 32, "surprisal"),          # fp32, d = 64, G = 4
    ("c2", dict(n=4096, L=2), 32, "softmax"),                    # bf16, d = 128, G = 4
    ("c2", dict(n=3000, L=1, B=2, Hq=16, Hkv=2), 64, "uniform"),  # G = 8, dr = 64
    ("c2", dict(n=2048, L=1, d=64, Hq=8, Hkv=8), 32, "uniform"),  # G = 1, d = 64
]


@pytest.mark.parametrize("name,over,dr,wmode", SUMMARY_CASES)
def test_routing_summaries_parity(name, over, dr, wmode):
    P = _lib()
    wl = WORKLOADS[name].scaled(wmode=wmode, **over)
    H, K, V = T.make_inputs(wl)
    W = gen.route_projection(wl, dr)
    c = _cache(wl, W)
    c.build(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode,
            steps=P.SEKV_BUILD_SCAN | P.SEKV_BUILD_LAYOUT | P.SEKV_BUILD_SUMMARY)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    segs = T.oracle_segments(H, wl)
    G = wl.Hq // wl.Hkv
    worst = 0.0
    for b in range(wl.B):
        m = len(segs[b].spans)
        for l in range(wl.L):
            for kvh in range(wl.Hkv):
                want = O.routing_summaries(T.f64(K[b, l, kvh]), T.f64(H[b]), segs[b], wl.wmode,
                                           T.f64(W[l, kvh * G:(kvh + 1) * G]), wl.dtype)
                got = T.f64(c.kbar_r[b, l, kvh * G:(kvh + 1) * G, :m])
                # unit vectors: one storage ulp of each component plus fp32 rounding of
                # the mean, the d-term projection and the norm (a few 1e-6 absolute)
                ulp = np.abs(want) * (2.0 ** -7 if wl.dtype == "bf16" else 2.0 ** -22)
                err = np.abs(got - want) - ulp
                worst = max(worst, float(np.abs(got - want).max()))
                assert (err <= 2e-6).all(), float(err.max())
                norms = np.sqrt((got ** 2).sum(-1))
                assert np.all(np.abs(norms - 1.0) <= (1e-2 if wl.dtype == "bf16" else 1e-5))
    print(f"{name} dr={dr}: worst |d kbar_r| = {worst:.2e}")


def _setup(wl, dr, quantile, gates=False):
    H, K, V = T.make_inputs(wl)
    W = gen.route_projection(wl, dr)
    segs = T.oracle_segments(H, wl)
    ac, mc = T.caps(wl)
    gt = gen.rank_gates(wl, mc) if gates else None
    units = T.oracle_units(K, V, H, segs, wl, W=W, gates=gt)
    q = gen.queries(wl)
    scale = 1.0 / math.sqrt(wl.d)
    theta, q = T.thetas_with_margin(q, units, segs, wl, scale, wl.G, quantile=quantile)
    return H, K, V, W, gt, segs, units, q, theta, scale


def _compare(wl, q, theta, scale, segs, units, O_gpu, lse_gpu, zmask, budget=None):
    Oo, lseo, zooms = T.oracle_decode(q, units, segs, theta, scale, wl.G, budget=budget)
    for (b, l, h), z in zooms.items():
        np.testing.assert_array_equal(T.zmask_bits(zmask, b, l, h, len(z)), z, err_msg=str((b, l, h)))
    err = np.abs(T.f64(O_gpu) - Oo).max()
    lerr = np.abs(T.f64(lse_gpu) - lseo).max()
    assert err <= _tol(wl), err
    assert lerr <= _tol(wl), lerr
    return err, lerr, sum(int(z.sum()) for z in zooms.values())


DECODE_CASES = [
    ("c1", dict(Hq=4, Hkv=2), 32, 0.7),                      # fp32, d = 64
    ("c2", dict(n=4096, L=2), 32, 0.9),                      # bf16 Llama shape
    ("c5", dict(n=4096, L=1, Hq=8, Hkv=2), 64, 0.75),        # rank 32, dr = 64
    ("c2", dict(n=2048, L=1, B=2, Hq=16, Hkv=2), 32, 0.8),   # batch, G = 8
]


@pytest.mark.parametrize("name,over,dr,quantile", DECODE_CASES)
def test_learned_decode_kernel_level(name, over, dr, quantile):
    wl = WORKLOADS[name].scaled(**over)
    H, K, V, W, _, segs, units, q, theta, scale = _setup(wl, dr, quantile)
    c = _cache(wl, W)
    T.upload_oracle_cache(c, segs, units)
    zmask = c.new_zmask()
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    logits = torch.zeros(wl.B, wl.L, wl.Hq, c.m_cap, dtype=torch.float32, device="cuda")
    O_gpu, lse_gpu = c.decode(q.cuda(), th, zmask=zmask, route_logits=logits)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    err, lerr, nz = _compare(wl, q, theta, scale, segs, units, O_gpu, lse_gpu, zmask)
    assert nz > 0
    # the routing logits the pass wrote are the learned ones (fp32 vs fp64)
    qn = T.f64(q)
    for (b, l, kvh), u in units.items():
        for g in range(wl.G):
            h = kvh * wl.G + g
            m = len(segs[b].spans)
            want = T.unit_route(qn[b, l, h], u, g, scale)
            assert np.abs(T.f64(logits[b, l, h, :m]) - want).max() <= 2e-3
    print(f"learned {name} dr={dr}: max|dO|={err:.2e} max|dlse|={lerr:.2e} zoomed={nz}")


def test_learned_decode_end_to_end():
    """library build (scan, summaries incl. routing summaries, bases) + decode"""
    wl = WORKLOADS["c2"].scaled(n=4096, L=2)
    H, K, V, W, _, segs, units, q, theta, scale = _setup(wl, 32, 0.9)
    c = _cache(wl, W)
    c.build(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode)
    zmask = c.new_zmask()
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    O_gpu, lse_gpu = c.decode(q.cuda(), th, zmask=zmask)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    err, lerr, nz = _compare(wl, q, theta, scale, segs, units, O_gpu, lse_gpu, zmask)
    print(f"learned e2e: max|dO|={err:.2e} max|dlse|={lerr:.2e} zoomed={nz}")


def test_learned_route_fetch_attend_equals_fused():
    P = _lib()
    wl = WORKLOADS["c3"].scaled(n=8192, L=2)
    H, K, V, W, _, segs, units, q, theta, scale = _setup(wl, 32, 0.9)
    hot = _cache(wl, W)
    T.upload_oracle_cache(hot, segs, units)
    cold = _cache(wl, W, home="host")
    T.upload_oracle_cache(cold, segs, units)
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    qd = q.cuda()
    zm_f = hot.new_zmask()
    O_f, lse_f = hot.decode(qd, th, zmask=zm_f)
    zm = cold.new_zmask()
    cold.decode(qd, th, phase=P.SEKV_ROUTE, zmask=zm)
    fetch = P.ColdFetcher(cold, arena_elems=cold.region * wl.L)
    info = fetch.fetch(zm)
    torch.cuda.current_stream().wait_event(fetch.done)
    O_a, lse_a = cold.decode(qd, th, phase=P.SEKV_ATTEND, slot=fetch.slot_dev, arena=fetch.arena, zmask=zm)
    torch.cuda.synchronize()
    assert cold.read_status() == 0 and hot.read_status() == 0
    assert torch.equal(zm, zm_f)
    assert info["spans"] > 0
    assert (O_a - O_f).abs().max().item() <= 1e-6
    assert (lse_a - lse_f).abs().max().item() <= 1e-6
    _compare(wl, q, theta, scale, segs, units, O_f, lse_f, zm_f)


def test_learned_routing_with_budget():
    wl = WORKLOADS["c2"].scaled(n=4096, L=2)
    H, K, V, W, _, segs, units, q, theta, scale = _setup(wl, 32, 0.8)
    k = T.budget_with_margin(q, units, segs, theta, scale, wl.G)
    assert k is not None
    c = _cache(wl, W)
    T.upload_oracle_cache(c, segs, units)
    zm = c.new_zmask()
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    O_gpu, lse_gpu = c.decode(q.cuda(), th, zmask=zm, budget=k)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    _compare(wl, q, theta, scale, segs, units, O_gpu, lse_gpu, zm, budget=k)
    per_head = zm.view(torch.int32).cpu().numpy().astype(np.uint32)
    pop = np.unpackbits(per_head.view(np.uint8), axis=-1).reshape(wl.B, wl.L, wl.Hq, -1).sum(-1)
    assert pop.max() <= k


GATE_CASES = [
    ("c1", dict(n=1024)),                                      # fp32, d = 64, r = 4
    ("c2", dict(n=3000, L=1, Hq=8, Hkv=2)),                    # bf16, d = 128, r = 16
    ("c2", dict(n=2048, L=1, B=2, Hq=4, Hkv=1, alpha=2.5)),    # long spans: |S| > d path
]


@pytest.mark.parametrize("name,over", GATE_CASES)
def test_rank_gate_bases_parity(name, over):
    from tests.test_gpu_build import _read_block
    P = _lib()
    wl = WORKLOADS[name].scaled(**over)
    H, K, V = T.make_inputs(wl)
    c = _cache(wl)
    gates = gen.rank_gates(wl, c.m_cap)
    c.build(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode, max_sweeps=30,
            rank_gate=gates.cuda())
    torch.cuda.synchronize()
    assert c.read_status() == 0, P.sekv.sekv_status_str(c.read_status())
    segs = T.oracle_segments(H, wl)
    tol = 1e-4 if wl.dtype == "f32" else 1e-2
    n_long = 0
    for b in range(wl.B):
        for l in range(wl.L):
            for h in range(wl.Hkv):
                Kb, Vb = T.f64(K[b, l, h]), T.f64(V[b, l, h])
                for S, (beg, end) in enumerate(segs[b].spans):
                    A, Bm, Cm, Dm = _read_block(c, b, l, h, S, int(beg), int(end))
                    n_long += (end - beg) > wl.d
                    for which, (X, F1, F2) in enumerate(((Kb[beg:end], A, Bm), (Vb[beg:end], Cm, Dm))):
                        g = T.f64(gates[b, l, h, S, which])
                        Ao, Bo = O.truncated_basis(X, wl.rank, wl.dtype, gate=g)
                        ref = Ao @ Bo
                        # relative to the ungated reconstruction (a gate of 0 leaves nothing)
                        A1, B1 = O.truncated_basis(X, wl.rank, wl.dtype)
                        scale_ = max(np.linalg.norm(A1 @ B1), 1e-30)
                        err = np.linalg.norm(F1 @ F2 - ref) / scale_
                        assert err <= tol, (b, l, h, S, which, end - beg, err)
    print(f"gated bases ok; spans longer than d: {n_long}")


def test_rank_gate_decode_matches_oracle():
    wl = WORKLOADS["c2"].scaled(n=4096, L=1, Hq=8, Hkv=2)
    H, K, V, W, gates, segs, units, q, theta, scale = _setup(wl, 32, 0.8, gates=True)
    c = _cache(wl, W)
    c.build(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode, rank_gate=gates.cuda())
    zmask = c.new_zmask()
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    O_gpu, lse_gpu = c.decode(q.cuda(), th, zmask=zmask)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    err, lerr, nz = _compare(wl, q, theta, scale, segs, units, O_gpu, lse_gpu, zmask)
    assert nz > 0
    print(f"gated decode: max|dO|={err:.2e} max|dlse|={lerr:.2e} zoomed={nz}")


def test_learned_routing_argument_errors():
    P = _lib()
    S = P.sekv
    wl = WORKLOADS["c2"].scaled(n=2048, L=1)
    W = gen.route_projection(wl, 32)
    c = _cache(wl, W)
    q = gen.queries(wl).cuda()
    th = torch.zeros(wl.L, wl.Hq, dtype=torch.float32, device="cuda")
    d = c.decode_desc(q, th, O=torch.zeros(1, device="cuda"), lse=torch.zeros(1, device="cuda"))
    d.kbar_r = None
    assert S.sekv_decode_attn(d, None) == S.SEKV_ERR_INVALID_ARG
    d = c.decode_desc(q, th)
    d.dr = 48
    assert S.sekv_decode_attn(d, None) == S.SEKV_ERR_UNSUPPORTED
    d = c.decode_desc(q, th)
    d.zmask = None
    assert S.sekv_decode_attn(d, None) == S.SEKV_ERR_INVALID_ARG
    H, K, V = T.make_inputs(wl)
    bd = c.build_desc(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode)
    bd.dr = 16
    assert S.sekv_build_spans(bd, None) == S.SEKV_ERR_UNSUPPORTED
    bd = c.build_desc(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode)
    bd.kbar_r = None
    assert S.sekv_build_spans(bd, None) == S.SEKV_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert c.read_status() == 0
