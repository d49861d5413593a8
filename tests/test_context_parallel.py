"""Context-parallel decode (one sequence split across ranks, parts merged by
log-sum-exp). Host pieces on the CPU: the cut plan never splits a span and the
shards partition the segmentation; over a world-size-2 gloo group, per-rank
oracle decodes of the shards, all-gathered and merged, equal the oracle decode
of the whole context. On one GPU: shards built and decoded by the library and
merged by sekv_merge_partials equal the unsharded decode."""
import math
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as tmp

import oracle as O
from sekv_synth import WORKLOADS, gen
from tests import helpers as T

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cp():
    from hierarchical_kv_cache_span_b200 import context_parallel as CP
    return CP


def _lse_merge(Os, ls):
    """textbook log-sum-exp merge of parts of one softmax"""
    Os, ls = np.asarray(Os), np.asarray(ls)
    M = ls.max(axis=0)
    w = np.exp(ls - M)
    return (w[..., None] * Os).sum(0) / w.sum(0)[..., None], M + np.log(w.sum(0))


def _slice_seg(seg, t0, t1):
    CP = _cp()
    a, sb, se = (x.numpy() for x in CP.shard_segmentation(seg.anchor_pos, seg.spans[:, 0], seg.spans[:, 1],
                                                          t0, t1))
    anchor = np.zeros(t1 - t0, dtype=bool)
    anchor[a] = True
    spans = np.stack([sb, se], axis=1) if len(sb) else np.zeros((0, 2), np.int64)
    return O.Segmentation(seg.mu, seg.sigma, seg.thr, anchor, a, spans)


@pytest.mark.parametrize("world", [2, 3, 5, 8])
def test_cuts_partition_without_splitting_spans(world):
    CP = _cp()
    for seed in range(6):
        wl = WORKLOADS["c1"].scaled(n=3000, seed=seed, window=(seed % 3) * 40)
        H, _ = gen.surprisal(wl)
        seg = O.segment(T.f64(H[0]), wl.alpha, wl.window)
        cuts = CP.shard_cuts(seg.anchor_pos, seg.spans[:, 0], wl.n, world)
        assert cuts[0] == 0 and cuts[-1] == wl.n and all(a <= b for a, b in zip(cuts, cuts[1:]))
        starts = set(seg.anchor_pos.tolist()) | set(seg.spans[:, 0].tolist())
        assert all(c in starts or c == wl.n for c in cuts[1:-1])
        for b, e in seg.spans:
            assert not any(b < c < e for c in cuts), "a span straddles a cut"
        # the shards partition anchors and spans exactly
        na = ns = 0
        for r in range(world):
            s = _slice_seg(seg, cuts[r], cuts[r + 1])
            na += len(s.anchor_pos)
            ns += len(s.spans)
            assert (s.spans[:, 1] <= cuts[r + 1] - cuts[r]).all() if len(s.spans) else True
        assert na == len(seg.anchor_pos) and ns == len(seg.spans)


def test_cuts_edge_cases():
    CP = _cp()
    # more ranks than places to cut: some shards are empty, cuts stay monotone
    cuts = CP.shard_cuts([0, 1, 50], [2, 51], 60, 8)
    assert cuts[0] == 0 and cuts[-1] == 60 and all(a <= b for a, b in zip(cuts, cuts[1:]))
    assert set(cuts[1:-1]) <= {0, 1, 2, 50, 51, 60}
    for r in range(8):
        a, sb, se = CP.shard_segmentation([0, 1, 50], [2, 51], [50, 60], cuts[r], cuts[r + 1])
        assert (se <= cuts[r + 1] - cuts[r]).all()
    # every token an anchor (no spans): cuts fall on anchors
    cuts = CP.shard_cuts(list(range(10)), [], 10, 3)
    assert cuts == [0, 3, 6, 10]
    # one span and nothing else: a single cut point, the other shards empty
    cuts = CP.shard_cuts([], [0], 100, 4)
    assert cuts == [0, 100, 100, 100, 100]
    a, sb, se = CP.shard_segmentation([], [0], [100], 0, 100)
    assert len(a) == 0 and sb.tolist() == [0] and se.tolist() == [100]
    with pytest.raises(ValueError):
        CP.shard_segmentation([], [0], [100], 0, 50)      # a cut inside a span is refused


def test_shard_gate_slices_the_global_span_range():
    CP = _cp()
    wl = WORKLOADS["c1"].scaled(n=2000, seed=3)
    H, _ = gen.surprisal(wl)
    seg = O.segment(T.f64(H[0]), wl.alpha, wl.window)
    m = len(seg.spans)
    L, Hkv, r, m_cap = 2, 3, 4, ((m + 31) // 32) * 32
    g = torch.arange(L * Hkv * m * 2 * r, dtype=torch.float32).reshape(1, L, Hkv, m, 2, r)
    world = 3
    seen = 0
    for rank in range(world):
        sh = CP.ContextShard(L, 4, Hkv, wl.n, 64, "f32", 64, m_cap, r, rank=rank, world=world, device="cpu")
        sh._seg = (seg.anchor_pos, seg.spans[:, 0], seg.spans[:, 1])
        sh.cuts = CP.shard_cuts(seg.anchor_pos, seg.spans[:, 0], wl.n, world)
        k0, k1 = sh.span_range()
        t0, t1 = sh.cuts[rank], sh.cuts[rank + 1]
        inside = np.flatnonzero((seg.spans[:, 0] >= t0) & (seg.spans[:, 0] < t1))
        assert (k0, k1) == ((int(inside[0]), int(inside[-1]) + 1) if len(inside) else (k0, k0))
        sg = sh.shard_gate(g)
        assert sg.shape == (1, L, Hkv, m_cap, 2, r)
        assert torch.equal(sg[:, :, :, :k1 - k0], g[:, :, :, k0:k1])
        assert (sg[:, :, :, k1 - k0:] == 0).all()
        seen += k1 - k0
    assert seen == m


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    from hierarchical_kv_cache_span_b200 import context_parallel as CP
    wl = WORKLOADS["c1"].scaled(n=1500, Hq=4, Hkv=2)
    H, K, V = T.make_inputs(wl)
    seg = O.segment(T.f64(H[0]), wl.alpha, wl.window)
    cuts = CP.shard_cuts(seg.anchor_pos, seg.spans[:, 0], wl.n, world)
    t0, t1 = cuts[rank], cuts[rank + 1]
    s = _slice_seg(seg, t0, t1)
    q = T.f64(gen.queries(wl))
    scale = 1.0 / math.sqrt(wl.d)
    G = wl.Hq // wl.Hkv
    O_r = np.zeros((wl.L, wl.Hq, wl.d))
    lse_r = np.full((wl.L, wl.Hq), -np.inf)
    for l in range(wl.L):
        for kvh in range(wl.Hkv):
            u = O.build_unit(T.f64(K[0, l, kvh, t0:t1]), T.f64(V[0, l, kvh, t0:t1]), T.f64(H[0, t0:t1]), s,
                             wl.wmode, wl.rank, wl.dtype)
            qg = q[0, l, kvh * G:(kvh + 1) * G]
            z = np.stack([O.zoom_decisions(O.routing_logits(qg[g], u.kbar, u.inv_norm, u.logS, scale), 0.0)
                          for g in range(G)]) if len(s.spans) else np.zeros((G, 0), bool)
            o, ls = O.decode_unit(qg, u.Ka, u.Va, u.kbar, u.vbar, u.logS, z, u.bases, scale)
            O_r[l, kvh * G:(kvh + 1) * G] = o
            lse_r[l, kvh * G:(kvh + 1) * G] = ls
    Ot = torch.tensor(O_r)
    lt = torch.tensor(lse_r)
    Oall = [torch.empty_like(Ot) for _ in range(world)]
    lall = [torch.empty_like(lt) for _ in range(world)]
    dist.all_gather(Oall, Ot)
    dist.all_gather(lall, lt)
    Om, lm = _lse_merge([o.numpy() for o in Oall], [x.numpy() for x in lall])
    if rank == 0:
        # the whole context on one "rank"
        Of = np.zeros_like(O_r)
        lf = np.zeros_like(lse_r)
        for l in range(wl.L):
            for kvh in range(wl.Hkv):
                u = O.build_unit(T.f64(K[0, l, kvh]), T.f64(V[0, l, kvh]), T.f64(H[0]), seg, wl.wmode, wl.rank,
                                 wl.dtype)
                qg = q[0, l, kvh * G:(kvh + 1) * G]
                z = np.stack([O.zoom_decisions(O.routing_logits(qg[g], u.kbar, u.inv_norm, u.logS, scale), 0.0)
                              for g in range(G)])
                o, ls = O.decode_unit(qg, u.Ka, u.Va, u.kbar, u.vbar, u.logS, z, u.bases, scale)
                Of[l, kvh * G:(kvh + 1) * G] = o
                lf[l, kvh * G:(kvh + 1) * G] = ls
        out.put((float(np.abs(Om - Of).max()), float(np.abs(lm - lf).max()), cuts))
    dist.barrier()
    dist.destroy_process_group()


def test_sharded_oracle_decodes_merge_to_the_whole_over_gloo():
    world, port = 2, 29541
    ctx = tmp.get_context("spawn")
    qq = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, qq)) for r in range(world)]
    for p in procs:
        p.start()
    dO, dl, cuts = qq.get(timeout=600)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert 0 < cuts[1] < cuts[2]
    assert dO <= 1e-12 and dl <= 1e-12


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 3])
def test_library_shards_merge_to_the_unsharded_decode(world):
    import hierarchical_kv_cache_span_b200 as P
    CP = _cp()
    wl = WORKLOADS["c2"].scaled(n=6000, L=2, Hq=8, Hkv=2)
    H, K, V = T.make_inputs(wl)
    ac, mc = T.caps(wl)
    Hd, Kd, Vd = H.cuda(), K.cuda(), V.cuda()
    full = P.SpanCache(1, wl.L, wl.Hq, wl.Hkv, wl.n, wl.d, wl.dtype, ac, mc, wl.rank)
    full.build(Hd, Kd, Vd, wl.alpha, wl.window, wl.wmode)
    q = gen.queries(wl).cuda()
    theta = torch.full((wl.L, wl.Hq), 3.5, dtype=torch.float32, device="cuda")   # a few % of spans zoom
    zm = full.new_zmask()
    O_f, lse_f = full.decode(q, theta, zmask=zm)
    parts_O, parts_l = [], []
    cuts = None
    for r in range(world):
        sh = CP.ContextShard(wl.L, wl.Hq, wl.Hkv, wl.n, wl.d, wl.dtype, ac, mc, wl.rank, rank=r, world=world)
        cuts = sh.plan(Hd, wl.alpha, wl.window)
        t0, t1 = cuts[r], cuts[r + 1]
        sh.build(Hd, Kd[:, :, :, t0:t1].contiguous(), Vd[:, :, :, t0:t1].contiguous(), wl.alpha, wl.window,
                 wl.wmode)
        o, l = sh.decode(q, theta)
        assert sh.cache.read_status() == 0
        parts_O.append(o)
        parts_l.append(l)
    O_m, lse_m = CP.merge_parts(torch.stack(parts_O), torch.stack(parts_l))
    torch.cuda.synchronize()
    assert full.read_status() == 0
    assert int(zm.ne(0).sum()) > 0
    # same entries, same factors (the bases of a span do not depend on the shard);
    # only the split-K / merge summation order differs
    assert (O_m - O_f).abs().max().item() <= 2e-3
    assert (lse_m - lse_f).abs().max().item() <= 2e-3


@pytest.mark.gpu
def test_learned_routing_shards_merge_to_the_unsharded_decode():
    """learned-form routing and a rank gate, split over 2 shards"""
    import hierarchical_kv_cache_span_b200 as P
    CP = _cp()
    wl = WORKLOADS["c2"].scaled(n=4000, L=2, Hq=8, Hkv=2)
    H, K, V = T.make_inputs(wl)
    ac, mc = T.caps(wl)
    W = gen.route_projection(wl, 32).cuda()
    gates = gen.rank_gates(wl, mc).cuda()
    Hd, Kd, Vd = H.cuda(), K.cuda(), V.cuda()
    full = P.SpanCache(1, wl.L, wl.Hq, wl.Hkv, wl.n, wl.d, wl.dtype, ac, mc, wl.rank)
    full.set_routing(W)
    full.build(Hd, Kd, Vd, wl.alpha, wl.window, wl.wmode, rank_gate=gates)
    q = gen.queries(wl).cuda()
    theta = torch.full((wl.L, wl.Hq), 2.0, dtype=torch.float32, device="cuda")
    zm = full.new_zmask()
    O_f, lse_f = full.decode(q, theta, zmask=zm)
    parts_O, parts_l = [], []
    for r in range(2):
        sh = CP.ContextShard(wl.L, wl.Hq, wl.Hkv, wl.n, wl.d, wl.dtype, ac, mc, wl.rank, rank=r, world=2,
                             route_W=W)
        cuts = sh.plan(Hd, wl.alpha, wl.window)
        t0, t1 = cuts[r], cuts[r + 1]
        sh.build(Hd, Kd[:, :, :, t0:t1].contiguous(), Vd[:, :, :, t0:t1].contiguous(), wl.alpha, wl.window,
                 wl.wmode, rank_gate=gates)
        o, l = sh.decode(q, theta)
        assert sh.cache.read_status() == 0
        parts_O.append(o)
        parts_l.append(l)
    O_m, lse_m = CP.merge_parts(torch.stack(parts_O), torch.stack(parts_l))
    torch.cuda.synchronize()
    assert full.read_status() == 0
    assert int(zm.ne(0).sum()) > 0
    assert (O_m - O_f).abs().max().item() <= 2e-3
    assert (lse_m - lse_f).abs().max().item() <= 2e-3


@pytest.mark.gpu
def test_merge_partials_edge_cases():
    CP = _cp()
    rows, d = 5, 64
    Op = torch.randn(3, rows, d, device="cuda")
    lp = torch.randn(3, rows, device="cuda")
    lp[1, 0] = -math.inf                      # a part with no entries for row 0
    lp[:, 4] = -math.inf                      # no part has entries for row 4
    Om, lm = CP.merge_parts(Op, lp)
    torch.cuda.synchronize()
    Oo, lo = _lse_merge(Op[:, :4].double().cpu().numpy(), lp[:, :4].double().cpu().numpy())
    assert np.abs(Om[:4].double().cpu().numpy() - Oo).max() <= 1e-5
    assert np.abs(lm[:4].double().cpu().numpy() - lo).max() <= 1e-5
    assert (Om[4] == 0).all() and lm[4].item() == -math.inf


# ---------------------------------------------------------------------------
# The exchange path itself: two processes on the one GPU, a gloo group, and
# context_parallel_decode (library decode of each shard, all-gather, library
# merge) against the oracle over the whole context. The two ranks' kernels never
# wait on each other: the exchange is a host-side collective between launches.
# ---------------------------------------------------------------------------
def _cp_case():
    wl = WORKLOADS["c2"].scaled(n=4096, L=2, Hq=8, Hkv=2)
    return wl


def _cp_gpu_rank(rank, world, port, theta, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from hierarchical_kv_cache_span_b200 import context_parallel as CP
        torch.cuda.set_device(0)
        wl = _cp_case()
        H, K, V = (x.cuda() for x in T.make_inputs(wl))      # the parent's inputs (CPU draws)
        ac, mc = T.caps(wl)
        sh = CP.ContextShard(wl.L, wl.Hq, wl.Hkv, wl.n, wl.d, wl.dtype, ac, mc, wl.rank, rank=rank, world=world)
        cuts = sh.plan(H, wl.alpha, wl.window)
        t0, t1 = cuts[rank], cuts[rank + 1]
        sh.build(H, K[:, :, :, t0:t1].contiguous(), V[:, :, :, t0:t1].contiguous(), wl.alpha, wl.window, wl.wmode)
        q = gen.queries(wl).cuda()
        th = torch.tensor(theta, dtype=torch.float32, device="cuda")
        zm = sh.cache.new_zmask()
        O_m, lse_m = CP.context_parallel_decode(sh, q, th, zmask=zm)
        torch.cuda.synchronize()
        st = sh.cache.read_status()
        k0, k1 = sh.span_range()
        out.put((rank, st, cuts, k0, k1, O_m.double().cpu().numpy(), lse_m.double().cpu().numpy(),
                 zm.cpu().numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_context_parallel_decode_over_gloo_matches_the_oracle():
    wl = _cp_case()
    scale = 1.0 / math.sqrt(wl.d)
    G = wl.Hq // wl.Hkv
    H, K, V = T.make_inputs(wl)
    segs = T.oracle_segments(H, wl)
    units = T.oracle_units(K, V, H, segs, wl)
    q = gen.queries(wl)
    # thresholds in gaps of the oracle's routing logits (~10 % zoom); q stays as drawn
    theta = np.zeros((wl.L, wl.Hq))
    qn = T.f64(q)
    for (b, l, kvh), u in units.items():
        for g in range(G):
            ell = T.unit_route(qn[b, l, kvh * G + g], u, g, scale)
            th = T.calibrate_theta(ell, 0.9)
            assert T.margin(ell, th) > T.DELTA_L
            theta[l, kvh * G + g] = th
    Oo, lo, zooms = T.oracle_decode(q, units, segs, theta, scale, G)

    world, port = 2, 29547
    ctx = tmp.get_context("spawn")
    qq = ctx.Queue()
    procs = [ctx.Process(target=_cp_gpu_rank, args=(r, world, port, theta, qq)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([qq.get(timeout=900) for _ in range(world)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    m = len(segs[0].spans)
    zoomed = 0
    for rank, st, cuts, k0, k1, O_m, lse_m, zm in res:
        assert st == 0
        assert 0 < cuts[1] < cuts[2]
        # every rank returns the merged whole-context result
        assert np.abs(O_m[0] - Oo[0]).max() <= 2e-2
        assert np.abs(lse_m[0] - lo[0]).max() <= 2e-2
        # this rank's zoom bits are the oracle's for its run of global spans
        for l in range(wl.L):
            for h in range(wl.Hq):
                w = zm[0, l, h].astype(np.uint32)
                bits = ((w[:, None] >> np.arange(32, dtype=np.uint32)[None, :]) & 1).reshape(-1).astype(bool)
                np.testing.assert_array_equal(bits[:k1 - k0], zooms[(0, l, h)][k0:k1])
                zoomed += int(bits[:k1 - k0].sum())
    assert sum(r[4] - r[3] for r in res) == m
    assert zoomed > 0
    assert np.abs(res[0][5] - res[1][5]).max() == 0.0
