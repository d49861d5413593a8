"""GPU parity of the prefill build against the fp64 oracle.

Boundary scan (SeKV blog 2.1): counts, anchor positions and span bounds bit-exact.
Summaries (SeKV blog 2.2, Eq. (2)): gathered anchors exact; kbar / vbar within one
storage ulp; 1/||kbar|| within fp32 rounding. Bases (Eq. (6)-(8)): products A B and
C D match the oracle's truncated SVD within 1e-4 (fp32) / 1e-2 (bf16) relative
Frobenius error, per span.
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


def _cache(wl, **kw):
    P = _lib()
    a_cap, m_cap = T.caps(wl)
    return P.SpanCache(wl.B, wl.L, wl.Hq, wl.Hkv, wl.n, wl.d, wl.dtype, kw.get("a_cap", a_cap),
                       kw.get("m_cap", m_cap), wl.rank, home=kw.get("home", "device"))


SCAN_CASES = [
    ("c1", dict()),
    ("c1", dict(n=2049, window=64)),                 # ragged n, window
    ("c2", dict(n=8192, B=2, L=1)),
    ("c4", dict(n=32768, B=3, L=1)),
    ("c3", dict(n=131072, L=1)),                     # full 128K sequence length
    ("c1", dict(n=1, window=0)),                     # single token
    ("c1", dict(n=37, window=100)),                  # window covers everything
]


@pytest.mark.parametrize("name,over", SCAN_CASES)
def test_scan_bit_exact(name, over):
    P = _lib()
    wl = WORKLOADS[name].scaled(**over)
    H, _ = gen.surprisal(wl)
    c = _cache(wl)
    c.build(H.cuda(), None, None, wl.alpha, wl.window, wl.wmode,
            steps=P.SEKV_BUILD_SCAN | P.SEKV_BUILD_LAYOUT)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    for b in range(wl.B):
        Hb = T.f64(H[b])
        seg = O.segment(Hb, wl.alpha, wl.window)
        assert T.h_margin_ok(Hb, seg) or wl.n < 4
        a, m = int(c.a_count[b]), int(c.m_count[b])
        assert a == len(seg.anchor_pos) and m == len(seg.spans)
        np.testing.assert_array_equal(c.anchor_pos[b, :a].cpu().numpy(), seg.anchor_pos)
        np.testing.assert_array_equal(c.span_beg[b, :m].cpu().numpy(), seg.spans[:, 0])
        np.testing.assert_array_equal(c.span_end[b, :m].cpu().numpy(), seg.spans[:, 1])
        st = c.stats[b].cpu().numpy()
        assert st[0] == pytest.approx(seg.mu, rel=1e-12, abs=1e-12)
        assert st[1] == pytest.approx(seg.sigma, rel=1e-10, abs=1e-12)
        lens = (seg.spans[:, 1] - seg.spans[:, 0]).astype(np.float64)
        np.testing.assert_allclose(c.logS[b, :m].cpu().numpy(), np.log(lens).astype(np.float32),
                                   rtol=2e-7, atol=0)
        # block offsets: exclusive prefix of the per-span block sizes
        sizes = [wl.Hkv * P.sekv.sekv_block_elems(int(x), wl.d, wl.rank) for x in lens]
        np.testing.assert_array_equal(c.blk_off[b, :m + 1].cpu().numpy(), np.concatenate([[0], np.cumsum(sizes)]))


def test_scan_degenerate_streams():
    """constant surprisal -> no boundary; alternating spikes -> singleton spans"""
    P = _lib()
    n = 64
    wl = WORKLOADS["c1"].scaled(n=n, B=2)
    H = torch.ones(2, n)
    H[1, ::2] = 10.0            # mu = 5.5, sigma = 4.5: alpha = 0.5 puts the threshold at 7.75
    c = _cache(wl)
    c.build(H.cuda(), None, None, 0.5, 0, "uniform", steps=P.SEKV_BUILD_SCAN | P.SEKV_BUILD_LAYOUT)
    torch.cuda.synchronize()
    assert int(c.a_count[0]) == 0 and int(c.m_count[0]) == 1
    assert int(c.span_beg[0, 0]) == 0 and int(c.span_end[0, 0]) == n
    seg = O.segment(T.f64(H[1]), 0.5, 0)
    assert int(c.a_count[1]) == len(seg.anchor_pos) == 32
    m = int(c.m_count[1])
    assert m == 32 and (c.span_end[1, :m] - c.span_beg[1, :m] == 1).all()


def test_scan_capacity_overflow_reports_status():
    P = _lib()
    wl = WORKLOADS["c1"].scaled(n=4096)
    H, _ = gen.surprisal(wl)
    c = _cache(wl, a_cap=8, m_cap=32)
    c.build(H.cuda(), None, None, wl.alpha, wl.window, wl.wmode, steps=P.SEKV_BUILD_SCAN)
    torch.cuda.synchronize()
    assert c.read_status() == P.sekv.SEKV_ERR_CAPACITY
    assert int(c.a_count[0]) == 8 and int(c.m_count[0]) == 32


# ---------------------------------------------------------------------------
def _ulp_bf16(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-30)))
    return 2.0 ** (e - 7)


SUMMARY_CASES = [
    ("c1", dict(), "uniform"),
    ("c1", dict(n=1500, window=33), "surprisal"),
    ("c1", dict(n=1024), "softmax"),
    ("c2", dict(n=4096, L=2), "softmax"),
    ("c2", dict(n=3000, L=1, B=2), "surprisal"),
    ("c2", dict(n=2048, L=1, d=64, Hq=8, Hkv=2), "uniform"),
]


@pytest.mark.parametrize("name,over,wmode", SUMMARY_CASES)
def test_summary_parity(name, over, wmode):
    P = _lib()
    wl = WORKLOADS[name].scaled(wmode=wmode, **over)
    H, K, V = T.make_inputs(wl)
    c = _cache(wl)
    c.build(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode,
            steps=P.SEKV_BUILD_SCAN | P.SEKV_BUILD_LAYOUT | P.SEKV_BUILD_SUMMARY)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    segs = T.oracle_segments(H, wl)
    units = T.oracle_units(K, V, H, segs, wl, with_bases=False)
    for (b, l, h), u in units.items():
        a, m = len(segs[b].anchor_pos), len(segs[b].spans)
        np.testing.assert_array_equal(T.f64(c.Ka[b, l, h, :a]), u.Ka)
        np.testing.assert_array_equal(T.f64(c.Va[b, l, h, :a]), u.Va)
        # one storage ulp, plus the fp32 accumulation bound where a mean cancels:
        # |S| * 2^-24 * max|row| (sequential fp32 sum of |S| weighted rows)
        lens = segs[b].lengths.astype(np.float64)[:, None]
        for X, got, want in ((K, T.f64(c.kbar[b, l, h, :m]), u.kbar), (V, T.f64(c.vbar[b, l, h, :m]), u.vbar)):
            rowmax = np.abs(T.f64(X[b, l, h])).max()
            acc = 4.0 * lens * 2.0 ** -24 * rowmax
            ulp = _ulp_bf16(want) if wl.dtype == "bf16" else np.abs(want) * 2.0 ** -23
            assert (np.abs(got - want) <= ulp * 1.0001 + acc).all()
        # 1/||kbar|| is consistent with the stored kbar (fp32) and close to the oracle's
        kb = T.f64(c.kbar[b, l, h, :m])
        nrm = np.sqrt((kb ** 2).sum(1))
        np.testing.assert_allclose(T.f64(c.inv_norm[b, l, h, :m]), 1.0 / nrm, rtol=2e-6)
        np.testing.assert_allclose(T.f64(c.inv_norm[b, l, h, :m]), u.inv_norm, rtol=2e-3)


# ---------------------------------------------------------------------------
def _read_block(c, b, l, kvh, S, beg, end):
    P = _lib()
    ln = end - beg
    rS = min(c.rank, ln, c.d)
    be = P.sekv.sekv_block_elems(ln, c.d, c.rank)
    o = int(c.blk_off[b, S]) + kvh * be
    blk = c.home[b, l, o:o + be].to("cpu", torch.float64).numpy()
    sec = T.block_sections(ln, rS, c.d)
    out = {}
    for name, (R, W) in (("A", (ln, rS)), ("C", (ln, rS)), ("B", (rS, c.d)), ("D", (rS, c.d))):
        off, n = sec[name]
        part = blk[off:off + n]
        out[name] = T.from_tiles8(part, R, W)
        # the padding of every section is exactly zero
        full = T.from_tiles8(part, T.r8(R), T.r8(W))
        mask = np.ones_like(full, dtype=bool)
        mask[:R, :W] = False
        assert not full[mask].any(), f"nonzero padding in {name}"
    return out["A"], out["B"], out["C"], out["D"]


BASIS_CASES = [
    ("c1", dict(n=1024)),                                      # fp32, d=64, r=4
    ("c2", dict(n=4096, L=1)),                                 # bf16, d=128, r=16, many |S| > d? (mean 64)
    ("c5", dict(n=4096, L=1, Hkv=2, Hq=8)),                    # bf16, r=32
    ("c2", dict(n=3000, L=1, d=64, Hq=8, Hkv=2, rank=8)),      # d=64: spans longer than d common
    ("c2", dict(n=2048, L=1, B=2, Hq=4, Hkv=1, alpha=2.5)),    # long spans (few boundaries): |S| > d path
]


@pytest.mark.parametrize("name,over", BASIS_CASES)
def test_basis_parity(name, over):
    P = _lib()
    wl = WORKLOADS[name].scaled(**over)
    H, K, V = T.make_inputs(wl)
    c = _cache(wl)
    c.build(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode, max_sweeps=30)
    torch.cuda.synchronize()
    assert c.read_status() == 0, P.sekv.sekv_status_str(c.read_status())
    segs = T.oracle_segments(H, wl)
    tol = 1e-4 if wl.dtype == "f32" else 1e-2
    worst = 0.0
    n_long = 0
    for b in range(wl.B):
        for l in range(wl.L):
            for h in range(wl.Hkv):
                Kb, Vb = T.f64(K[b, l, h]), T.f64(V[b, l, h])
                for S, (beg, end) in enumerate(segs[b].spans):
                    A, Bm, Cm, Dm = _read_block(c, b, l, h, S, int(beg), int(end))
                    n_long += (end - beg) > wl.d
                    for X, F1, F2 in ((Kb[beg:end], A, Bm), (Vb[beg:end], Cm, Dm)):
                        Ao, Bo = O.truncated_basis(X, wl.rank, wl.dtype)
                        ref = Ao @ Bo
                        err = np.linalg.norm(F1 @ F2 - ref) / max(np.linalg.norm(ref), 1e-30)
                        worst = max(worst, err)
                        assert err <= tol, (b, l, h, S, end - beg, err)
    print(f"worst relative Frobenius error {worst:.2e}; spans longer than d: {n_long}")


def test_basis_cold_home_in_pinned_memory():
    """the build writes the bases straight into pinned host memory"""
    P = _lib()
    wl = WORKLOADS["c2"].scaled(n=2048, L=1, Hq=8, Hkv=2)
    H, K, V = T.make_inputs(wl)
    dev = _cache(wl)
    host = _cache(wl, home="host")
    for c in (dev, host):
        c.build(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode)
    torch.cuda.synchronize()
    assert host.home.device.type == "cpu" and host.home.is_pinned()
    assert torch.equal(dev.home.cpu(), host.home)
