"""Shared test plumbing: oracle runs over generator inputs, threshold calibration
with margins, and moving oracle-built caches into the library's buffers."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle as O
from sekv_synth import WORKLOADS, gen


def _lib():
    import hierarchical_kv_cache_span_b200 as P
    return P

# zoom-threshold margin in logit space: no routing logit within DELTA_L of theta
DELTA_L = 1e-2


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def caps(wl, n=None):
    """capacities with headroom for every generator recipe (C1 has ~15% boundaries)"""
    n = wl.n if n is None else n
    a_cap = max(64, min(n, n // 4 + wl.window + 64))
    m_cap = max(64, ((min(n, n // 4 + 64) + 31) // 32) * 32)
    return a_cap, m_cap


def make_inputs(wl, device="cpu"):
    H, spikes = gen.surprisal(wl, device=device)
    K, V = gen.keys_values(wl, spikes, device=device)
    return H, K, V


def oracle_segments(H, wl):
    return [O.segment(f64(H[b]), wl.alpha, wl.window) for b in range(H.shape[0])]


def h_margin_ok(H_row: np.ndarray, seg) -> bool:
    return np.min(np.abs(H_row - seg.thr)) > 1e-9 * max(seg.sigma, 1e-30)


def oracle_units(K, V, H, segs, wl, with_bases=True, units=None, W=None, gates=None):
    """oracle caches per (b, l, kv head); W [L][Hq][dr][d] switches on the learned
    routing form, gates [B][L][Hkv][m_cap][2][rank] the rank gate"""
    out = {}
    B, L, Hkv = K.shape[0], K.shape[1], K.shape[2]
    G = wl.Hq // wl.Hkv
    todo = units if units is not None else [(b, l, h) for b in range(B) for l in range(L) for h in range(Hkv)]
    for (b, l, h) in todo:
        Wh = None if W is None else f64(W[l, h * G:(h + 1) * G])
        gh = None if gates is None else f64(gates[b, l, h, :len(segs[b].spans)])
        out[(b, l, h)] = O.build_unit(f64(K[b, l, h]), f64(V[b, l, h]), f64(H[b]), segs[b], wl.wmode,
                                      wl.rank, wl.dtype, with_bases=with_bases, W=Wh, gates=gh)
    return out


def unit_route(qh, unit, g, scale):
    """routing logits of query head g (within its kv head) for one unit: the learned
    form when the unit has routing summaries, else the identity form"""
    if unit.kbar_r is not None:
        return O.learned_routing_logits(qh, unit.W[g], unit.kbar_r[g], unit.logS)
    return O.routing_logits(qh, unit.kbar, unit.inv_norm, unit.logS, scale)


def oracle_route(q_np, unit, scale):
    """routing logits [G][m] for one unit"""
    return np.stack([unit_route(q_np[h], unit, h, scale) for h in range(q_np.shape[0])])


def calibrate_theta(ell_rows, quantile, delta=DELTA_L):
    """theta for one (layer, head): midpoint of the widest gap between sorted routing
    logits among those near the target quantile (at least 2*delta wide if possible)."""
    x = np.sort(np.asarray(ell_rows))
    if x.size == 0:
        return 0.0
    if x.size == 1:
        return float(x[0] - 1.0)
    k = int(round(quantile * (x.size - 1)))
    lo, hi = max(0, k - max(2, x.size // 50)), min(x.size - 2, k + max(2, x.size // 50))
    gaps = x[lo + 1:hi + 2] - x[lo:hi + 1]
    j = int(np.argmax(gaps)) + lo
    return float(0.5 * (x[j] + x[j + 1]))


def margin(ell, theta):
    return float(np.min(np.abs(np.asarray(ell) - theta))) if np.size(ell) else math.inf


def r8(x):
    return -(-int(x) // 8) * 8


def to_tiles8(M):
    """Flatten matrix M into the library's 8x8-blocked storage order (zero-padded
    to multiples of 8): a row-major grid of 8 x 8 tiles, each row-major inside."""
    R, W = M.shape
    P = np.zeros((r8(R), r8(W)), dtype=np.float64)
    P[:R, :W] = M
    return P.reshape(r8(R) // 8, 8, r8(W) // 8, 8).transpose(0, 2, 1, 3).reshape(-1)


def from_tiles8(flat, R, W):
    """Inverse of to_tiles8: the R x W matrix stored at ``flat``."""
    P = np.asarray(flat).reshape(r8(R) // 8, r8(W) // 8, 8, 8).transpose(0, 2, 1, 3).reshape(r8(R), r8(W))
    return P[:R, :W]


def block_sections(ln, rS, d):
    """(offset, elements) of A, C, B, D inside a span's block."""
    pa = r8(ln) * r8(rS)
    pb = r8(rS) * d
    return {"A": (0, pa), "C": (pa, pa), "B": (2 * pa, pb), "D": (2 * pa + pb, pb)}


def pack_bases(cache, segs, units):
    """Write oracle factors into the library's basis layout (device or pinned home)."""
    c = cache
    blk_off = c.blk_off.to("cpu").numpy()
    home = torch.zeros_like(c.home, device="cpu") if c.home.device.type != "cpu" else c.home
    home.zero_()
    flat = home.view(c.B, c.L, c.region)
    for (b, l, kvh), u in units.items():
        for S, (beg, end) in enumerate(segs[b].spans):
            ln = int(end - beg)
            A, Bm, Cm, Dm = u.bases[S]
            rS = A.shape[1]
            be = _lib().sekv.sekv_block_elems(ln, c.d, c.rank)
            o = int(blk_off[b, S]) + kvh * be
            seg = flat[b, l]
            for name, M in (("A", A), ("C", Cm), ("B", Bm), ("D", Dm)):
                off, n = block_sections(ln, rS, c.d)[name]
                seg[o + off:o + off + n] = torch.tensor(to_tiles8(M), dtype=c.dt)
    if c.home.device.type != "cpu":
        c.home.copy_(home)


def upload_oracle_cache(cache, segs, units, with_bases=True):
    """Fill segmentation + anchors + summaries (+ bases) of ``cache`` from the oracle."""
    P = _lib()
    c = cache
    for b, s in enumerate(segs):
        a, m = len(s.anchor_pos), len(s.spans)
        c.a_count[b] = a
        c.m_count[b] = m
        c.anchor_pos[b, :a] = torch.tensor(s.anchor_pos, dtype=torch.int32)
        if m:
            c.span_beg[b, :m] = torch.tensor(s.spans[:, 0], dtype=torch.int32)
            c.span_end[b, :m] = torch.tensor(s.spans[:, 1], dtype=torch.int32)
    # basis block offsets come from the library's layout step (storage layout only)
    c.build(None, None, None, 0.0, 0, "uniform", steps=P.SEKV_BUILD_LAYOUT)
    torch.cuda.synchronize()
    for (b, l, kvh), u in units.items():
        a, m = len(segs[b].anchor_pos), len(segs[b].spans)
        if a:
            c.Ka[b, l, kvh, :a] = torch.tensor(u.Ka, dtype=c.dt)
            c.Va[b, l, kvh, :a] = torch.tensor(u.Va, dtype=c.dt)
        if m:
            c.kbar[b, l, kvh, :m] = torch.tensor(u.kbar, dtype=c.dt)
            c.vbar[b, l, kvh, :m] = torch.tensor(u.vbar, dtype=c.dt)
            c.inv_norm[b, l, kvh, :m] = torch.tensor(u.inv_norm, dtype=torch.float32)
            c.logS[b, :m] = torch.tensor(u.logS, dtype=torch.float32)
            if u.kbar_r is not None and c.kbar_r is not None:
                G = c.Hq // c.Hkv
                c.kbar_r[b, l, kvh * G:(kvh + 1) * G, :m] = torch.tensor(u.kbar_r, dtype=c.dt)
    if with_bases:
        pack_bases(c, segs, units)
    torch.cuda.synchronize()


def budget_with_margin(q, units, segs, theta, scale, G, candidates=range(1, 41), delta=DELTA_L):
    """A zoom budget k such that, for every (b, l, query head) with more than k spans
    past theta, the k-th and (k+1)-th largest passing routing logits (oracle, fp64)
    are at least delta apart (so the fp32 kernel and the fp64 oracle keep the same
    spans), and at least one head is actually capped. None if no candidate works."""
    qn = f64(q)
    rows = []
    for (b, l, kvh), u in units.items():
        for g in range(G):
            h = kvh * G + g
            ell = unit_route(qn[b, l, h], u, g, scale)
            rows.append(np.sort(ell[ell > theta[l, h]])[::-1])
    for k in candidates:
        capped = [r for r in rows if len(r) > k]
        if capped and all(r[k - 1] - r[k] >= delta for r in capped):
            return k
    return None


def oracle_decode(q, units, segs, theta, scale, G, budget=None):
    """O [B][L][Hq][d], lse [B][L][Hq], zoom masks {(b,l,h): bool[m]} from the oracle."""
    B, L, Hq, d = q.shape
    Oo = np.zeros((B, L, Hq, d))
    lse = np.full((B, L, Hq), -np.inf)
    zooms = {}
    qn = f64(q)
    for (b, l, kvh), u in units.items():
        qg = qn[b, l, kvh * G:(kvh + 1) * G]
        z = np.zeros((G, len(segs[b].spans)), bool)
        for g in range(G):
            ell = unit_route(qg[g], u, g, scale)
            z[g] = O.zoom_decisions(ell, theta[l, kvh * G + g], budget=budget)
            zooms[(b, l, kvh * G + g)] = z[g]
        o, ls = O.decode_unit(qg, u.Ka, u.Va, u.kbar, u.vbar, u.logS, z, u.bases, scale)
        Oo[b, l, kvh * G:(kvh + 1) * G] = o
        lse[b, l, kvh * G:(kvh + 1) * G] = ls
    return Oo, lse, zooms


def zmask_bits(zmask: torch.Tensor, b, l, h, m) -> np.ndarray:
    w = zmask[b, l, h].to("cpu").numpy().astype(np.uint32)
    bits = ((w[:, None] >> np.arange(32, dtype=np.uint32)[None, :]) & 1).reshape(-1).astype(bool)
    return bits[:m]


def thetas_with_margin(q, units, segs, wl, scale, G, taus=None, quantile=None, max_tries=50):
    """Return (theta [L][Hq] float64, q) such that every routing logit of every
    unit is at least DELTA_L away from its head's theta.  With fixed/drawn taus
    the offending head's query is redrawn (seed + counter); with a quantile the
    threshold is put in a gap of the sorted logits."""
    B, L, Hq, d = q.shape
    q = q.clone()
    theta = np.zeros((L, Hq))
    for l in range(L):
        for h in range(Hq):
            kvh = h // G
            for attempt in range(max_tries):
                ells = [unit_route(f64(q[b, l, h]), units[(b, l, kvh)], h % G, scale)
                        for b in range(B) if (b, l, kvh) in units]
                allv = np.concatenate(ells) if ells else np.zeros(0)
                if quantile is not None:
                    th = calibrate_theta(allv, quantile)
                else:
                    th = float(O.tau_to_theta(taus[l, h]))
                if margin(allv, th) > DELTA_L:
                    theta[l, h] = th
                    break
                g = torch.Generator().manual_seed(gen.unit_seed(wl.seed, 99, l, h, attempt))
                fresh = torch.randn(B, d, generator=g).to(q.dtype)
                q[:, l, h] = fresh.to(q.device)
            else:
                raise RuntimeError(f"no theta with margin for layer {l} head {h}")
    return theta, q
