"""Plain fp64 CPU oracle for SeKV's mixed-resolution decode attention over a
span-structured KV cache.

TEST INFRASTRUCTURE ONLY. ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this module; the
product path (the CUDA library and its binding) never does, and this module
imports nothing from it. It shares no code, table or constant with the CUDA
side; the only common code is the seeded input generator in ``sekv_synth``.

Sources (cited by page title and section):

* [SeKV summary] "SeKV：支持分层语义记忆的分辨率自适应KV缓存，用于长上下文大语言模型推理"
  (paper.rainbus.top), the workflow paragraph: anchors and zoomed spans are
  attended with reconstructed token-level K/V; non-zoomed spans use the
  weighted mean key/value with a ``+log|S|`` correction; coarse entries and
  reconstructed tokens share ONE softmax.
* [SeKV blog] "SeKV：面向长上下文推理的分辨率自适应 KV Cache 与层级语义记忆"
  (liuzhao09.github.io): section 2.1 Eq. (1) and the boundary rule
  ``H_t > mu + alpha*sigma``; section 2.2 Eq. (2) weights, Eq. (3) routing
  summary, Fig. 2, Eq. (6)-(8) truncated SVD; section 2.3 Eq. (5) routing gate,
  Eq. (9) zoom decision; section 3.1 hyperparameters.

Readings fixed where the pages are silent:
mu/sigma are the per-sequence mean and population std over all n positions,
in fp64, with a strict ``>``; the last ``window`` positions are anchors too;
anchors are not members of any span, and spans are the maximal runs of
non-anchor positions; the routing projection is the identity (d' = d), so
the routing summary is ``kbar / ||kbar||``, unless a projection W is given (the
learned form, Eq. (3) and (5), with the query projected by the same W); all attention and routing logits
use the scale ``1/sqrt(d)`` and ``+log|S|`` is added after scaling; thresholds
are compared in logit space (``l > ln(tau/(1-tau))``, which is monotone-equal
to Eq. (9)); zoomed tokens use the reconstructed ``A_S B_S`` / ``C_S D_S``; a
unit with no entries has O = 0 and lse = -inf.

Parity pins for every function live in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "to_storage", "tau_to_theta", "Segmentation", "segment", "span_weights",
    "weighted_mean", "span_summaries", "truncated_basis", "span_bases",
    "routing_logits", "zoom_decisions", "decode_unit", "UnitCache", "build_unit",
    "routing_summary", "routing_summaries", "learned_routing_logits",
]


# ---------------------------------------------------------------------------
# storage rounding
# ---------------------------------------------------------------------------
def to_storage(x, dtype: str) -> np.ndarray:
    """Round fp64 values to the storage dtype ('f64', 'f32' or 'bf16') and return fp64.

    bf16 uses round-to-nearest-even on the fp32 bit pattern (the value is first
    rounded to fp32, as the GPU's fp32 results are).
    """
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f64":
        return x.copy()
    f = x.astype(np.float32)
    if dtype == "f32":
        return f.astype(np.float64)
    if dtype != "bf16":
        raise ValueError(dtype)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def tau_to_theta(tau) -> np.ndarray:
    """Eq. (9) in logit space: sigma(l) > tau  <=>  l > ln(tau / (1 - tau)).

    tau <= 0 zooms everything (theta = -inf); tau >= 1 zooms nothing (+inf).
    """
    tau = np.asarray(tau, dtype=np.float64)
    out = np.empty_like(tau)
    lo = tau <= 0.0
    hi = tau >= 1.0
    mid = ~(lo | hi)
    out[lo] = -np.inf
    out[hi] = np.inf
    out[mid] = np.log(tau[mid] / (1.0 - tau[mid]))
    return out


# ---------------------------------------------------------------------------
# prefill: segmentation  [SeKV blog, section 2.1, Eq. (1) and boundary rule]
# ---------------------------------------------------------------------------
@dataclass
class Segmentation:
    mu: float
    sigma: float
    thr: float
    anchor: np.ndarray          # bool [n]
    anchor_pos: np.ndarray      # int64 [a]
    spans: np.ndarray           # int64 [m][2]  (begin, end) half-open

    @property
    def lengths(self) -> np.ndarray:
        return (self.spans[:, 1] - self.spans[:, 0]) if len(self.spans) else np.zeros(0, np.int64)


def segment(H, alpha: float, window: int) -> Segmentation:
    """Boundaries are positions with H_t > mu + alpha*sigma (mu, sigma: mean and
    population std of the in-context surprisal); boundary tokens and the local
    window are anchors; spans are the maximal runs of the remaining tokens."""
    H = np.asarray(H, dtype=np.float64)
    n = H.shape[0]
    mu = float(np.mean(H))
    sigma = float(np.sqrt(np.mean((H - mu) ** 2)))
    thr = mu + alpha * sigma
    anchor = H > thr
    if window > 0:
        anchor[max(0, n - window):] = True
    spans: List[Tuple[int, int]] = []
    t = 0
    while t < n:
        if anchor[t]:
            t += 1
            continue
        beg = t
        while t < n and not anchor[t]:
            t += 1
        spans.append((beg, t))
    sp = np.array(spans, dtype=np.int64).reshape(-1, 2)
    return Segmentation(mu, sigma, thr, anchor, np.flatnonzero(anchor).astype(np.int64), sp)


# ---------------------------------------------------------------------------
# prefill: span summaries  [SeKV blog 2.2 Eq. (2); SeKV summary workflow]
# ---------------------------------------------------------------------------
def span_weights(Hs, wmode: str) -> np.ndarray:
    """Per-token weights inside one span.

    'surprisal' is Eq. (2), w_t = H_t / sum_{k in S} H_k (uniform if the sum is 0);
    'uniform' is w_t = 1; 'softmax' is w_t = exp(H_t) / sum_{k in S} exp(H_k).
    """
    Hs = np.asarray(Hs, dtype=np.float64)
    if wmode == "uniform":
        return np.ones_like(Hs)
    if wmode == "surprisal":
        s = Hs.sum()
        return Hs / s if s > 0.0 else np.ones_like(Hs)
    if wmode == "softmax":
        e = np.exp(Hs - Hs.max())
        return e / e.sum()
    raise ValueError(wmode)


def weighted_mean(X, w) -> np.ndarray:
    """kbar_S = sum_t w_t X_t / sum_t w_t (the same form gives vbar_S)."""
    X = np.asarray(X, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    return (w[:, None] * X).sum(axis=0) / w.sum()


def span_summaries(K, V, H, seg: Segmentation, wmode: str, dtype: str):
    """Per span: stored kbar, vbar; 1/||stored kbar|| (0 for a zero vector) and
    log|S|, both rounded to fp32 unless ``dtype`` is 'f64'.  The identity routing projection makes Eq. (3)'s routing
    summary kbar/||kbar||, so 1/||kbar|| is all the routing step needs."""
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    H = np.asarray(H, dtype=np.float64)
    m, d = len(seg.spans), K.shape[1]
    meta = "f64" if dtype == "f64" else "f32"     # inv_norm and log|S| are fp32 on the device
    kbar = np.zeros((m, d))
    vbar = np.zeros((m, d))
    inv_norm = np.zeros(m)
    logS = np.zeros(m)
    for i, (b, e) in enumerate(seg.spans):
        w = span_weights(H[b:e], wmode)
        kbar[i] = to_storage(weighted_mean(K[b:e], w), dtype)
        vbar[i] = to_storage(weighted_mean(V[b:e], w), dtype)
        nrm = np.sqrt(np.sum(kbar[i] ** 2))
        inv_norm[i] = to_storage(1.0 / nrm, meta) if nrm > 0.0 else 0.0
        logS[i] = to_storage(np.log(e - b), meta)
    return kbar, vbar, inv_norm, logS


# ---------------------------------------------------------------------------
# prefill: learned-form routing summaries  [SeKV blog 2.2 Eq. (3)]
# ---------------------------------------------------------------------------
def routing_summary(Ks, w, W) -> np.ndarray:
    """Eq. (3) for one span and one (layer, head): every token's key is projected
    into the routing space, the projections are summed with the span weights and
    the sum is scaled to unit length: sum_t w_t W K_t / ||sum_t w_t W K_t||_2.
    A zero sum gives the zero vector (a reading: the pages do not say)."""
    Ks = np.asarray(Ks, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    proj = Ks @ W.T                     # row t is W K_t
    y = (w[:, None] * proj).sum(axis=0)
    nrm = np.sqrt(np.sum(y * y))
    return y / nrm if nrm > 0.0 else np.zeros_like(y)


def routing_summaries(K, H, seg: Segmentation, wmode: str, W_heads, dtype: str) -> np.ndarray:
    """[G][m][d'] stored routing summaries of every span for the G query heads that
    share this key head (each head has its own W, [G][d'][d])."""
    W_heads = np.asarray(W_heads, dtype=np.float64)
    G, dr = W_heads.shape[0], W_heads.shape[1]
    out = np.zeros((G, len(seg.spans), dr))
    for i, (b, e) in enumerate(seg.spans):
        w = span_weights(np.asarray(H, dtype=np.float64)[b:e], wmode)
        for g in range(G):
            out[g, i] = to_storage(routing_summary(np.asarray(K)[b:e], w, W_heads[g]), dtype)
    return out


# ---------------------------------------------------------------------------
# prefill: truncated bases  [SeKV blog 2.2 Eq. (6)-(8)]
# ---------------------------------------------------------------------------
def truncated_basis(X, r: int, dtype: str, gate=None):
    """Rank-r_S truncated SVD of X (|S| x d), r_S = min(r, |S|, d), as two stored
    factors with A @ B = sum_{i <= r_S} m_i sigma_i u_i v_i^T (Eq. (6)); the rank
    gate m (components in descending singular-value order) is 1 when not given.

    Factor split: if |S| <= d, A = U_r (|S| x r_S) and B = M_r Sigma_r V_r^T;
    otherwise A = U_r Sigma_r and B = M_r V_r^T (r_S x d), M_r = diag(m_1..m_rS).
    """
    X = np.asarray(X, dtype=np.float64)
    ns, d = X.shape
    rs = min(r, ns, d)
    U, s, Vt = np.linalg.svd(X, full_matrices=False)
    m = np.ones(rs) if gate is None else np.asarray(gate, dtype=np.float64)[:rs]
    if ns <= d:
        A = U[:, :rs]
        B = (m * s[:rs])[:, None] * Vt[:rs]
    else:
        A = U[:, :rs] * s[None, :rs]
        B = m[:, None] * Vt[:rs]
    return to_storage(A, dtype), to_storage(B, dtype)


def span_bases(K, V, seg: Segmentation, r: int, dtype: str, gates=None):
    """(A_S, B_S, C_S, D_S) per span: K_S ~ A_S B_S and V_S ~ C_S D_S. ``gates``
    ([m][2][r], keys then values) is the rank gate of Eq. (6), 1 when absent."""
    out = []
    for i, (b, e) in enumerate(seg.spans):
        gk = None if gates is None else gates[i][0]
        gv = None if gates is None else gates[i][1]
        A, B = truncated_basis(np.asarray(K)[b:e], r, dtype, gk)
        C, D = truncated_basis(np.asarray(V)[b:e], r, dtype, gv)
        out.append((A, B, C, D))
    return out


# ---------------------------------------------------------------------------
# decode  [SeKV blog 2.3 Eq. (5), (9); SeKV summary workflow; Fig. 2 merge]
# ---------------------------------------------------------------------------
def routing_logits(qh, kbar, inv_norm, logS, scale: float) -> np.ndarray:
    """Eq. (5)'s pre-sigmoid logit with W = I: l_S = q . kbar_S / ||kbar_S|| * scale + log|S|."""
    s = np.asarray(kbar, dtype=np.float64) @ np.asarray(qh, dtype=np.float64)
    return s * np.asarray(inv_norm, dtype=np.float64) * scale + np.asarray(logS, dtype=np.float64)


def learned_routing_logits(qh, W, kbar_r, logS) -> np.ndarray:
    """Eq. (5)'s pre-sigmoid logit with a routing projection: the query is projected
    by the same W as the keys (a reading), q~ = W q, and
    l_S = q~ . Kbar_S / sqrt(d') + log|S| with Kbar_S the Eq. (3) summaries."""
    W = np.asarray(W, dtype=np.float64)
    qt = W @ np.asarray(qh, dtype=np.float64)
    dr = W.shape[0]
    return np.asarray(kbar_r, dtype=np.float64) @ qt / np.sqrt(dr) + np.asarray(logS, dtype=np.float64)


def zoom_decisions(ell, theta: float, budget=None) -> np.ndarray:
    """Eq. (9): z_S = 1[sigma(l_S) > tau], i.e. l_S > theta = ln(tau/(1-tau)).

    With a budget (SeKV blog 2.3, the paragraph under Eq. (9)): when more spans
    pass the threshold than the budget allows, the spans are kept in descending
    alpha~ order; alpha~ = sigma(l_S) is monotone in l_S, so the `budget` largest
    logits stay. Equal logits keep the lower span index first (a reading: the
    pages give no tie rule)."""
    ell = np.asarray(ell, dtype=np.float64)
    z = ell > theta
    if budget is None or int(z.sum()) <= int(budget):
        return z
    passing = [int(s) for s in np.flatnonzero(z)]
    passing.sort(key=lambda s: (-ell[s], s))       # descending logit, then lower span index
    keep = np.zeros(z.shape, dtype=bool)
    keep[passing[:int(budget)]] = True
    return keep


def decode_unit(q, Ka, Va, kbar, vbar, logS, zoom, bases, scale: float):
    """One KV head's decode for its G query heads.

    For head h the logit list is: every anchor, q.Ka_i * scale (value Va_i);
    every non-zoomed span, q.kbar_S * scale + log|S| (value vbar_S); every
    token t of every zoomed span, q.(A_S B_S)_t * scale (value (C_S D_S)_t).
    One softmax over the whole list gives O_h; lse_h is its log-sum-exp.
    """
    q = np.asarray(q, dtype=np.float64)
    G, d = q.shape
    Ka = np.asarray(Ka, dtype=np.float64).reshape(-1, d)
    Va = np.asarray(Va, dtype=np.float64).reshape(-1, d)
    kbar = np.asarray(kbar, dtype=np.float64).reshape(-1, d)
    vbar = np.asarray(vbar, dtype=np.float64).reshape(-1, d)
    logS = np.asarray(logS, dtype=np.float64)
    zoom = np.asarray(zoom, dtype=bool).reshape(G, -1)
    O = np.zeros((G, d))
    lse = np.full(G, -np.inf)
    for h in range(G):
        logits = [Ka @ q[h] * scale]
        values = [Va]
        coarse = ~zoom[h]
        logits.append(kbar[coarse] @ q[h] * scale + logS[coarse])
        values.append(vbar[coarse])
        for S in np.flatnonzero(zoom[h]):
            A, B, C, D = (np.asarray(z, dtype=np.float64) for z in bases[S])
            logits.append((A @ B) @ q[h] * scale)
            values.append(C @ D)
        x = np.concatenate(logits)
        Vall = np.concatenate(values, axis=0)
        if x.size == 0:
            continue
        mx = x.max()
        e = np.exp(x - mx)
        Z = e.sum()
        O[h] = (e @ Vall) / Z
        lse[h] = mx + np.log(Z)
    return O, lse


# ---------------------------------------------------------------------------
# convenience: everything the decode of one (sequence, layer, kv head) needs
# ---------------------------------------------------------------------------
@dataclass
class UnitCache:
    Ka: np.ndarray
    Va: np.ndarray
    kbar: np.ndarray
    vbar: np.ndarray
    inv_norm: np.ndarray
    logS: np.ndarray
    bases: Optional[list]
    W: Optional[np.ndarray] = None        # [G][d'][d] routing projections (learned form)
    kbar_r: Optional[np.ndarray] = None   # [G][m][d'] routing summaries (learned form)


def build_unit(K, V, H, seg: Segmentation, wmode: str, rank: int, dtype: str,
               with_bases: bool = True, W=None, gates=None) -> UnitCache:
    """Everything one (sequence, layer, kv head) needs. ``W`` ([G][d'][d]) switches
    on the learned routing form; ``gates`` ([m][2][r]) is the rank gate."""
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    kbar, vbar, inv_norm, logS = span_summaries(K, V, H, seg, wmode, dtype)
    bases = span_bases(K, V, seg, rank, dtype, gates) if with_bases else None
    kbar_r = None
    if W is not None:
        W = np.asarray(W, dtype=np.float64)
        kbar_r = routing_summaries(K, H, seg, wmode, W, dtype)
    return UnitCache(K[seg.anchor_pos].copy(), V[seg.anchor_pos].copy(), kbar, vbar,
                     inv_norm, logS, bases, W, kbar_r)
