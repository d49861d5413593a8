"""Pins of the fp64 oracle to facts other than itself: hand-derived fixtures,
closed forms, textbook / library routines and brute force on tiny inputs.

Each group names the passage of the SeKV pages it pins.
"""
import json
import math
import os
import statistics

import numpy as np
import pytest
from scipy.special import expit, logsumexp, softmax

import oracle as O
from tests.textbook import dense_attention

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# Segmentation  (SeKV blog 2.1: H_t > mu + alpha*sigma; boundary tokens -> anchors)
# ---------------------------------------------------------------------------
def _two_level():
    g = _gold("two_level_stream.json")
    H = np.full(g["n"], g["c"])
    H[g["spikes"]] = g["h"]
    return g, H


def test_segment_two_level_closed_form():
    g, H = _two_level()
    seg = O.segment(H, g["alpha"], g["window"])
    assert seg.mu == pytest.approx(g["mu"], abs=1e-14)
    assert seg.sigma == pytest.approx(math.sqrt(g["sigma_sq"]), abs=1e-14)
    assert seg.anchor_pos.tolist() == g["anchors"]
    assert seg.spans.tolist() == g["spans"]


def test_segment_threshold_above_spikes_gives_one_span():
    g, H = _two_level()
    # (h - mu) / sigma = 3.75 / 0.968 = 3.87 < alpha_none = 4, so nothing crosses.
    seg = O.segment(H, g["alpha_none"], 0)
    assert seg.anchor_pos.tolist() == []
    assert seg.spans.tolist() == g["spans_none"]


def test_segment_local_window():
    g, H = _two_level()
    seg = O.segment(H, g["alpha"], g["window_w"])
    assert seg.anchor_pos.tolist() == g["anchors_w"]
    assert seg.spans.tolist() == g["spans_w"]


def _brute_segment(H, alpha, window):
    mu = statistics.fmean(H)
    sigma = statistics.pstdev(H)
    thr = mu + alpha * sigma
    n = len(H)
    anchor = [H[t] > thr or t >= n - window for t in range(n)]
    spans, cur = [], None
    for t in range(n):
        if not anchor[t] and cur is None:
            cur = t
        if anchor[t] and cur is not None:
            spans.append([cur, t])
            cur = None
    if cur is not None:
        spans.append([cur, n])
    return [t for t in range(n) if anchor[t]], spans, thr


def test_segment_bruteforce_tiny():
    rng = np.random.default_rng(7)
    checked = 0
    for trial in range(400):
        n = int(rng.integers(1, 13))
        H = rng.gamma(2.0, 1.0, size=n)
        alpha = float(rng.choice([0.0, 0.5, 1.0, 1.5]))
        window = int(rng.integers(0, 3))
        anchors, spans, thr = _brute_segment(H.tolist(), alpha, window)
        if np.min(np.abs(H - thr)) < 1e-9:
            continue
        seg = O.segment(H, alpha, window)
        assert seg.anchor_pos.tolist() == anchors
        assert seg.spans.tolist() == spans
        checked += 1
    assert checked > 300


def test_segment_partition_and_maximality():
    rng = np.random.default_rng(3)
    H = rng.gamma(2.0, 1.0, size=3000)
    H[rng.random(3000) < 1 / 64] += 6
    seg = O.segment(H, 1.0, 37)
    cover = np.zeros(3000, int)
    cover[seg.anchor_pos] += 1
    for b, e in seg.spans:
        assert e > b
        cover[b:e] += 1
        assert b == 0 or seg.anchor[b - 1]
        assert e == 3000 or seg.anchor[e]
    assert (cover == 1).all()
    assert seg.anchor[-37:].all()


# ---------------------------------------------------------------------------
# Weights and weighted means (SeKV blog 2.2 Eq. (2); SeKV summary workflow)
# ---------------------------------------------------------------------------
def test_eq2_hand_example():
    g = _gold("eq2_weighted_mean.json")
    w = O.span_weights(g["H"], "surprisal")
    np.testing.assert_allclose(w, g["weights"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(O.weighted_mean(g["K"], w), g["kbar"], rtol=0, atol=1e-14)


def test_uniform_weights_are_arithmetic_mean():
    rng = np.random.default_rng(1)
    X = rng.normal(size=(17, 5))
    np.testing.assert_allclose(O.weighted_mean(X, O.span_weights(np.ones(17), "uniform")),
                               np.mean(X, axis=0), rtol=1e-14, atol=1e-14)


def test_softmax_weights_match_scipy():
    Hs = np.array([0.3, 2.5, 1.1, 7.0])
    np.testing.assert_allclose(O.span_weights(Hs, "softmax"), softmax(Hs), rtol=1e-14)


def test_eq2_zero_sum_falls_back_to_uniform():
    np.testing.assert_array_equal(O.span_weights(np.zeros(3), "surprisal"), np.ones(3))


@pytest.mark.parametrize("wmode", ["uniform", "surprisal", "softmax"])
def test_constant_span_summary_is_the_row(wmode):
    row = np.array([0.5, -1.25, 3.0])
    X = np.tile(row, (6, 1))
    w = O.span_weights(np.array([1.0, 2.0, 0.5, 3.0, 4.0, 0.1]), wmode)
    np.testing.assert_allclose(O.weighted_mean(X, w), row, rtol=1e-15)


def test_summary_norm_and_logS_closed_form():
    H = np.array([9.0, 1.0, 1.0, 1.0, 1.0, 9.0])
    seg = O.segment(H, 1.0, 0)                 # anchors 0 and 5, one span [1, 5)
    K = np.zeros((6, 2)); K[1:5] = [3.0, 4.0]
    V = np.ones((6, 2))
    kbar, vbar, inv_norm, logS = O.span_summaries(K, V, H, seg, "uniform", "f32")
    assert seg.spans.tolist() == [[1, 5]]
    assert inv_norm[0] == pytest.approx(0.2, rel=1e-7)
    assert logS[0] == pytest.approx(math.log(4), rel=1e-7)
    K[1:5] = 0.0
    _, _, inv_norm0, _ = O.span_summaries(K, V, H, seg, "uniform", "f32")
    assert inv_norm0[0] == 0.0


def test_bf16_rounding_matches_library_conversion():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.normal(size=2000) * 10 ** rng.uniform(-3, 3, 2000),
                        [1 + 2 ** -8, 1 + 3 * 2 ** -8, -1 - 2 ** -8, 0.0]])
    ref = torch.tensor(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.to_storage(x, "bf16"), ref)
    assert O.to_storage([1 + 2 ** -8], "bf16")[0] == 1.0          # tie to even
    assert O.to_storage([1 + 3 * 2 ** -8], "bf16")[0] == 1 + 2 ** -6


# ---------------------------------------------------------------------------
# Truncated bases (SeKV blog 2.2 Eq. (6)-(8), gate m_i = 1)
# ---------------------------------------------------------------------------
def _orth(rng, rows, cols):
    q, _ = np.linalg.qr(rng.normal(size=(rows, cols)))
    return q


@pytest.mark.parametrize("ns,d", [(12, 20), (20, 12), (16, 16)])
@pytest.mark.parametrize("r", [1, 3, 5])
def test_basis_known_singular_structure(ns, d, r):
    rng = np.random.default_rng(ns * 100 + d + r)
    k = min(ns, d)
    U, W = _orth(rng, ns, k), _orth(rng, d, k)
    s = np.linspace(10.0, 1.0, k) ** 1.5            # distinct, descending
    X = (U * s) @ W.T
    A, B = O.truncated_basis(X, r, "f64")
    expect = (U[:, :r] * s[:r]) @ W[:, :r].T
    np.testing.assert_allclose(A @ B, expect, rtol=0, atol=1e-10 * s[0])
    if ns <= d:
        np.testing.assert_allclose(A.T @ A, np.eye(r), atol=1e-12)
    else:
        np.testing.assert_allclose(B @ B.T, np.eye(r), atol=1e-12)


@pytest.mark.parametrize("ns,d,g", [(30, 16, 4), (9, 16, 4), (5, 8, 5)])
def test_basis_exact_for_low_rank_and_full_rank(ns, d, g):
    rng = np.random.default_rng(ns + d)
    X = rng.normal(size=(ns, g)) @ rng.normal(size=(g, d))
    for r in (g, g + 2, min(ns, d), 100):
        A, B = O.truncated_basis(X, r, "f64")
        np.testing.assert_allclose(A @ B, X, atol=1e-10 * np.abs(X).max())


@pytest.mark.parametrize("ns,d", [(40, 16), (10, 32)])
def test_basis_eckart_young(ns, d):
    rng = np.random.default_rng(11)
    X = rng.normal(size=(ns, d))
    lam = np.sort(np.linalg.eigvalsh(X.T @ X))[::-1]      # sigma_i^2, another routine
    for r in (1, 4, 7):
        A, B = O.truncated_basis(X, r, "f64")
        resid = np.sum((X - A @ B) ** 2)
        assert resid == pytest.approx(np.sum(lam[r:]), rel=1e-9, abs=1e-9)


# ---------------------------------------------------------------------------
# Routing (SeKV blog 2.3 Eq. (5), Eq. (9))
# ---------------------------------------------------------------------------
def test_tau_to_theta_closed_form():
    th = O.tau_to_theta(np.array([0.5, math.e / (1 + math.e), 0.0, 1.0, -0.2, 1.5]))
    assert th[0] == 0.0
    assert th[1] == pytest.approx(1.0, abs=1e-15)
    assert th[2] == -np.inf and th[4] == -np.inf
    assert th[3] == np.inf and th[5] == np.inf


def test_routing_hand_example():
    g = _gold("routing_example.json")
    kbar = np.array([g["kbar"]])
    inv = np.array([1.0 / np.linalg.norm(kbar)])
    ell = O.routing_logits(g["q"], kbar, inv, np.array([math.log(g["len"])]), 1 / math.sqrt(2))
    assert ell[0] == pytest.approx(g["ell"], abs=1e-14)
    assert O.zoom_decisions(ell, O.tau_to_theta(g["tau_zoom"]))[0]
    assert not O.zoom_decisions(ell, O.tau_to_theta(g["tau_nozoom"]))[0]


def test_logit_space_decision_equals_sigmoid_decision():
    rng = np.random.default_rng(2)
    ell = rng.normal(scale=3.0, size=5000)
    for tau in (0.05, 0.3, 0.5, 0.77, 0.99):
        th = O.tau_to_theta(tau)
        gap = np.abs(ell - th) > 1e-9
        np.testing.assert_array_equal(O.zoom_decisions(ell, th)[gap], (expit(ell) > tau)[gap])


def test_singleton_routing_has_no_size_prior():
    rng = np.random.default_rng(4)
    kb, q = rng.normal(size=(1, 8)), rng.normal(size=8)
    inv = np.array([1 / np.linalg.norm(kb)])
    ell = O.routing_logits(q, kb, inv, np.array([math.log(1)]), 0.5)
    cos = kb[0] @ q / np.linalg.norm(kb) / np.linalg.norm(q)
    assert ell[0] == pytest.approx(cos * np.linalg.norm(q) * 0.5, rel=1e-13)


# ---------------------------------------------------------------------------
# Stage-2 decode (SeKV summary workflow: one softmax over anchors,
# reconstructed zoomed tokens and log|S|-corrected summaries; Fig. 2 merge)
# ---------------------------------------------------------------------------
def _random_unit(rng, n, d, anchor_frac=0.2, identical=()):
    K = rng.normal(size=(n, d))
    V = rng.normal(size=(n, d))
    H = rng.gamma(2.0, 1.0, size=n)
    anchor = rng.random(n) < anchor_frac
    anchor[0] = True
    spans, cur = [], None
    for t in range(n):
        if not anchor[t] and cur is None:
            cur = t
        if anchor[t] and cur is not None:
            spans.append((cur, t)); cur = None
    if cur is not None:
        spans.append((cur, n))
    seg = O.Segmentation(0.0, 0.0, 0.0, anchor, np.flatnonzero(anchor),
                         np.array(spans, dtype=np.int64).reshape(-1, 2))
    for S in identical:
        b, e = seg.spans[S]
        K[b:e] = K[b]
        V[b:e] = V[b]
    return K, V, H, seg


def _decode(K, V, H, seg, wmode, rank, zoom, q, scale):
    c = O.build_unit(K, V, H, seg, wmode, rank, "f64")
    return O.decode_unit(q, c.Ka, c.Va, c.kbar, c.vbar, c.logS, zoom, c.bases, scale)


def test_singleton_spans_equal_dense_attention():
    rng = np.random.default_rng(21)
    n, d, G = 60, 8, 3
    K, V = rng.normal(size=(n, d)), rng.normal(size=(n, d))
    anchor = rng.random(n) < 0.3
    spans = np.array([[t, t + 1] for t in range(n) if not anchor[t]])
    seg = O.Segmentation(0, 0, 0, anchor, np.flatnonzero(anchor), spans)
    q = rng.normal(size=(G, d))
    for wmode in ("uniform", "surprisal", "softmax"):
        Oo, lse = _decode(K, V, rng.gamma(2, 1, n), seg, wmode, 4, np.zeros((G, len(spans)), bool), q, 0.35)
        for h in range(G):
            o_ref, l_ref = dense_attention(q[h], K, V, 0.35)
            np.testing.assert_allclose(Oo[h], o_ref, atol=1e-12)
            assert lse[h] == pytest.approx(l_ref, abs=1e-12)


def test_all_zoom_full_rank_equals_dense_attention():
    rng = np.random.default_rng(22)
    n, d, G = 80, 6, 2
    K, V, H, seg = _random_unit(rng, n, d)
    q = rng.normal(size=(G, d))
    zoom = np.ones((G, len(seg.spans)), bool)
    Oo, lse = _decode(K, V, H, seg, "softmax", d, zoom, q, 0.4)
    for h in range(G):
        o_ref, l_ref = dense_attention(q[h], K, V, 0.4)
        np.testing.assert_allclose(Oo[h], o_ref, atol=1e-11)
        assert lse[h] == pytest.approx(l_ref, abs=1e-11)


def test_identical_span_is_represented_exactly():
    rng = np.random.default_rng(23)
    n, d, G = 70, 5, 2
    K, V, H, seg = _random_unit(rng, n, d)
    long_spans = [i for i, (b, e) in enumerate(seg.spans) if e - b >= 2]
    K, V, H, seg = _random_unit(np.random.default_rng(23), n, d, identical=())
    # make EVERY span constant, so every coarse entry must be exact
    for b, e in seg.spans:
        K[b:e] = K[b]
        V[b:e] = V[b]
    q = rng.normal(size=(G, d))
    zoom = np.zeros((G, len(seg.spans)), bool)
    Oo, lse = _decode(K, V, H, seg, "surprisal", 2, zoom, q, 0.5)
    assert long_spans
    for h in range(G):
        o_ref, l_ref = dense_attention(q[h], K, V, 0.5)
        np.testing.assert_allclose(Oo[h], o_ref, atol=1e-12)
        assert lse[h] == pytest.approx(l_ref, abs=1e-12)


def test_coarse_entry_equals_replicated_summary():
    """Brute force: each non-zoomed summary replicated |S| times in a plain
    softmax (no correction) equals the oracle's +log|S| entry; zoomed spans
    with full-rank bases contribute their exact tokens."""
    rng = np.random.default_rng(24)
    n, d, G = 90, 7, 4
    K, V, H, seg = _random_unit(rng, n, d)
    m = len(seg.spans)
    q = rng.normal(size=(G, d))
    zoom = rng.random((G, m)) < 0.4
    c = O.build_unit(K, V, H, seg, "softmax", d, "f64")
    Oo, lse = O.decode_unit(q, c.Ka, c.Va, c.kbar, c.vbar, c.logS, zoom, c.bases, 0.3)
    for h in range(G):
        rowsK, rowsV = [K[t] for t in seg.anchor_pos], [V[t] for t in seg.anchor_pos]
        for S, (b, e) in enumerate(seg.spans):
            if zoom[h, S]:
                rowsK += list(K[b:e]); rowsV += list(V[b:e])
            else:
                rowsK += [c.kbar[S]] * (e - b); rowsV += [c.vbar[S]] * (e - b)
        o_ref, l_ref = dense_attention(q[h], np.array(rowsK), np.array(rowsV), 0.3)
        np.testing.assert_allclose(Oo[h], o_ref, atol=1e-11)
        assert lse[h] == pytest.approx(l_ref, abs=1e-11)


def test_zoomed_low_rank_span_uses_reconstruction():
    """A zoomed span contributes the tokens of A@B / C@D, not the originals."""
    rng = np.random.default_rng(25)
    n, d = 40, 6
    K, V, H, seg = _random_unit(rng, n, d, anchor_frac=0.1)
    q = rng.normal(size=(1, d))
    zoom = np.ones((1, len(seg.spans)), bool)
    c = O.build_unit(K, V, H, seg, "uniform", 2, "f64")
    Oo, lse = O.decode_unit(q, c.Ka, c.Va, c.kbar, c.vbar, c.logS, zoom, c.bases, 0.4)
    rowsK, rowsV = [K[seg.anchor_pos]], [V[seg.anchor_pos]]
    for S, (b, e) in enumerate(seg.spans):
        A, B, C, D = c.bases[S]
        rowsK.append(A @ B); rowsV.append(C @ D)
    o_ref, l_ref = dense_attention(q[0], np.concatenate(rowsK), np.concatenate(rowsV), 0.4)
    np.testing.assert_allclose(Oo[0], o_ref, atol=1e-12)
    o_orig, _ = dense_attention(q[0], K, V, 0.4)
    assert np.abs(Oo[0] - o_orig).max() > 1e-3      # rank 2 is lossy here


def test_empty_unit():
    Oo, lse = O.decode_unit(np.ones((2, 4)), np.zeros((0, 4)), np.zeros((0, 4)), np.zeros((0, 4)),
                            np.zeros((0, 4)), np.zeros(0), np.zeros((2, 0), bool), [], 0.5)
    assert (Oo == 0).all() and np.isneginf(lse).all()


def test_lse_is_log_partition():
    rng = np.random.default_rng(26)
    K, V, H, seg = _random_unit(rng, 50, 4)
    q = rng.normal(size=(1, 4))
    zoom = np.zeros((1, len(seg.spans)), bool)
    c = O.build_unit(K, V, H, seg, "uniform", 2, "f64")
    _, lse = O.decode_unit(q, c.Ka, c.Va, c.kbar, c.vbar, c.logS, zoom, c.bases, 0.7)
    x = np.concatenate([c.Ka @ q[0] * 0.7, c.kbar @ q[0] * 0.7 + c.logS])
    assert lse[0] == pytest.approx(logsumexp(x), abs=1e-13)


# ---------------------------------------------------------------------------
# Planted mistakes: each pin above must catch a plausible oracle bug.
# ---------------------------------------------------------------------------
def test_planted_dropped_log_correction_is_caught():
    rng = np.random.default_rng(24)
    K, V, H, seg = _random_unit(rng, 60, 5)
    for b, e in seg.spans:
        K[b:e] = K[b]; V[b:e] = V[b]
    q = rng.normal(size=(1, 5))
    c = O.build_unit(K, V, H, seg, "uniform", 2, "f64")
    zoom = np.zeros((1, len(seg.spans)), bool)
    bad, _ = O.decode_unit(q, c.Ka, c.Va, c.kbar, c.vbar, 0 * c.logS, zoom, c.bases, 0.5)
    o_ref, _ = dense_attention(q[0], K, V, 0.5)
    assert np.abs(bad[0] - o_ref).max() > 1e-3


def test_planted_sample_std_is_caught(monkeypatch):
    g, H = _two_level()
    real_sqrt = np.sqrt

    def ddof1_sqrt(x):                     # turns the population variance into the sample one
        return real_sqrt(x * g["n"] / (g["n"] - 1))
    monkeypatch.setattr(O.sekv_oracle.np, "sqrt", ddof1_sqrt)
    seg = O.segment(H, g["alpha"], 0)
    monkeypatch.undo()
    assert seg.sigma != pytest.approx(math.sqrt(g["sigma_sq"]), abs=1e-6)


def test_planted_swapped_basis_factors_are_caught():
    rng = np.random.default_rng(9)
    U, W = _orth(rng, 12, 8), _orth(rng, 20, 8)
    X = (U * np.arange(8, 0, -1.0)) @ W.T
    A, B = O.truncated_basis(X, 3, "f64")
    expect = (U[:, :3] * np.arange(8, 5, -1.0)) @ W[:, :3].T
    assert np.abs(A @ B - expect).max() < 1e-10
    A2, B2 = O.truncated_basis(X.T, 3, "f64")       # a transposed operand
    assert (A2 @ B2).shape != expect.shape or np.abs(A2 @ B2 - expect).max() > 1e-3


# ---------------------------------------------------------------------------
# Zoom budget cap (SeKV blog 2.3, paragraph under Eq. (9)): keep the passing
# spans in descending alpha~ order up to the budget.
def test_budget_cap_worked_example():
    # logits [0.5, 2.0, 1.0, 2.0, -1.0], theta 0: spans 0..3 pass. Descending alpha~
    # (equivalently descending l): span 1 and span 3 (equal, lower index first), then
    # span 2, then span 0.
    ell = [0.5, 2.0, 1.0, 2.0, -1.0]
    assert np.flatnonzero(O.zoom_decisions(ell, 0.0, budget=1)).tolist() == [1]
    assert np.flatnonzero(O.zoom_decisions(ell, 0.0, budget=2)).tolist() == [1, 3]
    assert np.flatnonzero(O.zoom_decisions(ell, 0.0, budget=3)).tolist() == [1, 2, 3]
    assert np.flatnonzero(O.zoom_decisions(ell, 0.0, budget=4)).tolist() == [0, 1, 2, 3]
    assert np.flatnonzero(O.zoom_decisions(ell, 0.0, budget=9)).tolist() == [0, 1, 2, 3]
    assert not O.zoom_decisions(ell, 0.0, budget=0).any()
    # the cap never adds a span the threshold rejected
    assert np.flatnonzero(O.zoom_decisions(ell, 1.5, budget=3)).tolist() == [1, 3]


def test_budget_cap_is_top_k_of_the_passing_set_brute_force():
    """Against the definition: the kept set is the unique size-min(k, #pass) subset of
    the passing spans such that no dropped passing span ranks before a kept one in
    (descending logit, ascending index) order; checked by enumerating subsets."""
    import itertools
    rng = np.random.default_rng(11)
    for trial in range(200):
        m = int(rng.integers(1, 8))
        # few distinct values so that ties are common
        ell = rng.integers(-3, 4, size=m).astype(np.float64) / 2.0
        theta = float(rng.choice([-10.0, -0.5, 0.0, 0.75]))
        k = int(rng.integers(0, m + 2))
        got = O.zoom_decisions(ell, theta, budget=k)
        passing = [s for s in range(m) if ell[s] > theta]
        want = None
        for sub in itertools.combinations(passing, min(k, len(passing))):
            dropped = [t for t in passing if t not in sub]
            ok = all((ell[s] > ell[t]) or (ell[s] == ell[t] and s < t) for s in sub for t in dropped)
            if ok:
                assert want is None, "the kept set must be unique"
                want = set(sub)
        assert want is not None
        assert set(np.flatnonzero(got).tolist()) == want


def test_budget_cap_none_is_the_threshold_rule():
    rng = np.random.default_rng(5)
    ell = rng.standard_normal(300)
    for theta in (-1.0, 0.0, 0.7):
        z = O.zoom_decisions(ell, theta)
        np.testing.assert_array_equal(O.zoom_decisions(ell, theta, budget=None), z)
        np.testing.assert_array_equal(O.zoom_decisions(ell, theta, budget=int(z.sum())), z)
        capped = O.zoom_decisions(ell, theta, budget=7)
        assert capped.sum() == min(7, z.sum()) and not (capped & ~z).any()
        # the kept logits are the 7 largest passing ones
        np.testing.assert_allclose(np.sort(ell[capped]), np.sort(ell[z])[-7:])


# ---------------------------------------------------------------------------
# Learned-form routing (SeKV blog 2.2 Eq. (3), 2.3 Eq. (5)) and the rank gate
# (SeKV blog 2.2 Eq. (6))
# ---------------------------------------------------------------------------
def _pin_learned_hand_example():
    g = _gold("learned_routing_example.json")
    Kb = O.routing_summary(g["K"], g["w"], g["W"])
    np.testing.assert_allclose(Kb, np.array(g["y"]) / math.sqrt(g["y_norm_sq"]), rtol=0, atol=1e-15)
    ell = O.learned_routing_logits(g["q"], g["W"], Kb[None, :], np.array([math.log(g["len"])]))
    expect = g["qW_dot_y"] / math.sqrt(g["y_norm_sq"]) / math.sqrt(3) + math.log(g["len"])
    assert ell[0] == pytest.approx(expect, abs=1e-14)


def test_learned_routing_hand_example():
    _pin_learned_hand_example()


def test_identity_projection_is_the_degenerate_form():
    """W = I (d' = d): Eq. (3) is kbar / ||kbar|| and Eq. (5) is the identity-form
    routing logit with scale 1/sqrt(d) (pinned by its own hand example)."""
    rng = np.random.default_rng(21)
    d = 16
    K = rng.normal(size=(9, d))
    w = rng.uniform(0.1, 2.0, size=9)
    kbar = (w[:, None] * K).sum(0) / w.sum()               # weighted mean, written out
    Kb = O.routing_summary(K, w, np.eye(d))
    np.testing.assert_allclose(Kb, kbar / np.linalg.norm(kbar), atol=1e-14)
    q = rng.normal(size=d)
    logS = np.array([math.log(9)])
    ell = O.learned_routing_logits(q, np.eye(d), Kb[None, :], logS)
    ref = O.routing_logits(q, kbar[None, :], np.array([1 / np.linalg.norm(kbar)]), logS, 1 / math.sqrt(d))
    assert ell[0] == pytest.approx(ref[0], abs=1e-13)


def test_routing_summary_invariances():
    rng = np.random.default_rng(22)
    d, dr = 12, 5
    K = rng.normal(size=(7, d))
    w = rng.uniform(0.1, 1.0, size=7)
    W = rng.normal(size=(dr, d))
    Kb = O.routing_summary(K, w, W)
    assert np.linalg.norm(Kb) == pytest.approx(1.0, abs=1e-14)
    # positive scalings of W or of the weights cancel in the normalisation
    np.testing.assert_allclose(O.routing_summary(K, w, 3.5 * W), Kb, atol=1e-14)
    np.testing.assert_allclose(O.routing_summary(K, 0.2 * w, W), Kb, atol=1e-14)
    # a rotation of the routing space rotates the summary and leaves the logit unchanged
    Q = _orth(rng, dr, dr)
    np.testing.assert_allclose(O.routing_summary(K, w, Q @ W), Q @ Kb, atol=1e-13)
    q = rng.normal(size=d)
    l1 = O.learned_routing_logits(q, W, Kb[None, :], np.array([0.7]))
    l2 = O.learned_routing_logits(q, Q @ W, (Q @ Kb)[None, :], np.array([0.7]))
    assert l1[0] == pytest.approx(l2[0], abs=1e-13)
    # a one-token span: the normalised projection of its key
    np.testing.assert_allclose(O.routing_summary(K[:1], [2.0], W), W @ K[0] / np.linalg.norm(W @ K[0]),
                               atol=1e-14)


def test_zero_projection_leaves_the_size_prior():
    rng = np.random.default_rng(23)
    K = rng.normal(size=(4, 8))
    Kb = O.routing_summary(K, np.ones(4), np.zeros((3, 8)))
    assert (Kb == 0).all()
    ell = O.learned_routing_logits(rng.normal(size=8), np.zeros((3, 8)), Kb[None, :], np.array([math.log(4)]))
    assert ell[0] == pytest.approx(math.log(4), abs=1e-15)


def _pin_rank_gate_known_components(ns, d):
    """Eq. (6) on a matrix of known singular structure: the gated reconstruction is
    sum_i m_i sigma_i u_i v_i^T over the top r components, in descending order."""
    rng = np.random.default_rng(ns * 7 + d)
    k = min(ns, d)
    U, V = _orth(rng, ns, k), _orth(rng, d, k)
    s = np.linspace(9.0, 1.0, k) ** 1.3
    X = (U * s) @ V.T
    r = 5
    m = np.array([1.0, 0.0, 0.25, 0.9, 0.5])
    A, B = O.truncated_basis(X, r, "f64", gate=m)
    expect = (U[:, :r] * (m * s[:r])) @ V[:, :r].T
    np.testing.assert_allclose(A @ B, expect, rtol=0, atol=1e-10 * s[0])
    A1, B1 = O.truncated_basis(X, r, "f64", gate=np.ones(r))
    A0, B0 = O.truncated_basis(X, r, "f64")
    np.testing.assert_allclose(A1 @ B1, A0 @ B0, atol=1e-12 * s[0])
    Az, Bz = O.truncated_basis(X, r, "f64", gate=np.zeros(r))
    assert np.abs(Az @ Bz).max() == 0.0


@pytest.mark.parametrize("ns,d", [(12, 20), (20, 12)])
def test_rank_gate_scales_known_components(ns, d):
    _pin_rank_gate_known_components(ns, d)


def test_rank_gate_prefix_meets_eckart_young():
    rng = np.random.default_rng(31)
    X = rng.normal(size=(24, 16))
    lam = np.sort(np.linalg.eigvalsh(X.T @ X))[::-1]      # sigma_i^2 from another routine
    for k in (1, 3, 6):
        gate = np.r_[np.ones(k), np.zeros(8 - k)]
        A, B = O.truncated_basis(X, 8, "f64", gate=gate)
        assert np.sum((X - A @ B) ** 2) == pytest.approx(np.sum(lam[k:]), rel=1e-9)


def test_planted_learned_routing_mistakes_are_caught(monkeypatch):
    """Plausible misreadings of Eq. (3) / (5), planted in the oracle, fail the hand pin."""
    real_sum, real_logits = O.routing_summary, O.learned_routing_logits

    def per_token_normalised(Ks, w, W):            # normalises each projected key first
        P = np.asarray(Ks, float) @ np.asarray(W, float).T
        P = P / np.linalg.norm(P, axis=1, keepdims=True)
        y = (np.asarray(w, float)[:, None] * P).sum(0)
        return y / np.linalg.norm(y)

    def unweighted(Ks, w, W):                      # drops the span weights
        return real_sum(Ks, np.ones(len(w)), W)

    def key_dim_scale(qh, W, kbar_r, logS):         # 1/sqrt(d) instead of 1/sqrt(d')
        d, dr = np.asarray(W).shape[1], np.asarray(W).shape[0]
        return (real_logits(qh, W, kbar_r, logS) - np.asarray(logS)) * math.sqrt(dr) / math.sqrt(d) + logS

    for name, bad in (("routing_summary", per_token_normalised), ("routing_summary", unweighted),
                      ("learned_routing_logits", key_dim_scale)):
        monkeypatch.setattr(O, name, bad)
        with pytest.raises(AssertionError):
            _pin_learned_hand_example()
        monkeypatch.undo()
    _pin_learned_hand_example()


def test_planted_reversed_rank_gate_is_caught(monkeypatch):
    """A gate applied in ascending singular-value order fails the Eq. (6) pin."""
    real = O.truncated_basis

    def reversed_gate(X, r, dtype, gate=None):
        return real(X, r, dtype, None if gate is None else np.asarray(gate)[:min(r, *np.shape(X))][::-1])
    monkeypatch.setattr(O, "truncated_basis", reversed_gate)
    with pytest.raises(AssertionError):
        _pin_rank_gate_known_components(12, 20)
    monkeypatch.undo()
    _pin_rank_gate_known_components(12, 20)


# ---------------------------------------------------------------------------
# Per-head routing summaries of a key head's spans (SeKV blog 2.2 Eq. (2), (3)):
# each query head uses its own W, each span its own weights
# ---------------------------------------------------------------------------
def _pin_routing_summaries():
    g = _gold("routing_summaries_example.json")
    seg = O.segment(g["H"], 1.0, 0)
    assert seg.spans.tolist() == g["spans"] and seg.anchor_pos.tolist() == g["anchors"]
    out = O.routing_summaries(g["K"], g["H"], seg, "surprisal", g["W"], "f64")
    assert out.shape == (2, 2, 3)
    for h in range(2):
        for s in range(2):
            expect = np.array(g["direction"][h][s]) / math.sqrt(g["norm_sq"][h][s])
            np.testing.assert_allclose(out[h, s], expect, rtol=0, atol=1e-15)


def test_routing_summaries_hand_example():
    _pin_routing_summaries()


def test_planted_routing_summaries_mistakes_are_caught(monkeypatch):
    """A swapped head index, or a span read one token too far (into the anchor that
    follows it), planted in the oracle, fails the hand pin."""
    real = O.routing_summaries

    def swapped_heads(K, H, seg, wmode, W_heads, dtype):
        return real(K, H, seg, wmode, np.asarray(W_heads)[::-1], dtype)

    def span_plus_one(K, H, seg, wmode, W_heads, dtype):
        W_heads = np.asarray(W_heads, dtype=np.float64)
        out = np.zeros((W_heads.shape[0], len(seg.spans), W_heads.shape[1]))
        for i, (b, e) in enumerate(seg.spans):
            w = O.span_weights(np.asarray(H, float)[b:e + 1], wmode)
            for h in range(W_heads.shape[0]):
                out[h, i] = O.routing_summary(np.asarray(K, float)[b:e + 1], w, W_heads[h])
        return out

    for bad in (swapped_heads, span_plus_one):
        monkeypatch.setattr(O, "routing_summaries", bad)
        with pytest.raises(AssertionError):
            _pin_routing_summaries()
        monkeypatch.undo()
    _pin_routing_summaries()


# ---------------------------------------------------------------------------
# Rank gates routed per span and per side (SeKV blog 2.2 Eq. (6)): gates[S][0]
# scales the key truncation of span S, gates[S][1] its value truncation
# ---------------------------------------------------------------------------
def _known_matrix(rng, ns, d, top):
    k = min(ns, d)
    U, V = _orth(rng, ns, k), _orth(rng, d, k)
    s = np.linspace(top, 1.0, k)
    return U, s, V, (U * s) @ V.T


def _pin_span_bases_gates():
    rng = np.random.default_rng(41)
    d, r = 10, 4
    lens = (6, 14)                         # one span shorter than d, one longer
    spans = [(0, lens[0]), (lens[0] + 1, lens[0] + 1 + lens[1])]
    n = spans[1][1]
    K = rng.normal(size=(n, d))            # the anchor row between the spans is noise
    V = rng.normal(size=(n, d))
    known = []
    for (b, e), top in zip(spans, (9.0, 7.0)):
        kk = _known_matrix(rng, e - b, d, top)
        vv = _known_matrix(rng, e - b, d, top + 3.0)
        K[b:e], V[b:e] = kk[3], vv[3]
        known.append((kk, vv))
    anchor = np.zeros(n, bool)
    anchor[lens[0]] = True
    seg = O.Segmentation(0.0, 0.0, 0.0, anchor, np.array([lens[0]]), np.array(spans))
    gates = np.array([[[1.0, 0.0, 0.5, 0.25], [0.75, 1.0, 0.0, 0.5]],
                      [[0.0, 0.5, 1.0, 1.0], [1.0, 0.25, 0.75, 0.0]]])
    out = O.span_bases(K, V, seg, r, "f64", gates)
    for i, ((Uk, sk, Vk, _), (Uv, sv, Vv, _)) in enumerate(known):
        A, B, C, D = out[i]
        # sum_j m_j sigma_j u_j v_j^T over the top r components, written from the construction
        np.testing.assert_allclose(A @ B, (Uk[:, :r] * (gates[i, 0] * sk[:r])) @ Vk[:, :r].T, rtol=0, atol=1e-10)
        np.testing.assert_allclose(C @ D, (Uv[:, :r] * (gates[i, 1] * sv[:r])) @ Vv[:, :r].T, rtol=0, atol=1e-10)


def test_span_bases_route_key_and_value_gates():
    _pin_span_bases_gates()


def test_planted_span_bases_gate_mistakes_are_caught(monkeypatch):
    """Key and value gates swapped, or the first span's gates used for every span,
    planted in the oracle, fail the pin."""
    real = O.span_bases

    def swapped_sides(K, V, seg, r, dtype, gates=None):
        return real(K, V, seg, r, dtype, None if gates is None else np.asarray(gates)[:, ::-1])

    def first_span_only(K, V, seg, r, dtype, gates=None):
        g = None if gates is None else np.repeat(np.asarray(gates)[:1], len(seg.spans), axis=0)
        return real(K, V, seg, r, dtype, g)

    for bad in (swapped_sides, first_span_only):
        monkeypatch.setattr(O, "span_bases", bad)
        with pytest.raises(AssertionError):
            _pin_span_bases_gates()
        monkeypatch.undo()
    _pin_span_bases_gates()
