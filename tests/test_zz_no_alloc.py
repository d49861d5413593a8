"""sekv_decode_attn_static: the decode entry point for callers that cannot
allocate device memory on the decode path (a serving loop inside a memory pool it
does not own, a plugin whose host framework forbids allocations after start-up,
code that must not call cudaMalloc because it can synchronize the device).

It must give the same result as sekv_decode_attn with a caller workspace, bit for
bit, on every call: the static scratch array keeps the previous call's contents,
so the check runs calls in a row with different inputs. This file is collected
last so that a failure here stops a `-x` run only after every other test has run;
it also passes on its own in a fresh process.
"""
import math

import pytest
import torch

from sekv_synth import WORKLOADS, gen

pytestmark = pytest.mark.gpu


def _lib():
    import hierarchical_kv_cache_span_b200 as P
    return P


def _built_cache(wl):
    P = _lib()
    H, spikes = gen.surprisal(wl)
    K, V = gen.keys_values(wl, spikes)
    a_cap = min(wl.n, wl.n // 4 + wl.window + 64)
    m_cap = ((min(wl.n, wl.n // 4 + 64) + 31) // 32) * 32
    c = P.SpanCache(wl.B, wl.L, wl.Hq, wl.Hkv, wl.n, wl.d, wl.dtype, a_cap, m_cap, wl.rank)
    c.build(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    return c


def _static_call(c, q, theta, zm, budget=0):
    P = _lib()
    S = P.sekv
    O, lse = c.new_outputs()
    O.fill_(float("nan"))
    lse.fill_(float("nan"))
    d = c.decode_desc(q, theta, O=O, lse=lse, zmask=zm, budget=budget)
    d.workspace, d.workspace_bytes = None, 0          # the static entry point needs none
    S.check(S.sekv_decode_attn_static(d, torch.cuda.current_stream().cuda_stream), "sekv_decode_attn_static")
    return O, lse


def _workspace_call(c, q, theta, zm, budget=0):
    return c.decode(q, theta, zmask=zm, budget=budget)


def _draws(wl):
    """two (query, threshold) pairs with different zoom sets: the first zooms a
    good share of the spans, the second almost none, so the two calls write
    different split-K partials into the same static array"""
    q1 = gen.queries(wl).cuda()
    g = torch.Generator().manual_seed(gen.unit_seed(wl.seed, 7, 0, 0, 1))
    q2 = torch.randn(q1.shape, generator=g).to(q1.dtype).cuda()
    th1 = torch.full((wl.L, wl.Hq), 3.5, dtype=torch.float32, device="cuda")
    th2 = torch.full((wl.L, wl.Hq), 5.5, dtype=torch.float32, device="cuda")
    return (q1, th1), (q2, th2)


@pytest.mark.parametrize("budget", [0, 3])
def test_static_scratch_decode_matches_workspace_decode(budget):
    """Two static calls in a row with different inputs; each must equal the
    workspace decode of the same inputs bit for bit (same kernels, same split plan),
    so partials left in the static array by the earlier call cannot leak into a
    later result. With a budget and no route_logits buffer, the routing logits of
    the cap live in the static array too."""
    wl = WORKLOADS["c2"].scaled(n=4096, L=2)
    c = _built_cache(wl)
    draws = _draws(wl)
    refs = []
    for q, th in draws:
        zm = c.new_zmask()
        O, lse = _workspace_call(c, q, th, zm, budget)
        torch.cuda.synchronize()
        assert c.read_status() == 0
        refs.append((O, lse, zm))
    assert int(refs[0][2].ne(0).sum()) > int(refs[1][2].ne(0).sum())
    assert int(refs[0][2].ne(0).sum()) > 0
    if budget:
        assert not torch.equal(refs[0][2], _no_cap_mask(c, *draws[0]))   # the cap actually bites
    for rep in range(2):
        for (q, th), (O_ref, lse_ref, zm_ref) in zip(draws, refs):
            zm = c.new_zmask()
            O, lse = _static_call(c, q, th, zm, budget)
            torch.cuda.synchronize()
            assert c.read_status() == 0
            assert torch.equal(zm, zm_ref)
            assert torch.equal(O, O_ref), (O - O_ref).abs().max().item()
            assert torch.equal(lse, lse_ref), (lse - lse_ref).abs().max().item()


def _no_cap_mask(c, q, th):
    zm = c.new_zmask()
    c.decode(q, th, zmask=zm)
    torch.cuda.synchronize()
    return zm


def test_static_scratch_rejects_oversized_calls():
    """A call whose split-K partials exceed the static array is refused before
    any launch (the descriptor below is never dereferenced)."""
    P = _lib()
    S = P.sekv
    d = S.sekv_decode_desc()
    fake = 1 << 20                                        # aligned, never touched
    for f in ("q", "a_count", "m_count", "span_beg", "span_end", "logS", "blk_off", "Ka", "Va", "kbar",
              "vbar", "inv_norm", "theta", "arena", "O", "lse", "dev_status"):
        setattr(d, f, fake)
    d.B, d.L, d.Hq, d.Hkv, d.d, d.dtype = 64, 32, 32, 8, 128, S.SEKV_BF16
    d.l0, d.l1, d.a_cap, d.m_cap, d.rank, d.phase, d.nsplit = 0, 32, 4096, 4096, 16, S.SEKV_FUSED, 16
    d.region_elems, d.scale = 1 << 20, 1.0 / math.sqrt(128)
    assert S.sekv_decode_workspace_bytes(d) > S.SEKV_STATIC_SCRATCH_BYTES
    assert S.sekv_decode_attn_static(d, 0) == S.SEKV_ERR_CAPACITY
    assert "static array" in S.sekv_last_error()
