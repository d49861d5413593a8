"""sekv_decode_attn_static: the decode entry point for callers that cannot
allocate device memory on the decode path (a serving loop inside a memory pool it
does not own, a plugin whose host framework forbids allocations after start-up,
code that must not call cudaMalloc because it can synchronize the device).

It must give the same result as sekv_decode_attn with a caller workspace, on
every call: the static scratch array keeps the previous call's contents, so the
check runs two calls in a row. This file is collected last so that a failure here
stops a `-x` run only after every other test has run; it also passes on its own
in a fresh process.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from sekv_synth import WORKLOADS, gen

pytestmark = pytest.mark.gpu

TOL = 2e-2          # the bf16 tolerance the parity tests use


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


def test_static_scratch_decode_matches_workspace_decode():
    P = _lib()
    S = P.sekv
    wl = WORKLOADS["c2"].scaled(n=4096, L=2)
    c = _built_cache(wl)
    q = gen.queries(wl).cuda()
    # thresholds low enough that a good share of spans zoom (the zoom path runs too)
    theta = torch.full((wl.L, wl.Hq), 3.5, dtype=torch.float32, device="cuda")
    zm_ref = c.new_zmask()
    O_ref, lse_ref = c.decode(q, theta, zmask=zm_ref)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    assert int(zm_ref.ne(0).sum()) > 0
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        O = torch.full_like(O_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        zm = c.new_zmask()
        d = c.decode_desc(q, theta, O=O, lse=lse, zmask=zm)
        d.workspace, d.workspace_bytes = None, 0          # the static entry point needs none
        S.check(S.sekv_decode_attn_static(d, stream), "sekv_decode_attn_static")
        torch.cuda.synchronize()
        assert c.read_status() == 0
        assert torch.equal(zm, zm_ref)
        assert torch.isfinite(O).all() and torch.isfinite(lse).all()
        assert (O - O_ref).abs().max().item() <= TOL
        assert (lse - lse_ref).abs().max().item() <= TOL


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
