"""Failure detection on the device: a bounded wait that runs out.

Every mbarrier wait of the decode kernels gives up after a poll limit and reports
SEKV_ERR_TIMEOUT in *dev_status instead of hanging or trapping. The test hook
(sekv_decode_desc.test_flags bit 0) makes the producer issue no copy at all and
shortens the limit, so the consumers' first waits run out with nothing in flight;
the call must return, the status must read SEKV_ERR_TIMEOUT, and a normal call on
the same stream afterwards must give the same result as before (bit for bit) and
match the oracle.
"""
import math

import numpy as np
import pytest
import torch

from sekv_synth import WORKLOADS, gen
from tests import helpers as T

pytestmark = pytest.mark.gpu


def _lib():
    import hierarchical_kv_cache_span_b200 as P
    return P


@pytest.mark.parametrize("phase", ["fused", "route"])
def test_starved_waits_report_timeout_and_the_context_stays_usable(phase):
    P = _lib()
    S = P.sekv
    wl = WORKLOADS["c2"].scaled(n=2048, L=2, Hq=8, Hkv=2)
    H, K, V = T.make_inputs(wl)
    a_cap, m_cap = T.caps(wl)
    c = P.SpanCache(wl.B, wl.L, wl.Hq, wl.Hkv, wl.n, wl.d, wl.dtype, a_cap, m_cap, wl.rank)
    c.build(H.cuda(), K.cuda(), V.cuda(), wl.alpha, wl.window, wl.wmode)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    G = wl.Hq // wl.Hkv
    scale = 1.0 / math.sqrt(wl.d)
    segs = T.oracle_segments(H, wl)
    units = T.oracle_units(K, V, H, segs, wl)
    q = gen.queries(wl)
    theta, q = T.thetas_with_margin(q, units, segs, wl, scale, G, quantile=0.9)
    th = torch.tensor(theta, dtype=torch.float32, device="cuda")
    qd = q.cuda()
    stream = torch.cuda.current_stream().cuda_stream

    zm0 = c.new_zmask()
    O0, lse0 = c.decode(qd, th, zmask=zm0)
    torch.cuda.synchronize()
    assert c.read_status() == 0

    # the starved call: returns, reports the timeout, writes empty results
    ph = S.SEKV_FUSED if phase == "fused" else S.SEKV_ROUTE
    O1, lse1 = c.new_outputs()
    O1.fill_(7.0)
    zm1 = c.new_zmask()
    d = c.decode_desc(qd, th, phase=ph, O=O1, lse=lse1, zmask=zm1)
    d.test_flags = 1
    S.check(S.sekv_decode_attn(d, stream), "starved decode")
    torch.cuda.synchronize()
    assert c.read_status() == S.SEKV_ERR_TIMEOUT
    assert S.sekv_status_str(c.read_status()) == "bounded device wait ran out"
    if ph == S.SEKV_FUSED:
        assert (O1 == 0).all() and torch.isneginf(lse1).all()
    assert int(zm1.ne(0).sum()) == 0

    # the context is still usable: the same normal call gives the same bits
    c.clear_status()
    zm2 = c.new_zmask()
    O2, lse2 = c.decode(qd, th, zmask=zm2)
    torch.cuda.synchronize()
    assert c.read_status() == 0
    assert torch.equal(O2, O0) and torch.equal(lse2, lse0) and torch.equal(zm2, zm0)
    Oo, lo, zooms = T.oracle_decode(q, units, segs, theta, scale, G)
    for (b, l, h), z in zooms.items():
        np.testing.assert_array_equal(T.zmask_bits(zm2, b, l, h, len(segs[b].spans)), z)
    assert np.abs(T.f64(O2) - Oo).max() <= 2e-2
    assert np.abs(T.f64(lse2) - lo).max() <= 2e-2
