"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, the ctypes descriptors match the C structs, and argument
validation rejects bad calls before any launch."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "sekv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sekv_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    from hierarchical_kv_cache_span_b200 import sekv as S
    names = _header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(S.LIB, n), n
        assert hasattr(S, n), f"binding lacks {n}"


def test_descriptor_layouts_match():
    from hierarchical_kv_cache_span_b200 import sekv as S
    for i, cls in enumerate([S.sekv_build_desc, S.sekv_decode_desc, S.sekv_fetch_desc]):
        assert ctypes.sizeof(cls) == S.sekv_desc_size(i)


def test_version_and_status_strings():
    from hierarchical_kv_cache_span_b200 import sekv as S
    assert S.sekv_version() == 1
    assert S.sekv_status_str(S.SEKV_ERR_COLD_SPAN).startswith("zoomed span")
    assert S.sekv_status_str(99) == "unknown status"


def test_block_layout_formula():
    from hierarchical_kv_cache_span_b200 import sekv as S
    # rS = min(r, |S|, d); A, C are len8 x r8; B, D are r8 x d (8x8-blocked, zero-padded)
    for ln, d, r in [(1, 128, 16), (5, 128, 16), (64, 128, 16), (300, 128, 32), (7, 64, 4), (13, 64, 12)]:
        rs = min(r, ln, d)
        r8 = -(-rs // 8) * 8
        l8 = -(-ln // 8) * 8
        want = 2 * l8 * r8 + 2 * r8 * d
        assert want % 64 == 0
        assert S.sekv_block_elems(ln, d, r) == want
    assert S.sekv_block_elems(0, 128, 16) == 0


def test_tiles8_order_is_the_documented_one():
    """Element (r, c) of a matrix of padded width w8 sits at
    ((r/8) * (w8/8) + c/8) * 64 + (r%8) * 8 + c%8 (the layout the header states)."""
    from tests.helpers import to_tiles8, from_tiles8
    rng = np.random.default_rng(3)
    M = rng.standard_normal((13, 20))
    flat = to_tiles8(M)
    assert flat.size == 16 * 24
    for r in range(13):
        for c in range(20):
            assert flat[((r // 8) * 3 + c // 8) * 64 + (r % 8) * 8 + c % 8] == M[r, c]
    assert np.array_equal(from_tiles8(flat, 13, 20), M)
    pad = np.ones(flat.size, dtype=bool)
    for r in range(13):
        for c in range(20):
            pad[((r // 8) * 3 + c // 8) * 64 + (r % 8) * 8 + c % 8] = False
    assert not flat[pad].any()


def test_region_bound_covers_worst_case():
    from hierarchical_kv_cache_span_b200 import sekv as S
    for n, m_cap, Hkv, d, r in [(1000, 512, 2, 64, 8), (1000, 1000, 1, 128, 16), (4096, 700, 8, 128, 12)]:
        bound = S.sekv_basis_region_bound(n, m_cap, Hkv, d, r)
        # any segmentation: spans of total length <= n, count <= m_cap
        cases = ([1] * min(m_cap, n), [2] * min(m_cap, n // 2), [n], [3] * min(m_cap, n // 3),
                 [9] * min(m_cap, n // 9), [r + 1] * min(m_cap, n // (r + 1)))
        for lens in cases:
            assert Hkv * sum(S.sekv_block_elems(x, d, r) for x in lens) <= bound


def test_invalid_build_arguments_are_rejected_before_launch():
    from hierarchical_kv_cache_span_b200 import sekv as S
    d = S.sekv_build_desc()
    assert S.sekv_build_spans(d, 0) == S.SEKV_ERR_INVALID_ARG
    d.B, d.L, d.Hkv, d.n, d.d, d.dtype, d.steps = 1, 1, 1, 16, 128, S.SEKV_BF16, S.SEKV_BUILD_SCAN
    d.a_cap, d.m_cap = 16, 30                        # m_cap not a multiple of 32
    assert S.sekv_build_spans(d, 0) == S.SEKV_ERR_INVALID_ARG
    assert "multiple of 32" in S.sekv_last_error()
    d.m_cap = 32
    assert S.sekv_build_spans(d, 0) == S.SEKV_ERR_INVALID_ARG   # no dev_status / buffers


def test_invalid_decode_arguments_are_rejected_before_launch():
    from hierarchical_kv_cache_span_b200 import sekv as S
    d = S.sekv_decode_desc()
    d.B, d.L, d.Hq, d.Hkv, d.d, d.dtype, d.l0, d.l1 = 1, 1, 12, 4, 128, S.SEKV_BF16, 0, 1
    d.a_cap, d.m_cap, d.rank = 32, 32, 16
    assert S.sekv_decode_attn(d, 0) == S.SEKV_ERR_UNSUPPORTED        # G = 3 not compiled
    d.Hq = 8
    d.rank = 65
    assert S.sekv_decode_attn(d, 0) == S.SEKV_ERR_UNSUPPORTED        # rank above 64
    d.rank = 16
    assert S.sekv_decode_attn(d, 0) == S.SEKV_ERR_INVALID_ARG        # pointers missing
    d.phase = 7
    assert S.sekv_decode_attn(d, 0) == S.SEKV_ERR_INVALID_ARG


def test_invalid_fetch_arguments_are_rejected():
    from hierarchical_kv_cache_span_b200 import sekv as S
    d = S.sekv_fetch_desc()
    assert S.sekv_fetch_bases(d, 0, 0, 0) == S.SEKV_ERR_INVALID_ARG


def test_product_path_has_no_oracle_or_cpu_fallback():
    pkg = os.path.join(ROOT, "hierarchical_kv_cache_span_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg, fn)).read()
            assert "oracle" not in src.replace("no oracle", ""), fn
            assert "import numpy" not in src, fn


def test_tau_to_theta_through_the_abi_matches_the_oracle():
    """sekv_tau_to_theta (SeKV blog 2.3, Eq. (9) in logit space) against the oracle's
    fp64 conversion rounded to fp32, including tau <= 0, tau >= 1 and interior values."""
    import torch
    import oracle as O
    from hierarchical_kv_cache_span_b200 import cache, sekv as S
    rng = np.random.default_rng(5)
    tau = np.r_[0.0, -0.3, 1.0, 1.7, 0.5, 1e-12, 1 - 1e-12, rng.uniform(0.3, 0.9, 61)]
    th = cache.tau_to_theta(torch.tensor(tau, dtype=torch.float64)).numpy()
    assert th.dtype == np.float32
    np.testing.assert_array_equal(th, O.tau_to_theta(tau).astype(np.float32))
    assert th[0] == -np.inf and th[1] == -np.inf and th[2] == np.inf and th[3] == np.inf and th[4] == 0.0
    # the shape of the table is kept ([L][Hq])
    t2 = torch.full((3, 4), 0.75, dtype=torch.float64)
    assert tuple(cache.tau_to_theta(t2).shape) == (3, 4)
    # NaN or null pointers: rejected before anything is written
    out = np.full(2, 7.0, np.float32)
    bad = np.array([0.5, np.nan])
    assert S.sekv_tau_to_theta(bad.ctypes.data, out.ctypes.data, 2) == S.SEKV_ERR_INVALID_ARG
    assert (out == 7.0).all()
    assert S.sekv_tau_to_theta(0, 0, 3) == S.SEKV_ERR_INVALID_ARG
    assert S.sekv_tau_to_theta(0, 0, 0) == S.SEKV_OK
