"""ctypes binding of ``include/sekv.h`` (argument marshalling only).

Every function here forwards to the C ABI of ``libsekv.so`` with the same
name; the descriptor classes mirror the C structs field by field. Nothing in
this module computes any step of the method. Importing it fails loudly when
the library has not been built: there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# the in-tree build; SEKV_LIBRARY may point at another build of the same ABI
LIB_PATH = os.environ.get("SEKV_LIBRARY") or os.path.join(_HERE, "libsekv.so")

SEKV_OK = 0
SEKV_ERR_INVALID_ARG = 1
SEKV_ERR_CAPACITY = 2
SEKV_ERR_CUDA = 3
SEKV_ERR_COLD_SPAN = 4
SEKV_ERR_TIMEOUT = 5
SEKV_ERR_UNSUPPORTED = 6
SEKV_WARN_NOT_CONVERGED = 7

SEKV_F32 = 0
SEKV_BF16 = 1
SEKV_W_UNIFORM, SEKV_W_SURPRISAL, SEKV_W_SOFTMAX = 0, 1, 2
SEKV_BUILD_SCAN, SEKV_BUILD_LAYOUT, SEKV_BUILD_SUMMARY, SEKV_BUILD_BASES = 1, 2, 4, 8
SEKV_BUILD_ALL = 15
SEKV_FUSED, SEKV_ROUTE, SEKV_ATTEND = 0, 1, 2

_p = C.c_void_p
_i32 = C.c_int32
_i64 = C.c_int64


class sekv_build_desc(C.Structure):
    _fields_ = [
        ("H", _p), ("K", _p), ("V", _p),
        ("a_count", _p), ("m_count", _p), ("anchor_pos", _p), ("span_beg", _p), ("span_end", _p),
        ("logS", _p), ("blk_off", _p), ("stats", _p),
        ("Ka", _p), ("Va", _p), ("kbar", _p), ("vbar", _p), ("inv_norm", _p),
        ("basis_home", _p), ("dev_status", _p), ("workspace", _p),
        ("route_W", _p), ("kbar_r", _p), ("rank_gate", _p),
        ("region_elems", _i64), ("workspace_bytes", _i64), ("alpha", C.c_double),
        ("B", _i32), ("L", _i32), ("Hkv", _i32), ("n", _i32), ("d", _i32), ("dtype", _i32),
        ("l0", _i32), ("l1", _i32), ("a_cap", _i32), ("m_cap", _i32), ("window", _i32),
        ("wmode", _i32), ("rank", _i32), ("max_sweeps", _i32), ("steps", _i32), ("Hq", _i32),
        ("dr", _i32), ("reserved", _i32),
    ]


class sekv_decode_desc(C.Structure):
    _fields_ = [
        ("q", _p), ("a_count", _p), ("m_count", _p), ("span_beg", _p), ("span_end", _p),
        ("logS", _p), ("blk_off", _p), ("Ka", _p), ("Va", _p), ("kbar", _p), ("vbar", _p),
        ("inv_norm", _p), ("theta", _p), ("arena", _p), ("slot", _p), ("O", _p), ("lse", _p),
        ("zmask", _p), ("route_logits", _p), ("route_W", _p), ("kbar_r", _p), ("dev_status", _p),
        ("workspace", _p), ("arrive", _p),
        ("region_elems", _i64), ("workspace_bytes", _i64), ("scale", C.c_float),
        ("B", _i32), ("L", _i32), ("Hq", _i32), ("Hkv", _i32), ("d", _i32), ("dtype", _i32),
        ("l0", _i32), ("l1", _i32), ("a_cap", _i32), ("m_cap", _i32), ("rank", _i32),
        ("phase", _i32), ("nsplit", _i32), ("rows_hint", _i32), ("budget", _i32), ("zoom_hint", _i32),
        ("dr", _i32), ("test_flags", _i32), ("static_ready", _i32),
    ]


class sekv_fetch_desc(C.Structure):
    _fields_ = [
        ("zmask_dev", _p), ("zmask_host", _p), ("m_count_host", _p), ("blk_off_host", _p), ("blk_off_dev", _p),
        ("home", _p), ("arena", _p), ("slot_dev", _p), ("slot_host", _p), ("stats", _p),
        ("arena_used", _p), ("arena_top", _p), ("last_use", _p), ("route_done", _p),
        ("region_elems", _i64), ("arena_elems", _i64), ("step", _i64),
        ("B", _i32), ("L", _i32), ("Hq", _i32), ("Hkv", _i32), ("d", _i32), ("dtype", _i32),
        ("l0", _i32), ("l1", _i32), ("m_cap", _i32), ("rank", _i32), ("keep", _i32), ("reserved", _i32),
    ]


# every symbol include/sekv.h declares, with its ctypes signature
_SIGS = {
    "sekv_block_elems": (_i64, [_i32, _i32, _i32]),
    "sekv_basis_region_bound": (_i64, [_i32, _i32, _i32, _i32, _i32]),
    "sekv_build_workspace_bytes": (C.c_size_t, [C.POINTER(sekv_build_desc)]),
    "sekv_build_spans": (_i32, [C.POINTER(sekv_build_desc), _p]),
    "sekv_decode_workspace_bytes": (C.c_size_t, [C.POINTER(sekv_decode_desc)]),
    "sekv_decode_attn": (_i32, [C.POINTER(sekv_decode_desc), _p]),
    "sekv_decode_attn_static": (_i32, [C.POINTER(sekv_decode_desc), _p]),
    "sekv_fetch_bases": (_i32, [C.POINTER(sekv_fetch_desc), _p, _p, _p]),
    "sekv_merge_partials": (_i32, [_p, _p, _i32, _i64, _i32, _p, _p, _p]),
    "sekv_tau_to_theta": (_i32, [_p, _p, _i64]),
    "sekv_status_str": (C.c_char_p, [_i32]),
    "sekv_last_error": (C.c_char_p, []),
    "sekv_desc_size": (C.c_size_t, [_i32]),
    "sekv_version": (_i32, []),
}


def load_library(path: str = LIB_PATH) -> C.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"libsekv.so not found at {path}; build it with "
            "`python -m hierarchical_kv_cache_span_b200.build` (there is no fallback)")
    lib = C.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = load_library()
LIB = _lib


class SekvError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = int(status)
        msg = _lib.sekv_status_str(self.status).decode()
        detail = _lib.sekv_last_error().decode()
        super().__init__(f"{where}: {msg} ({self.status}){': ' + detail if detail else ''}")


def check(status: int, where: str = "sekv") -> int:
    if status != SEKV_OK:
        raise SekvError(status, where)
    return status


def sekv_block_elems(length: int, d: int, rank: int) -> int:
    return int(_lib.sekv_block_elems(length, d, rank))


def sekv_basis_region_bound(n: int, m_cap: int, Hkv: int, d: int, rank: int) -> int:
    return int(_lib.sekv_basis_region_bound(n, m_cap, Hkv, d, rank))


def sekv_build_workspace_bytes(desc: sekv_build_desc) -> int:
    return int(_lib.sekv_build_workspace_bytes(C.byref(desc)))


def sekv_build_spans(desc: sekv_build_desc, stream: int = 0) -> int:
    return int(_lib.sekv_build_spans(C.byref(desc), C.c_void_p(stream or None)))


def sekv_decode_workspace_bytes(desc: sekv_decode_desc) -> int:
    return int(_lib.sekv_decode_workspace_bytes(C.byref(desc)))


def sekv_decode_attn(desc: sekv_decode_desc, stream: int = 0) -> int:
    return int(_lib.sekv_decode_attn(C.byref(desc), C.c_void_p(stream or None)))


def sekv_decode_attn_static(desc: sekv_decode_desc, stream: int = 0) -> int:
    return int(_lib.sekv_decode_attn_static(C.byref(desc), C.c_void_p(stream or None)))


SEKV_STATIC_SCRATCH_BYTES = 8 << 20


def sekv_merge_partials(O_parts: int, lse_parts: int, nparts: int, rows: int, d: int, O: int, lse: int,
                        stream: int = 0) -> int:
    return int(_lib.sekv_merge_partials(C.c_void_p(O_parts), C.c_void_p(lse_parts), nparts, rows, d,
                                        C.c_void_p(O), C.c_void_p(lse), C.c_void_p(stream or None)))


def sekv_fetch_bases(desc: sekv_fetch_desc, compute: int, copy: int, done: int) -> int:
    return int(_lib.sekv_fetch_bases(C.byref(desc), C.c_void_p(compute or None),
                                     C.c_void_p(copy or None), C.c_void_p(done or None)))


def sekv_tau_to_theta(tau: int, theta: int, n: int) -> int:
    return int(_lib.sekv_tau_to_theta(C.c_void_p(tau), C.c_void_p(theta), n))


def sekv_status_str(status: int) -> str:
    return _lib.sekv_status_str(status).decode()


def sekv_last_error() -> str:
    return _lib.sekv_last_error().decode()


def sekv_desc_size(which: int) -> int:
    return int(_lib.sekv_desc_size(which))


def sekv_version() -> int:
    return int(_lib.sekv_version())
