"""Buffer plumbing around the C ABI: torch owns the device / pinned memory, the
descriptors hand raw pointers to ``libsekv.so``. No step of the method runs here.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import sekv as S

_DT = {"f32": (torch.float32, S.SEKV_F32), "bf16": (torch.bfloat16, S.SEKV_BF16)}
_WMODE = {"uniform": S.SEKV_W_UNIFORM, "surprisal": S.SEKV_W_SURPRISAL, "softmax": S.SEKV_W_SOFTMAX}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def tau_to_theta(tau: torch.Tensor) -> torch.Tensor:
    """Zoom thresholds in logit space from tau (SeKV blog 2.3, Eq. (9)), computed by
    the library's ``sekv_tau_to_theta``: marshals tau as host fp64 and returns the
    host fp32 theta table of the same shape."""
    t = tau.detach().to("cpu", torch.float64).contiguous()
    th = torch.empty(t.shape, dtype=torch.float32)
    S.check(S.sekv_tau_to_theta(t.data_ptr(), th.data_ptr(), t.numel()), "sekv_tau_to_theta")
    return th


class SpanCache:
    """The span-structured KV cache of B sequences x L layers x Hkv kv heads.

    Device: segmentation (counts, anchor positions, span bounds, log|S|, basis
    block offsets), anchors Ka/Va, summaries kbar/vbar + 1/||kbar||. Bases live
    in ``home``: device memory (hot) or pinned host memory (cold). With
    ``set_routing(W)`` the summary step also writes per-query-head routing
    summaries ``kbar_r`` and decode routes with them; ``build(..., rank_gate=g)``
    folds a rank gate into the bases.
    """

    def __init__(self, B, L, Hq, Hkv, n, d, dtype, a_cap, m_cap, rank, home="device",
                 device="cuda"):
        if m_cap % 32:
            raise ValueError("m_cap must be a multiple of 32")
        self.B, self.L, self.Hq, self.Hkv, self.n, self.d = B, L, Hq, Hkv, n, d
        self.a_cap, self.m_cap, self.rank = a_cap, m_cap, rank
        self.dtype_name = dtype
        self.dt, self.code = _DT[dtype]
        self.device = torch.device(device)
        dev = self.device
        i32 = dict(dtype=torch.int32, device=dev)
        self.a_count = torch.zeros(B, **i32)
        self.m_count = torch.zeros(B, **i32)
        self.anchor_pos = torch.zeros(B, a_cap, **i32)
        self.span_beg = torch.zeros(B, m_cap, **i32)
        self.span_end = torch.zeros(B, m_cap, **i32)
        self.logS = torch.zeros(B, m_cap, dtype=torch.float32, device=dev)
        self.blk_off = torch.zeros(B, m_cap + 1, dtype=torch.int64, device=dev)
        self.stats = torch.zeros(B, 3, dtype=torch.float64, device=dev)
        self.Ka = torch.zeros(B, L, Hkv, a_cap, d, dtype=self.dt, device=dev)
        self.Va = torch.zeros_like(self.Ka)
        self.kbar = torch.zeros(B, L, Hkv, m_cap, d, dtype=self.dt, device=dev)
        self.vbar = torch.zeros_like(self.kbar)
        self.inv_norm = torch.zeros(B, L, Hkv, m_cap, dtype=torch.float32, device=dev)
        self.status = torch.zeros(1, **i32)
        self.home_kind = home
        self.home = None
        self.region = S.sekv_basis_region_bound(n, m_cap, Hkv, d, rank)
        if home is not None:
            self.alloc_home(home)
        self._bws = None
        self._dws = {}
        self.route_W = None      # learned-form routing projections [L][Hq][dr][d]
        self.kbar_r = None       # routing summaries [B][L][Hq][m_cap][dr]
        self.dr = 0
        self._zscratch = None
        self._arrive = None             # arrival counters of the in-kernel split merge

    def set_routing(self, W: Optional[torch.Tensor]):
        """Learned-form routing (SeKV blog 2.2 Eq. (3), 2.3 Eq. (5)): W [L][Hq][dr][d] in
        the storage dtype on the cache's device, dr 32 or 64; None returns to the
        identity form. The summaries are written by the next SUMMARY build step."""
        if W is None:
            self.route_W, self.kbar_r, self.dr = None, None, 0
            return self
        if tuple(W.shape[:2]) != (self.L, self.Hq) or W.shape[3] != self.d or W.dtype != self.dt:
            raise ValueError(f"W must be [{self.L}][{self.Hq}][dr][{self.d}] {self.dt}")
        self.route_W = W.to(self.device).contiguous()
        self.dr = int(W.shape[2])
        self.kbar_r = torch.zeros(self.B, self.L, self.Hq, self.m_cap, self.dr, dtype=self.dt, device=self.device)
        return self

    def alloc_home(self, kind: str, region: Optional[int] = None):
        """Allocate the basis home: ``kind`` 'device' (hot) or 'host' (pinned, cold).
        ``region`` (elements per (b, l)) defaults to the worst-case bound; after a
        SCAN+LAYOUT pass ``exact_region()`` gives the realised size."""
        if region is not None:
            self.region = int(region)
        self.home_kind = kind
        self.home = None
        if kind == "device":
            self.home = torch.zeros(self.B, self.L, self.region, dtype=self.dt, device=self.device)
        else:
            self.home = torch.empty(self.B, self.L, self.region, dtype=self.dt, pin_memory=True)
        return self.home

    def exact_region(self) -> int:
        """Elements per (b, l) region the realised segmentation needs (after LAYOUT)."""
        m = self.m_count.to("cpu").long()
        tot = self.blk_off.to("cpu").gather(1, m.view(-1, 1)).max().item()
        return max(64, int((tot + 63) // 64 * 64))

    # ------------------------------------------------------------------ build
    def build_desc(self, H, K, V, alpha, window, wmode, max_sweeps=15, steps=S.SEKV_BUILD_ALL,
                   l0=0, l1=None, rank_gate=None) -> S.sekv_build_desc:
        d = S.sekv_build_desc()
        d.H, d.K, d.V = _ptr(H), _ptr(K), _ptr(V)
        d.a_count, d.m_count, d.anchor_pos = _ptr(self.a_count), _ptr(self.m_count), _ptr(self.anchor_pos)
        d.span_beg, d.span_end, d.logS = _ptr(self.span_beg), _ptr(self.span_end), _ptr(self.logS)
        d.blk_off, d.stats = _ptr(self.blk_off), _ptr(self.stats)
        d.Ka, d.Va, d.kbar, d.vbar = _ptr(self.Ka), _ptr(self.Va), _ptr(self.kbar), _ptr(self.vbar)
        d.inv_norm, d.basis_home, d.dev_status = _ptr(self.inv_norm), _ptr(self.home), _ptr(self.status)
        d.region_elems = self.region
        d.alpha = float(alpha)
        d.B, d.L, d.Hkv, d.n, d.d, d.dtype = self.B, self.L, self.Hkv, self.n, self.d, self.code
        d.l0, d.l1 = l0, self.L if l1 is None else l1
        d.a_cap, d.m_cap, d.window = self.a_cap, self.m_cap, window
        d.wmode = _WMODE[wmode] if isinstance(wmode, str) else int(wmode)
        d.rank, d.max_sweeps, d.steps = self.rank, max_sweeps, steps
        d.route_W, d.kbar_r, d.Hq, d.dr = _ptr(self.route_W), _ptr(self.kbar_r), self.Hq, self.dr
        if rank_gate is not None:
            if tuple(rank_gate.shape) != (self.B, self.L, self.Hkv, self.m_cap, 2, self.rank) or \
                    rank_gate.dtype != torch.float32 or not rank_gate.is_contiguous():
                raise ValueError("rank_gate must be contiguous fp32 [B][L][Hkv][m_cap][2][rank]")
        d.rank_gate = _ptr(rank_gate)
        need = S.sekv_build_workspace_bytes(d)
        if need and (self._bws is None or self._bws.numel() < need):
            self._bws = torch.empty(need, dtype=torch.uint8, device=self.device)
        d.workspace = _ptr(self._bws) if need else None
        d.workspace_bytes = need
        return d

    def build(self, H, K, V, alpha, window, wmode, max_sweeps=15, steps=S.SEKV_BUILD_ALL, l0=0,
              l1=None, stream=None, rank_gate=None):
        d = self.build_desc(H, K, V, alpha, window, wmode, max_sweeps, steps, l0, l1, rank_gate)
        S.check(S.sekv_build_spans(d, _stream(stream)), "sekv_build_spans")
        if steps & S.SEKV_BUILD_SCAN:
            self._rows_hint = None          # re-read from the new counts at the next decode_desc
        return self

    @property
    def rows_hint(self) -> int:
        """Largest anchors + spans over the batch (one device read per build)."""
        if getattr(self, "_rows_hint", None) is None:
            self._rows_hint = int((self.a_count.clamp(max=self.a_cap) +
                                   self.m_count.clamp(max=self.m_cap)).max().item())
        return self._rows_hint

    # ------------------------------------------------------------------ decode
    def decode_desc(self, q, theta, phase=S.SEKV_FUSED, scale=None, O=None, lse=None, zmask=None,
                    route_logits=None, nsplit=0, slot=None, arena=None, l0=0, l1=None,
                    workspace=None, rows_hint=None, budget=0, zoom_hint=0,
                    static_ready=False) -> S.sekv_decode_desc:
        """static_ready=True promises that nothing still in flight on the stream writes
        the cache's build outputs (e.g. the stream was synchronised after build()), so
        the kernels may read the counts and their first tiles while the previous kernel
        finishes (sekv_decode_desc.static_ready)."""
        d = S.sekv_decode_desc()
        d.q = _ptr(q)
        d.a_count, d.m_count, d.span_beg, d.span_end = (_ptr(self.a_count), _ptr(self.m_count),
                                                        _ptr(self.span_beg), _ptr(self.span_end))
        d.logS, d.blk_off = _ptr(self.logS), _ptr(self.blk_off)
        d.Ka, d.Va, d.kbar, d.vbar = _ptr(self.Ka), _ptr(self.Va), _ptr(self.kbar), _ptr(self.vbar)
        d.inv_norm, d.theta = _ptr(self.inv_norm), _ptr(theta)
        if arena is None and self.home_kind == "device":
            arena = self.home
        d.arena, d.slot = _ptr(arena), _ptr(slot)
        if zmask is None and self.route_W is not None:
            # the learned routing pass hands its decisions to attention through a mask
            if self._zscratch is None:
                self._zscratch = self.new_zmask()
            zmask = self._zscratch
        d.O, d.lse, d.zmask, d.route_logits = _ptr(O), _ptr(lse), _ptr(zmask), _ptr(route_logits)
        d.route_W, d.kbar_r, d.dr = _ptr(self.route_W), _ptr(self.kbar_r), self.dr
        d.dev_status = _ptr(self.status)
        d.region_elems = self.region
        d.scale = float(1.0 / math.sqrt(self.d) if scale is None else scale)
        d.B, d.L, d.Hq, d.Hkv, d.d, d.dtype = self.B, self.L, self.Hq, self.Hkv, self.d, self.code
        d.l0, d.l1 = l0, self.L if l1 is None else l1
        d.a_cap, d.m_cap, d.rank, d.phase, d.nsplit = self.a_cap, self.m_cap, self.rank, phase, nsplit
        d.rows_hint = self.rows_hint if rows_hint is None else int(rows_hint)
        d.budget = int(budget)
        d.zoom_hint = int(zoom_hint)
        d.static_ready = 1 if static_ready else 0
        need = S.sekv_decode_workspace_bytes(d)
        if workspace is None:
            key = (d.l0, d.l1, nsplit, d.rows_hint, d.budget > 0 and phase != S.SEKV_ATTEND)
            ws = self._dws.get(key)
            if ws is None or ws.numel() < need:
                ws = torch.empty(max(need, 256), dtype=torch.uint8, device=self.device)
                self._dws[key] = ws
            workspace = ws
        d.workspace, d.workspace_bytes = _ptr(workspace), workspace.numel()
        if phase != S.SEKV_ROUTE:
            # arrival counters: the last CTA of each (b, l, kv head) merges the splits
            if self._arrive is None:
                self._arrive = torch.zeros(self.B * self.L * self.Hkv, dtype=torch.int32, device=self.device)
            d.arrive = _ptr(self._arrive)
        return d

    def new_outputs(self, l0=0, l1=None):
        L = self.L
        O = torch.zeros(self.B, L, self.Hq, self.d, dtype=torch.float32, device=self.device)
        lse = torch.zeros(self.B, L, self.Hq, dtype=torch.float32, device=self.device)
        return O, lse

    def new_zmask(self):
        return torch.zeros(self.B, self.L, self.Hq, self.m_cap // 32, dtype=torch.int32, device=self.device)

    def decode(self, q, theta, phase=S.SEKV_FUSED, O=None, lse=None, stream=None, **kw):
        if phase != S.SEKV_ROUTE and (O is None or lse is None):
            O, lse = self.new_outputs()
        d = self.decode_desc(q, theta, phase=phase, O=O, lse=lse, **kw)
        S.check(S.sekv_decode_attn(d, _stream(stream)), "sekv_decode_attn")
        return O, lse

    def read_status(self) -> int:
        return int(self.status.item())

    def clear_status(self):
        self.status.zero_()


class ColdFetcher:
    """Pinned mirrors, device arena and slot table for fetching cold bases.

    keep=False: every fetch refills the arena with the step's zoomed spans.
    keep=True: the arena is a device cache across fetches: resident spans are not
    copied again, misses go to free space, and the least recently used spans not
    needed by this step or the previous one are evicted when space runs out.
    ``step`` (keep mode) is the caller's decode-step counter; ``route_done`` (keep
    mode) an event recorded after the ROUTE call whose mask is fetched, so that the
    copies may overlap work queued after it (the previous layer's ATTEND)."""

    def __init__(self, cache: SpanCache, arena_elems: int, keep: bool = False):
        self.c = cache
        self.keep = bool(keep)
        self.arena_used = torch.zeros(1, dtype=torch.int64)
        self.arena_top = torch.zeros(1, dtype=torch.int64)     # keep mode: end of the highest entry
        B, L, Hq, m_cap = cache.B, cache.L, cache.Hq, cache.m_cap
        dev = cache.device
        self.arena = torch.zeros(max(arena_elems, 64), dtype=cache.dt, device=dev)
        self.slot_dev = torch.full((B, L, m_cap), -1, dtype=torch.int64, device=dev)
        self.slot_host = torch.full((B, L, m_cap), -1, dtype=torch.int64, pin_memory=True)
        self.last_use = torch.full((B, L, m_cap), -1, dtype=torch.int64)
        self.zmask_host = torch.zeros(B, L, Hq, m_cap // 32, dtype=torch.int32, pin_memory=True)
        self.m_count_host = cache.m_count.to("cpu")
        self.blk_off_host = cache.blk_off.to("cpu")
        self.stats = torch.zeros(5, dtype=torch.int64)
        self.copy_stream = torch.cuda.Stream(device=dev)
        self.done = torch.cuda.Event()
        self.done.record(self.copy_stream)

    def refresh_segmentation(self):
        self.m_count_host = self.c.m_count.to("cpu")
        self.blk_off_host = self.c.blk_off.to("cpu")

    def fetch(self, zmask: torch.Tensor, l0=0, l1=None, compute=None, step=0, route_done=None):
        c = self.c
        d = S.sekv_fetch_desc()
        d.zmask_dev, d.zmask_host = _ptr(zmask), _ptr(self.zmask_host)
        d.m_count_host, d.blk_off_host = _ptr(self.m_count_host), _ptr(self.blk_off_host)
        d.blk_off_dev = _ptr(c.blk_off)
        d.home, d.arena = _ptr(c.home), _ptr(self.arena)
        d.slot_dev, d.slot_host, d.stats = _ptr(self.slot_dev), _ptr(self.slot_host), _ptr(self.stats)
        d.arena_used, d.last_use = _ptr(self.arena_used), _ptr(self.last_use) if self.keep else None
        d.arena_top = _ptr(self.arena_top) if self.keep else None
        d.route_done = route_done.cuda_event if route_done is not None else None
        d.region_elems, d.arena_elems, d.step = c.region, self.arena.numel(), int(step)
        d.B, d.L, d.Hq, d.Hkv, d.d, d.dtype = c.B, c.L, c.Hq, c.Hkv, c.d, c.code
        d.l0, d.l1, d.m_cap, d.rank = l0, c.L if l1 is None else l1, c.m_cap, c.rank
        d.keep = int(self.keep)
        cs = _stream(compute)
        st = S.sekv_fetch_bases(d, cs, self.copy_stream.cuda_stream, self.done.cuda_event)
        S.check(st, "sekv_fetch_bases")
        return dict(bytes=int(self.stats[0]), spans=int(self.stats[1]), copies=int(self.stats[2]),
                    resident=int(self.stats[3]), evicted=int(self.stats[4]))
