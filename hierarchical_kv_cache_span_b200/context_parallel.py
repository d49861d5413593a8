"""Context-parallel decode: one sequence's context split across ranks.

SeKV summary, workflow paragraph (Stage 2): the attention over anchors, coarse
span entries and reconstructed tokens of zoomed spans is ONE softmax over the
whole logit list. A partition of that list therefore recombines exactly: each
rank decodes the anchors and spans of its slice of the context into (O_r, lse_r)
and the parts merge by log-sum-exp (`sekv_merge_partials`) after an all-gather.

Exactness needs the same segmentation everywhere and no span cut in two:
  * every rank runs the boundary scan (SeKV blog 2.1) on the full surprisal row
    of the sequence (n floats, small), so mu and sigma are the global ones;
  * the cut between rank r-1 and r is the first token at or after r * n / world
    that starts an anchor or a span, so spans never straddle a cut.
Each rank then builds (layout, summaries, bases) only its own slice of K/V: the
memory for the context is divided by the number of ranks, which is the reason to
split the context at all beyond 128K.

The zoom decision of a span depends on that span alone, so it is the same as on
one GPU. A zoom budget (sekv_decode_desc.budget) is applied per rank here, not
across the whole context. Batch size 1 (each sequence has its own cuts).
"""
from __future__ import annotations

from typing import List, Optional, Tuple

import torch

from . import sekv as S
from .cache import SpanCache, _ptr, _stream


def shard_cuts(anchor_pos, span_beg, n: int, world: int) -> List[int]:
    """Token cuts 0 = t_0 <= t_1 <= ... <= t_world = n; rank r owns [t_r, t_r+1).
    Every token of a segmented sequence is an anchor or lies in a span, so the
    anchor positions and span starts are exactly the places a cut can go without
    splitting a span; t_r is the first of them at or after r * n / world."""
    starts = torch.unique(torch.cat([torch.as_tensor(anchor_pos, dtype=torch.int64).reshape(-1).cpu(),
                                     torch.as_tensor(span_beg, dtype=torch.int64).reshape(-1).cpu()]))
    cuts = [0]
    for r in range(1, world):
        target = (r * n) // world
        i = int(torch.searchsorted(starts, torch.tensor(target, dtype=torch.int64), right=False))
        c = int(starts[i]) if i < starts.numel() else n
        cuts.append(max(c, cuts[-1]))
    cuts.append(n)
    return cuts


def shard_segmentation(anchor_pos, span_beg, span_end, t0: int, t1: int):
    """The anchors and spans of [t0, t1), as int64 CPU tensors of positions relative to t0."""
    ap = torch.as_tensor(anchor_pos, dtype=torch.int64).reshape(-1).cpu()
    sb = torch.as_tensor(span_beg, dtype=torch.int64).reshape(-1).cpu()
    se = torch.as_tensor(span_end, dtype=torch.int64).reshape(-1).cpu()
    a = ap[(ap >= t0) & (ap < t1)] - t0
    keep = (sb >= t0) & (sb < t1)
    if bool((se[keep] > t1).any()):
        raise ValueError("a span crosses the shard end: cuts must come from shard_cuts")
    return a, sb[keep] - t0, se[keep] - t0


class ContextShard:
    """Rank `rank` of `world`: its slice of one sequence's context as a SpanCache.

    build() takes the full surprisal row (device, [1][n]) and this rank's K/V
    slice ([1][L][Hkv][t1 - t0][d], device); `cuts` gives the slice. Use
    plan() first to learn the cuts from the global segmentation."""

    def __init__(self, L, Hq, Hkv, n, d, dtype, a_cap, m_cap, rank_basis, rank: int, world: int,
                 device="cuda", route_W: Optional[torch.Tensor] = None):
        self.L, self.Hq, self.Hkv, self.n, self.d, self.dtype = L, Hq, Hkv, n, d, dtype
        self.a_cap, self.m_cap, self.r = a_cap, m_cap, rank_basis
        self.rank, self.world, self.device = rank, world, torch.device(device)
        self.route_W = route_W          # learned-form routing projections, the same on every rank
        self.cuts = None
        self.cache = None
        self._seg = None

    def plan(self, H_full: torch.Tensor, alpha: float, window: int) -> List[int]:
        """Global boundary scan of the full row (the same on every rank) and the cuts."""
        scan = SpanCache(1, 1, self.Hq, self.Hkv, self.n, self.d, self.dtype, self.a_cap, self.m_cap, self.r,
                         home=None, device=self.device)
        scan.build(H_full, None, None, alpha, window, "uniform", steps=S.SEKV_BUILD_SCAN)
        torch.cuda.synchronize(self.device)
        st = scan.read_status()
        if st != 0:
            S.check(st, "context shard: scan")
        a, m = int(scan.a_count[0]), int(scan.m_count[0])
        ap = scan.anchor_pos[0, :a].cpu()
        sb = scan.span_beg[0, :m].cpu()
        se = scan.span_end[0, :m].cpu()
        self._seg = (ap, sb, se)
        self.cuts = shard_cuts(ap, sb, self.n, self.world)
        return self.cuts

    def span_range(self):
        """[k0, k1): the global indices of this rank's spans (spans are ordered by
        position, so a shard's spans are a contiguous run of them)."""
        t0, t1 = self.cuts[self.rank], self.cuts[self.rank + 1]
        sb = torch.as_tensor(self._seg[1], dtype=torch.int64).reshape(-1).cpu().contiguous()
        k0 = int(torch.searchsorted(sb, torch.tensor(t0, dtype=torch.int64)))
        k1 = int(torch.searchsorted(sb, torch.tensor(t1, dtype=torch.int64)))
        return k0, k1

    def shard_gate(self, rank_gate: torch.Tensor) -> torch.Tensor:
        """A global rank gate [1][L][Hkv][>= m][2][rank] cut to this shard's spans, in
        the shard cache's [1][L][Hkv][m_cap][2][rank] layout (zero past its spans)."""
        k0, k1 = self.span_range()
        out = torch.zeros(1, self.L, self.Hkv, self.m_cap, 2, self.r, dtype=torch.float32,
                          device=rank_gate.device)
        out[:, :, :, :k1 - k0] = rank_gate[:, :, :, k0:k1].to(torch.float32)
        return out

    def build(self, H_full: torch.Tensor, K_slice: torch.Tensor, V_slice: torch.Tensor, alpha: float,
              window: int, wmode: str, max_sweeps: int = 15, rank_gate: Optional[torch.Tensor] = None):
        """``rank_gate`` is the sequence's global gate tensor (indexed by global span)."""
        if self.cuts is None:
            self.plan(H_full, alpha, window)
        t0, t1 = self.cuts[self.rank], self.cuts[self.rank + 1]
        ns = max(t1 - t0, 1)
        if K_slice.shape[3] != t1 - t0:
            raise ValueError(f"K slice has {K_slice.shape[3]} tokens, the shard owns {t1 - t0}")
        a, sb, se = shard_segmentation(*self._seg, t0, t1)
        if len(a) > self.a_cap or len(sb) > self.m_cap:
            raise ValueError(f"shard {self.rank}: {len(a)} anchors / {len(sb)} spans exceed the caps "
                             f"{self.a_cap} / {self.m_cap}")
        c = SpanCache(1, self.L, self.Hq, self.Hkv, ns, self.d, self.dtype, self.a_cap, self.m_cap, self.r,
                      home=None, device=self.device)
        if self.route_W is not None:
            c.set_routing(self.route_W)
        c.a_count[0], c.m_count[0] = len(a), len(sb)
        if len(a):
            c.anchor_pos[0, :len(a)] = torch.as_tensor(a, dtype=torch.int32)
        if len(sb):
            c.span_beg[0, :len(sb)] = torch.as_tensor(sb, dtype=torch.int32)
            c.span_end[0, :len(sb)] = torch.as_tensor(se, dtype=torch.int32)
        H_slice = H_full[:, t0:t1].contiguous() if t1 > t0 else H_full[:, :1].contiguous()
        c.build(H_slice, None, None, alpha, window, wmode, steps=S.SEKV_BUILD_LAYOUT)
        torch.cuda.synchronize(self.device)
        c.alloc_home("device", c.exact_region())
        if t1 > t0:
            gate = None if rank_gate is None else self.shard_gate(rank_gate).to(self.device)
            c.build(H_slice, K_slice, V_slice, alpha, window, wmode, max_sweeps=max_sweeps,
                    steps=S.SEKV_BUILD_SUMMARY | S.SEKV_BUILD_BASES, rank_gate=gate)
        self.cache = c
        return self

    def decode(self, q: torch.Tensor, theta: torch.Tensor, **kw) -> Tuple[torch.Tensor, torch.Tensor]:
        """This rank's part: (O_r, lse_r) over its anchors and spans."""
        O, lse = self.cache.new_outputs()
        self.cache.decode(q, theta, O=O, lse=lse, **kw)
        return O, lse


def merge_parts(O_parts: torch.Tensor, lse_parts: torch.Tensor, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """O_parts [P][...][d], lse_parts [P][...] (fp32, device) -> the merged (O, lse)."""
    P = O_parts.shape[0]
    d = O_parts.shape[-1]
    rows = lse_parts[0].numel()
    O_parts = O_parts.contiguous()
    lse_parts = lse_parts.contiguous()
    O = torch.empty(O_parts.shape[1:], dtype=torch.float32, device=O_parts.device)
    lse = torch.empty(lse_parts.shape[1:], dtype=torch.float32, device=lse_parts.device)
    S.check(S.sekv_merge_partials(_ptr(O_parts), _ptr(lse_parts), P, rows, d, _ptr(O), _ptr(lse),
                                  _stream(stream)), "sekv_merge_partials")
    return O, lse


def context_parallel_decode(shard: ContextShard, q: torch.Tensor, theta: torch.Tensor, group=None, **kw):
    """Every rank decodes its shard, the parts are all-gathered and merged on the
    device; every rank returns the full (O, lse). With NCCL the gather runs on the
    device tensors; a host-side group (gloo) gathers host copies of them."""
    import torch.distributed as dist
    O_r, lse_r = shard.decode(q, theta, **kw)
    world = dist.get_world_size(group)
    on_host = dist.get_backend(group) == "gloo"
    dev = O_r.device
    src_O = O_r.contiguous().cpu() if on_host else O_r.contiguous()
    src_l = lse_r.contiguous().cpu() if on_host else lse_r.contiguous()
    O_all = torch.empty((world,) + tuple(O_r.shape), dtype=O_r.dtype, device=src_O.device)
    lse_all = torch.empty((world,) + tuple(lse_r.shape), dtype=lse_r.dtype, device=src_l.device)
    if on_host:
        dist.all_gather(list(O_all.unbind(0)), src_O, group=group)
        dist.all_gather(list(lse_all.unbind(0)), src_l, group=group)
    else:
        dist.all_gather_into_tensor(O_all, src_O, group=group)
        dist.all_gather_into_tensor(lse_all, src_l, group=group)
    return merge_parts(O_all.to(dev), lse_all.to(dev))
