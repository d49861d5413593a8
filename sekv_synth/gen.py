"""Seeded generators for the five SeKV workloads (surprisal, K/V, queries, thresholds).

The pages measure on LongBench / RULER / InfiniteBench / NIAH / GSM8K with
LLaMA-3-8B-class backbones (SeKV blog walkthrough, section 3.1). None of those
datasets or weights exist here, so these generators stand in for them and take
only the context lengths (32K / 128K) and the Llama-3-8B attention shape
(32 layers, 32 query heads, 8 KV heads, head_dim 128).

Recipes (all draws from torch generators seeded per (batch, layer, kind)):

* surprisal ``H[B][n]`` (float32): i.i.d. Gamma(2, 1) (drawn as -ln(U1 U2)),
  optionally truncated to [0, 3) by redrawing; at Bernoulli(1/64) "spike"
  positions an untruncated Gamma(2, 1) + 6 is drawn instead.
* keys / values ``[B][L][Hkv][n][d]``: the spikes cut the sequence into
  generator segments. A non-spike token t in segment j gets
  ``a_t @ F_j + noise`` with ``a_t ~ N(0, I_g)``, ``F_j ~ N(0, 1/g)`` (g x d)
  and ``noise ~ N(0, noise_std^2)``; spike tokens get ``N(0, I_d)`` rows.
  Keys and values are drawn independently.
* queries ``q[B][L][Hq][d]``: N(0, 1).
* thresholds ``tau[L][Hq]``: fixed, U(lo, hi), or left to calibration.

Nothing here computes a boundary, a weight, a summary, a basis, a routing
logit or an attention value.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional

import torch

_MASK64 = (1 << 64) - 1


def unit_seed(*parts: int) -> int:
    """Mix integers into a 63-bit seed (splitmix64 finaliser applied per part)."""
    x = 0x9E3779B97F4A7C15
    for p in parts:
        x = (x ^ (int(p) & _MASK64)) & _MASK64
        x = (x + 0x9E3779B97F4A7C15) & _MASK64
        z = x
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        x = z ^ (z >> 31)
    return x & ((1 << 63) - 1)


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    L: int
    Hq: int
    Hkv: int
    d: int
    n: int
    dtype: str           # "f32" or "bf16": storage type of K, V, q and every stored output
    alpha: float         # boundary sensitivity
    window: int          # local window kept at full resolution
    wmode: str           # "uniform" | "surprisal" | "softmax"
    rank: int            # basis rank r
    h_trunc: bool        # truncate the non-spike Gamma draws to [0, 3)
    kv_rank: int         # generator rank g of the per-segment K/V factors
    kv_noise: float      # std of the additive K/V noise
    tau_kind: str        # "fixed" | "uniform" | "quantile"
    tau_a: float         # fixed value, lower bound, or quantile
    tau_b: float = 0.0   # upper bound for "uniform"
    basis_home: str = "device"   # "device" (hot) or "host" (cold, pinned)
    spike_rate: float = 1.0 / 64.0
    spike_height: float = 6.0
    seed: int = 20260

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def describe(self) -> dict:
        return dataclasses.asdict(self)


_LLAMA = dict(L=32, Hq=32, Hkv=8, d=128, dtype="bf16", window=512, wmode="softmax")

WORKLOADS = {
    # tiny fp32 case the oracle finishes in seconds
    "c1": Workload("c1", B=1, L=1, Hq=4, Hkv=4, d=64, n=2048, dtype="f32", alpha=1.0,
                   window=0, wmode="uniform", rank=4, h_trunc=False, kv_rank=4,
                   kv_noise=0.1, tau_kind="fixed", tau_a=0.5, seed=20261),
    # Llama-3-8B-shaped decode at 32K, ~2% zoom
    "c2": Workload("c2", B=1, n=32768, alpha=1.5, rank=16, h_trunc=True, kv_rank=8,
                   kv_noise=0.05, tau_kind="quantile", tau_a=0.98, seed=20262, **_LLAMA),
    # 128K, cold bases in pinned host memory
    "c3": Workload("c3", B=1, n=131072, alpha=1.5, rank=16, h_trunc=True, kv_rank=8,
                   kv_noise=0.05, tau_kind="quantile", tau_a=0.98, basis_home="host",
                   seed=20263, **_LLAMA),
    # batch 8 x 32K, tau ~ U(0.3, 0.9) per (layer, head)
    "c4": Workload("c4", B=8, n=32768, alpha=1.5, rank=16, h_trunc=True, kv_rank=8,
                   kv_noise=0.05, tau_kind="uniform", tau_a=0.3, tau_b=0.9, seed=20264, **_LLAMA),
    # prefill build at rank 32 + 25% zoom at 128K
    "c5": Workload("c5", B=1, n=131072, alpha=1.5, rank=32, h_trunc=True, kv_rank=16,
                   kv_noise=0.05, tau_kind="quantile", tau_a=0.75, seed=20265, **_LLAMA),
}


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(unit_seed(*parts))
    return g


def _gamma2(shape, g, device) -> torch.Tensor:
    u1 = 1.0 - torch.rand(shape, generator=g, device=device, dtype=torch.float64)
    u2 = 1.0 - torch.rand(shape, generator=g, device=device, dtype=torch.float64)
    return -(torch.log(u1) + torch.log(u2))


def surprisal(wl: Workload, device="cpu", seed: Optional[int] = None):
    """Return (H [B][n] float32, spikes [B][n] bool) for ``wl``."""
    seed = wl.seed if seed is None else seed
    H = torch.empty(wl.B, wl.n, dtype=torch.float32, device=device)
    spikes = torch.empty(wl.B, wl.n, dtype=torch.bool, device=device)
    for b in range(wl.B):
        g = _gen(device, seed, 1, b)
        base = _gamma2((wl.n,), g, device)
        if wl.h_trunc:
            for _ in range(64):
                bad = base >= 3.0
                nb = int(bad.sum())
                if nb == 0:
                    break
                base[bad] = _gamma2((nb,), g, device)
            base = torch.where(base >= 3.0, torch.full_like(base, 2.5), base)
        sp = torch.rand((wl.n,), generator=g, device=device, dtype=torch.float64) < wl.spike_rate
        peak = _gamma2((wl.n,), g, device) + wl.spike_height
        H[b] = torch.where(sp, peak, base).to(torch.float32)
        spikes[b] = sp
    return H, spikes


def keys_values(wl: Workload, spikes: torch.Tensor, device="cpu", seed: Optional[int] = None,
                layers: Optional[range] = None, out=None):
    """Return (K, V), each [B][L'][Hkv][n][d] in the workload's storage dtype.

    ``layers`` selects a layer range (default: all); the draws of a layer do
    not depend on which other layers are generated.
    """
    seed = wl.seed if seed is None else seed
    layers = range(wl.L) if layers is None else layers
    dt = wl.torch_dtype()
    Lr = len(layers)
    if out is None:
        K = torch.empty(wl.B, Lr, wl.Hkv, wl.n, wl.d, dtype=dt, device=device)
        V = torch.empty_like(K)
    else:
        K, V = out
    g_rank = wl.kv_rank
    for b in range(wl.B):
        sp = spikes[b].to(device)
        seg = torch.cumsum(sp.to(torch.int64), 0)          # segment id per token
        nseg = int(seg[-1].item()) + 1
        for li, l in enumerate(layers):
            for which, dst in ((0, K), (1, V)):
                g = _gen(device, seed, 2, b, l, which)
                a = torch.randn(wl.Hkv, wl.n, g_rank, generator=g, device=device)
                f = torch.randn(wl.Hkv, nseg, g_rank, wl.d, generator=g, device=device)
                f.mul_(1.0 / (g_rank ** 0.5))
                x = torch.randn(wl.Hkv, wl.n, wl.d, generator=g, device=device)
                x.mul_(wl.kv_noise)
                for gi in range(g_rank):
                    x.add_(a[:, :, gi:gi + 1] * f[:, seg, gi, :])
                anchors_rows = torch.randn(wl.Hkv, wl.n, wl.d, generator=g, device=device)
                x = torch.where(sp.view(1, -1, 1), anchors_rows, x)
                dst[b, li].copy_(x.to(dt))
                del a, f, x, anchors_rows
    return K, V


def queries(wl: Workload, step: int = 0, device="cpu", seed: Optional[int] = None) -> torch.Tensor:
    """Return q [B][L][Hq][d] ~ N(0, 1) in the storage dtype for decode step ``step``."""
    seed = wl.seed if seed is None else seed
    g = _gen(device, seed, 3, step)
    q = torch.randn(wl.B, wl.L, wl.Hq, wl.d, generator=g, device=device)
    return q.to(wl.torch_dtype())


def route_projection(wl: Workload, dr: int = 32, device="cpu", seed: Optional[int] = None) -> torch.Tensor:
    """W [L][Hq][dr][d] ~ N(0, dr/d) in the storage dtype: a seeded stand-in for the
    trained per-(layer, head) routing projections (no trained weights exist). With
    q ~ N(0, I) each of the dr projected coordinates then has variance dr, so a dot
    product with a unit vector divided by sqrt(dr) has unit variance, the same order
    as the spread of log|S| over the spans."""
    seed = wl.seed if seed is None else seed
    g = _gen(device, seed, 5, dr)
    W = torch.randn(wl.L, wl.Hq, dr, wl.d, generator=g, device=device) * (dr / wl.d) ** 0.5
    return W.to(wl.torch_dtype())


def rank_gates(wl: Workload, m_cap: int, device="cpu", seed: Optional[int] = None) -> torch.Tensor:
    """Gates [B][L][Hkv][m_cap][2][rank] (fp32) for the keys and the values of every
    span: a seeded stand-in for a rank predictor's output. About 30 % exactly 1,
    15 % exactly 0 and the rest uniform in (0.15, 0.7)."""
    seed = wl.seed if seed is None else seed
    g = _gen(device, seed, 6, m_cap)
    u = torch.rand(wl.B, wl.L, wl.Hkv, m_cap, 2, wl.rank, generator=g, device=device)
    return torch.where(u > 0.7, torch.ones_like(u), torch.where(u < 0.15, torch.zeros_like(u), u))


def taus(wl: Workload, seed: Optional[int] = None) -> Optional[torch.Tensor]:
    """Return tau [L][Hq] (float64, CPU) or None when the workload calibrates tau."""
    seed = wl.seed if seed is None else seed
    if wl.tau_kind == "fixed":
        return torch.full((wl.L, wl.Hq), float(wl.tau_a), dtype=torch.float64)
    if wl.tau_kind == "uniform":
        g = _gen("cpu", seed, 4)
        u = torch.rand(wl.L, wl.Hq, generator=g, dtype=torch.float64)
        return wl.tau_a + (wl.tau_b - wl.tau_a) * u
    return None
