// K-d: split-K mixed-resolution flash-decoding over the span-structured cache.
//
// SeKV blog walkthrough, section 2.3: Eq. (5) routing gate
//   alpha_S = sigmoid(q . Kbar_S / sqrt(d') + log|S|), Kbar_S = kbar_S / ||kbar_S|| (W = I, d' = d)
// and Eq. (9) zoom decision z_S = 1[alpha_S > tau^(l,h)], compared here in logit
// space against theta = ln(tau / (1 - tau)). SeKV summary page, workflow paragraph
// (Stage 2): anchors and zoomed spans enter with token-level keys/values (zoomed
// ones reconstructed from their bases), non-zoomed spans with (kbar_S, vbar_S) and
// a +log|S| logit correction, all in ONE softmax (Fig. 2's "merge").
//
// Work decomposition: one CTA per (split, kv head, sequence x layer); a producer
// warp and four consumer warps. Phase 1 streams the split's anchor rows (K, V)
// and then its span rows (kbar, vbar, 1/||kbar||, log|S|) through a ring of
// shared-memory stages:
//   bf16: 2-D TMA tensor copies with 128-byte swizzle; each consumer warp takes
//         16 rows of a 64-row tile and runs q.K^T and p.V on the tensor cores
//         (mma.sync m16n8k16, the G query heads of the kv head padded to M = 16:
//         GQA, one K/V read serves all G heads). The q.kbar accumulator of a span
//         row is both its routing logit and its coarse attention logit.
//   fp32: 1-D bulk copies and CUDA-core dot products (each lane owns d/32 dims,
//         a 32-way transpose-reduce finishes the dots).
// Spans zoomed by any head of the group are queued. Phase 2 attends them without
// materialising K_S: each consumer warp pulls spans from the queue and streams
// B_S rows, A_S/C_S token chunks and D_S rows through its own 3-slot ring:
// u = B_S q, scores A_S u, y = C_S^T p, contribution y^T D_S. Softmax state is
// kept in the log2 domain; the CTA merges its warps' states, a second small
// kernel merges the splits by log-sum-exp.
#include <cuda.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "sekv_common.cuh"
#include "sekv_internal.h"

namespace sekv {

constexpr int kNW = 4;          // consumer warps per CTA
constexpr int kRMax = 64;       // largest basis rank the decode accepts

template <int DT, int D, int G>
struct DecCfg {
    static constexpr bool MMA = DT == SEKV_BF16;
    static constexpr int DPL = D / 32;                      // dims per lane (CUDA-core layout)
    static constexpr int ESZ = Elt<DT>::bytes;
    static constexpr int ROWB = D * ESZ;                    // bytes of one K/V row
    // rows per warp per tile: 16 on the tensor-core path, 32/G on the CUDA-core path
    static constexpr int R = MMA ? 16 : 32 / G;
    static constexpr int TR = kNW * R;                      // rows per tile
    static constexpr int NBOX = D / 64;                     // 128-byte-wide TMA boxes per row
    static constexpr int TILE = TR * ROWB;                  // bytes of one K (or V) tile
    static constexpr int META = 2 * TR * 4;                 // inv_norm + logS of a span tile
    static constexpr int STAGE0 = 2 * TILE + META;
    static constexpr int STAGE = MMA ? (STAGE0 + 1023) / 1024 * 1024 : STAGE0;
    static constexpr int NS0 = (MMA ? 68 * 1024 : 64 * 1024) / STAGE;     // 2 CTAs / SM on the bf16 path
    static constexpr int NS = NS0 < 2 ? 2 : (NS0 > 6 ? 6 : NS0);   // ring depth
    static constexpr int YPL = kRMax * G / 32;              // y entries per lane (zoom)
    static constexpr int WSCR = MMA ? 0 : (64 * G) + 2 * kRMax * G;   // per-warp scratch floats (fp32 zoom)
    // zoom phase: per-warp ring of ZNS slots of ZSLOT bytes, carved from the stage ring
    static constexpr int ZNS = 3;
    static constexpr int ZSLOT = 4096;
    static constexpr int RB = ZSLOT / ROWB;                 // B / D rows per slot
    static constexpr int ZBYTES = kNW * ZNS * ZSLOT;
    // partial softmax states merged at the end: per warp one for the stream and,
    // on the tensor-core path, one for its zoomed spans
    static constexpr int NSTATE = kNW;
    static constexpr int SBYTES = NSTATE * (G * D + 2 * G) * 4;
    // tensor-core zoom scratch per warp: u^T and (beta y)^T as hi/lo bf16 [2][8][72], p^T [8][72]
    static constexpr int ZSCR = 5888;
    static constexpr int RING0 = NS * STAGE;
    static constexpr int RING1 = ZBYTES + (MMA ? kNW * ZSCR : 0) > SBYTES ? ZBYTES + (MMA ? kNW * ZSCR : 0) : SBYTES;
    static constexpr int RING = RING0 > RING1 ? RING0 : RING1;
    static constexpr int HDR = 1024;                        // mbarriers + counters (keeps stages 1 KB aligned)
};

struct DecArgs {
    const char* q;
    const int32_t* a_count;
    const int32_t* m_count;
    const int32_t* span_beg;
    const int32_t* span_end;
    const float* logS;
    const int64_t* blk_off;
    const char* Ka;
    const char* Va;
    const char* kbar;
    const char* vbar;
    const float* inv_norm;
    const float* theta;
    const char* arena;
    const int64_t* slot;
    uint32_t* zmask;
    float* route_logits;
    int32_t* status;
    float* part_o;    // [B*Lr*Hkv][G][nsplit][D]
    float* part_ml;   // [B*Lr*Hkv][G][nsplit][2]  (max, sum) in the log2 domain
    int64_t region;
    float scale;
    int L, l0, Lr, Hq, Hkv, a_cap, m_cap, rank, phase, nsplit, sch_max, qcap, mw;
};

// TMA descriptors of the anchor and summary stores (bf16 path), viewed as 2-D
// [rows][d] tensors with 64 x 64 boxes and 128-byte swizzle.
struct DecMaps {
    CUtensorMap Ka, Va, kbar, vbar;
};

template <int DT, int D, int G>
static size_t decode_smem_bytes(int sch_max, int qcap) {
    using C = DecCfg<DT, D, G>;
    size_t s = C::HDR;
    s += (size_t)C::RING;
    s += (size_t)kNW * qcap * 4;                               // zoom queues
    s += (size_t)G * (sch_max / 32) * 4;                       // zoom-mask words
    s += (size_t)kNW * C::WSCR * 4;                            // per-warp scratch
    return round_up(s, 128) + 1024;                            // + alignment slack
}

// A zoomed span as the zoom pipeline sees it (warp-uniform values).
struct ZSpan {
    const char* blk;     // the span's block for this kv head
    int S;
    uint32_t hm;         // query heads of the group that zoom it
    int len, rS, nB, nAC, TC;
    int64_t pa;          // elements of the A (and of the C) section
    bool valid;
};

// shared-memory carve-up common to both paths
struct DecSmem {
    uint64_t* full;      // [NS]
    uint64_t* empty;     // [NS]
    uint64_t* zbar;      // [kNW][ZNS]
    int* qcnt;           // [kNW]
    int* zq_next;
    unsigned char* stages;
    int* zq;             // [kNW][qcap]
    uint32_t* zw;        // [G][zwords]
    float* wscr;         // [kNW][WSCR]
    float* st_m;         // [NSTATE][G]   (in the ring, once the zoom phase is over)
    float* st_l;         // [NSTATE][G]
    float* st_o;         // [NSTATE][G][D]
};

template <class C, int G, int D>
SEKV_DEV DecSmem carve_smem(unsigned char* base, int qcap, int zwords) {
    DecSmem s;
    s.full = reinterpret_cast<uint64_t*>(base);
    s.empty = s.full + 8;
    s.zbar = s.full + 16;
    s.qcnt = reinterpret_cast<int*>(base + 256);
    s.zq_next = s.qcnt + kNW;
    s.stages = base + C::HDR;
    s.zq = reinterpret_cast<int*>(s.stages + C::RING);
    s.zw = reinterpret_cast<uint32_t*>(s.zq + kNW * qcap);
    s.wscr = reinterpret_cast<float*>(s.zw + G * zwords);
    s.st_m = reinterpret_cast<float*>(s.stages);             // written after the zoom phase
    s.st_l = s.st_m + C::NSTATE * G;
    s.st_o = s.st_l + C::NSTATE * G;
    return s;
}

// ---------------------------------------------------------------------------
// Phase 2: attend the queued zoomed spans (one warp per span at a time).
// (m_run, l_run, o, m_lane) is the softmax state the spans are merged into.
// ---------------------------------------------------------------------------
template <int DT, int D, int G>
SEKV_DEV void zoom_phase(const DecArgs& a, const DecSmem& sm, int warp, int lane, int b, int l, int kvh,
                         float (&m_run)[G], float (&l_run)[G], float (&o)[G][D / 32], float& m_lane) {
    using C = DecCfg<DT, D, G>;
    constexpr int DPL = C::DPL;
    constexpr int R = 32 / G;                      // rows per transpose-reduce batch
    const int rL = lane / G, hL = lane % G;
    const float sl2 = a.scale * kLog2e;
    float q[G][DPL];
    {
        const char* qp = a.q + (((int64_t)b * a.L + l) * a.Hq + (int64_t)kvh * G) * C::ROWB + lane * DPL * C::ESZ;
#pragma unroll
        for (int h = 0; h < G; ++h) Vec<DT, DPL>::load(qp + h * C::ROWB, q[h]);
    }
    const int nq_total = sm.qcnt[0] + sm.qcnt[1] + sm.qcnt[2] + sm.qcnt[3];
    unsigned char* zring = sm.stages + (size_t)warp * C::ZNS * C::ZSLOT;
    uint64_t* zb = sm.zbar + warp * C::ZNS;
    float* pb = sm.wscr + warp * C::WSCR;          // 64*G floats (token p of a chunk)
    float* ub = pb + 64 * G;                       // kRMax*G floats
    float* yb = ub + kRMax * G;                    // kRMax*G floats

    auto grab = [&]() -> ZSpan {
        ZSpan sp;
        sp.valid = false;
        sp.blk = nullptr;
        sp.S = 0; sp.hm = 0u; sp.len = 0; sp.rS = 1; sp.nB = 0; sp.nAC = 0; sp.TC = 8; sp.pa = 0;
        int e = 0;
        if (lane == 0) e = atomicAdd(sm.zq_next, 1);
        e = __shfl_sync(0xffffffffu, e, 0);
        if (e >= nq_total) return sp;
        int w = 0;
        while (w < kNW - 1 && e >= sm.qcnt[w]) { e -= sm.qcnt[w]; ++w; }
        const int ent = sm.zq[w * a.qcap + e];
        sp.S = ent & 0xffffff;
        sp.hm = (uint32_t)ent >> 24;
        const int beg = a.span_beg[(int64_t)b * a.m_cap + sp.S];
        sp.len = a.span_end[(int64_t)b * a.m_cap + sp.S] - beg;
        if (sp.len < 1) {
            set_status(a.status, SEKV_ERR_INVALID_ARG);
            sp.len = 0;
        }
        sp.rS = sp.len > 0 ? block_rank(sp.len, D, a.rank) : 1;
        sp.pa = block_ac_elems(sp.len, sp.rS);
        const int64_t be = block_elems(sp.len > 0 ? sp.len : 1, D, a.rank);
        int64_t off = -1;
        if (sp.len > 0) {
            if (a.slot) {
                off = a.slot[((int64_t)b * a.L + l) * a.m_cap + sp.S];
                if (off < 0) set_status(a.status, SEKV_ERR_COLD_SPAN);
            } else {
                off = ((int64_t)b * a.L + l) * a.region + a.blk_off[(int64_t)b * (a.m_cap + 1) + sp.S];
            }
        }
        sp.blk = off >= 0 ? a.arena + (off + (int64_t)kvh * be) * C::ESZ : nullptr;
        int tc = (C::ZSLOT / 2) / (sp.rS * C::ESZ);
        tc = tc > 64 ? 64 : tc;
        sp.TC = (tc & ~7) < 8 ? 8 : (tc & ~7);
        sp.nB = (sp.rS + C::RB - 1) / C::RB;
        sp.nAC = (sp.len + sp.TC - 1) / sp.TC;
        sp.valid = true;
        return sp;
    };
    auto nslots = [](const ZSpan& sp) { return sp.blk ? 2 * sp.nB + sp.nAC : 0; };

    ZSpan cur = grab(), nxt;
    nxt.valid = false;
    nxt.blk = nullptr;
    nxt.nB = nxt.nAC = 0;
    bool i_next = false;       // the issue cursor is in nxt
    int i_k = 0;               // slots issued of the span under the issue cursor
    uint32_t nis = 0, ncons = 0;
    bool zok = true;

    auto issue = [&]() {
        // order this warp's earlier shared-memory reads of a slot before the bulk
        // copy that refills it
        fence_proxy_async();
        while (nis - ncons < (uint32_t)C::ZNS) {
            if (!i_next && i_k >= nslots(cur)) {
                if (!cur.valid) break;
                nxt = grab();
                i_next = true;
                i_k = 0;
            }
            // fields of the span under the issue cursor, selected by value
            const bool sv = i_next ? nxt.valid : cur.valid;
            const char* sblk = i_next ? nxt.blk : cur.blk;
            const int snB = i_next ? nxt.nB : cur.nB, snAC = i_next ? nxt.nAC : cur.nAC;
            const int srS = i_next ? nxt.rS : cur.rS, slen = i_next ? nxt.len : cur.len;
            const int sTC = i_next ? nxt.TC : cur.TC;
            const int64_t spa = i_next ? nxt.pa : cur.pa;
            if (!sv || !sblk || i_k >= 2 * snB + snAC) break;
            const int slot = nis % C::ZNS;
            unsigned char* dst = zring + slot * C::ZSLOT;
            if (lane == 0) {
                const int k = i_k;
                if (k < snB || k >= snB + snAC) {
                    const bool isD = k >= snB;
                    const int j = isD ? k - snB - snAC : k;
                    const int r0 = j * C::RB;
                    const uint32_t bytes = (uint32_t)min(C::RB, srS - r0) * C::ROWB;
                    const char* src = sblk + (2 * spa + (isD ? (int64_t)srS * D : 0) + (int64_t)r0 * D) * C::ESZ;
                    mbar_arrive_expect_tx(&zb[slot], bytes);
                    bulk_g2s(dst, src, bytes, &zb[slot]);
                } else {
                    const int t0 = (k - snB) * sTC;
                    const int nt = min(sTC, slen - t0);
                    const uint32_t bytes = (uint32_t)round_up((int64_t)nt * srS * C::ESZ, 16);
                    const int64_t off = (int64_t)t0 * srS * C::ESZ;
                    mbar_arrive_expect_tx(&zb[slot], 2 * bytes);
                    bulk_g2s(dst, sblk + off, bytes, &zb[slot]);
                    bulk_g2s(dst + C::ZSLOT / 2, sblk + spa * C::ESZ + off, bytes, &zb[slot]);
                }
            }
            ++i_k;
            ++nis;
        }
    };

    while (cur.valid && zok) {
        const int total = nslots(cur);
        float msp[G], lsp[G];
#pragma unroll
        for (int h = 0; h < G; ++h) { msp[h] = -INFINITY; lsp[h] = 0.f; }
        float y[C::YPL];
#pragma unroll
        for (int j = 0; j < C::YPL; ++j) y[j] = 0.f;
        float betaL = 0.f;
        for (int k = 0; k < total; ++k) {
            issue();
            const int slot = ncons % C::ZNS;
            if (!mbar_wait(&zb[slot], (ncons / C::ZNS) & 1)) {
                set_status(a.status, SEKV_ERR_TIMEOUT);
                zok = false;
                break;
            }
            const unsigned char* zs = zring + slot * C::ZSLOT;
            if (k < cur.nB) {
                // (1) u[i][h] = B_i . q_h for the slot's rows
                const int r0 = k * C::RB;
                const int rows = min(C::RB, cur.rS - r0);
                for (int i0 = 0; i0 < rows; i0 += R) {
                    float part[32];
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        float kk[DPL];
                        if (i0 + r < rows) {
                            Vec<DT, DPL>::load(zs + (i0 + r) * C::ROWB + lane * DPL * C::ESZ, kk);
                        } else {
#pragma unroll
                            for (int t = 0; t < DPL; ++t) kk[t] = 0.f;
                        }
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            float acc = 0.f;
#pragma unroll
                            for (int t = 0; t < DPL; ++t) acc = fmaf(kk[t], q[h][t], acc);
                            part[r * G + h] = acc;
                        }
                    }
                    const float u = transpose_reduce32(part, lane);
                    if (i0 + rL < rows) ub[(r0 + i0 + rL) * G + hL] = u;
                }
            } else if (k < cur.nB + cur.nAC) {
                // (2) token scores A u (lane owns tokens lane and lane+32 of the chunk),
                //     span-local online softmax, y = C^T p
                __syncwarp();
                const int t0 = (k - cur.nB) * cur.TC;
                const int nt = min(cur.TC, cur.len - t0);
                const unsigned char* As = zs;
                const unsigned char* Cs = zs + C::ZSLOT / 2;
                const int rS = cur.rS;
                float xs[2][G];
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int h = 0; h < G; ++h) xs[tt][h] = 0.f;
                if (DT == SEKV_BF16 && (rS & 7) == 0) {
                    for (int i0 = 0; i0 < rS; i0 += 8) {
                        float av[2][8];
#pragma unroll
                        for (int tt = 0; tt < 2; ++tt) {
                            const int t = lane + 32 * tt;
                            if (t < nt) {
                                const uint4 w = *reinterpret_cast<const uint4*>(As + ((int64_t)t * rS + i0) * 2);
                                av[tt][0] = bf16_lo(w.x); av[tt][1] = bf16_hi(w.x);
                                av[tt][2] = bf16_lo(w.y); av[tt][3] = bf16_hi(w.y);
                                av[tt][4] = bf16_lo(w.z); av[tt][5] = bf16_hi(w.z);
                                av[tt][6] = bf16_lo(w.w); av[tt][7] = bf16_hi(w.w);
                            } else {
#pragma unroll
                                for (int e = 0; e < 8; ++e) av[tt][e] = 0.f;
                            }
                        }
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            float uv[G];
                            if constexpr (G == 4) {
                                const float4 u4 = *reinterpret_cast<const float4*>(ub + (i0 + e) * 4);
                                uv[0] = u4.x; uv[1] = u4.y; uv[2] = u4.z; uv[3] = u4.w;
                            } else {
#pragma unroll
                                for (int h = 0; h < G; ++h) uv[h] = ub[(i0 + e) * G + h];
                            }
#pragma unroll
                            for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                                for (int h = 0; h < G; ++h) xs[tt][h] = fmaf(av[tt][e], uv[h], xs[tt][h]);
                        }
                    }
                } else {
#pragma unroll
                    for (int tt = 0; tt < 2; ++tt) {
                        const int t = lane + 32 * tt;
                        if (t < nt) {
                            for (int i = 0; i < rS; ++i) {
                                const float av = load1<DT>(As, (int64_t)t * rS + i);
#pragma unroll
                                for (int h = 0; h < G; ++h) xs[tt][h] = fmaf(av, ub[i * G + h], xs[tt][h]);
                            }
                        }
                    }
                }
                // logits of the heads that zoom this span; the others get no entries here
                float mx[G], ps[G], al[G];
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const bool zh = (cur.hm >> h) & 1u;
#pragma unroll
                    for (int tt = 0; tt < 2; ++tt)
                        xs[tt][h] = (zh && lane + 32 * tt < nt) ? xs[tt][h] * sl2 : -INFINITY;
                    mx[h] = fmaxf(xs[0][h], xs[1][h]);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                    for (int h = 0; h < G; ++h) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], off));
                float alL = 1.f;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float mnew = fmaxf(msp[h], mx[h]);
                    al[h] = (mnew == -INFINITY) ? 1.f : exp2f(msp[h] - mnew);
                    ps[h] = 0.f;
#pragma unroll
                    for (int tt = 0; tt < 2; ++tt) {
                        const float pv = (xs[tt][h] == -INFINITY) ? 0.f : exp2f(xs[tt][h] - mnew);
                        ps[h] += pv;
                        pb[(lane + 32 * tt) * G + h] = pv;
                    }
                    msp[h] = mnew;
                    if (h == hL) alL = al[h];
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                    for (int h = 0; h < G; ++h) ps[h] += __shfl_xor_sync(0xffffffffu, ps[h], off);
#pragma unroll
                for (int h = 0; h < G; ++h) lsp[h] = fmaf(lsp[h], al[h], ps[h]);
                __syncwarp();
                // y[i][h] += sum_t p[t][h] C[t][i]; lanes own (i, h) pairs
#pragma unroll
                for (int j = 0; j < C::YPL; ++j) {
                    const int i = (lane + 32 * j) / G;
                    if (i < rS) {
                        float acc0 = y[j] * alL, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
                        int tt = 0;
                        for (; tt + 4 <= nt; tt += 4) {
                            acc0 = fmaf(pb[(tt + 0) * G + hL], load1<DT>(Cs, (int64_t)(tt + 0) * rS + i), acc0);
                            acc1 = fmaf(pb[(tt + 1) * G + hL], load1<DT>(Cs, (int64_t)(tt + 1) * rS + i), acc1);
                            acc2 = fmaf(pb[(tt + 2) * G + hL], load1<DT>(Cs, (int64_t)(tt + 2) * rS + i), acc2);
                            acc3 = fmaf(pb[(tt + 3) * G + hL], load1<DT>(Cs, (int64_t)(tt + 3) * rS + i), acc3);
                        }
                        for (; tt < nt; ++tt)
                            acc0 = fmaf(pb[tt * G + hL], load1<DT>(Cs, (int64_t)tt * rS + i), acc0);
                        y[j] = (acc0 + acc1) + (acc2 + acc3);
                    }
                }
                __syncwarp();
            } else {
                if (k == cur.nB + cur.nAC) {
                    // (3) merge the span's softmax state into the running state
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        float al = 1.f, be2 = 0.f;
                        if ((cur.hm >> h) & 1u) {
                            const float mnew = fmaxf(m_run[h], msp[h]);
                            al = (m_run[h] == -INFINITY) ? 0.f : exp2f(m_run[h] - mnew);
                            be2 = exp2f(msp[h] - mnew);
                            l_run[h] = l_run[h] * al + lsp[h] * be2;
                            m_run[h] = mnew;
                        }
#pragma unroll
                        for (int t = 0; t < DPL; ++t) o[h][t] *= al;
                        if (h == hL) { betaL = be2; m_lane = m_run[h]; }
                    }
#pragma unroll
                    for (int j = 0; j < C::YPL; ++j) {
                        const int i = (lane + 32 * j) / G;
                        if (i < cur.rS) yb[i * G + hL] = y[j] * betaL;
                    }
                    __syncwarp();
                }
                // o += sum_i (beta y_i) D_i over the slot's rows
                const int r0 = (k - cur.nB - cur.nAC) * C::RB;
                const int rows = min(C::RB, cur.rS - r0);
                for (int r = 0; r < rows; ++r) {
                    float dv[DPL];
                    Vec<DT, DPL>::load(zs + r * C::ROWB + lane * DPL * C::ESZ, dv);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float yv = yb[(r0 + r) * G + h];
#pragma unroll
                        for (int t = 0; t < DPL; ++t) o[h][t] = fmaf(yv, dv[t], o[h][t]);
                    }
                }
            }
            __syncwarp();
            ++ncons;
        }
        if (!zok) break;
        // advance to the next span (the issue cursor may already be in it)
        if (i_next) {
            cur = nxt;
            i_next = false;
            nxt.valid = false;
        } else {
            cur = grab();
            i_k = 0;
        }
    }
    // drain anything still in flight (only after an error)
    while (ncons < nis) {
        if (!mbar_wait(&zb[ncons % C::ZNS], (ncons / C::ZNS) & 1)) set_status(a.status, SEKV_ERR_TIMEOUT);
        ++ncons;
    }
}

// ---------------------------------------------------------------------------
// Phase 2 on the tensor cores (bf16). Per zoomed span and the heads h that zoom
// it, with r = rank of the span:
//   u = B_S q          (mma: M = r basis rows, K = d, N = heads)
//   s = A_S u          (mma: M = 16 tokens, K = r)             -> online softmax p
//   y = C_S^T p        (mma: M = r, K = 16 tokens)
//   O += (beta y)^T D_S (mma: M = heads, K = r, N = d)  into the stream accumulators
// u and beta*y are rounded to bf16 as a hi + lo pair (about 16 significant bits);
// p is rounded to bf16 as on the streaming path. The span's (max, sum) merge into
// the warp's stream state (mm, lm, oc) for head gid = lane/4.
// ---------------------------------------------------------------------------
template <int D, int G>
SEKV_DEV void zoom_phase_mma(const DecArgs& a, const DecSmem& sm, int warp, int lane, int b, int l, int kvh,
                             const uint32_t (&qa)[D / 16][2], float& mm, float& lm, float (&oc)[D / 8][4]) {
    using C = DecCfg<SEKV_BF16, D, G>;
    constexpr int ROWB = C::ROWB;
    constexpr int RB = C::RB;
    const int gid = lane >> 2, cq = lane & 3;
    const float sl2 = a.scale * kLog2e;
    const int nq_total = sm.qcnt[0] + sm.qcnt[1] + sm.qcnt[2] + sm.qcnt[3];
    unsigned char* zring = sm.stages + (size_t)warp * C::ZNS * C::ZSLOT;
    uint64_t* zb = sm.zbar + warp * C::ZNS;
    __nv_bfloat16* ut = reinterpret_cast<__nv_bfloat16*>(sm.stages + C::ZBYTES + warp * C::ZSCR);  // [2][8][72]
    __nv_bfloat16* yt = ut + 2 * 8 * 72;                                                        // [2][8][72]
    __nv_bfloat16* pt = yt + 2 * 8 * 72;                                                        // [8][72]

    auto grab = [&]() -> ZSpan {
        ZSpan sp;
        sp.valid = false;
        sp.blk = nullptr;
        sp.S = 0; sp.hm = 0u; sp.len = 0; sp.rS = 1; sp.nB = 0; sp.nAC = 0; sp.TC = 8; sp.pa = 0;
        int e = 0;
        if (lane == 0) e = atomicAdd(sm.zq_next, 1);
        e = __shfl_sync(0xffffffffu, e, 0);
        if (e >= nq_total) return sp;
        int w = 0;
        while (w < kNW - 1 && e >= sm.qcnt[w]) { e -= sm.qcnt[w]; ++w; }
        const int ent = sm.zq[w * a.qcap + e];
        sp.S = ent & 0xffffff;
        sp.hm = (uint32_t)ent >> 24;
        const int beg = a.span_beg[(int64_t)b * a.m_cap + sp.S];
        sp.len = a.span_end[(int64_t)b * a.m_cap + sp.S] - beg;
        if (sp.len < 1) {
            set_status(a.status, SEKV_ERR_INVALID_ARG);
            sp.len = 0;
        }
        sp.rS = sp.len > 0 ? block_rank(sp.len, D, a.rank) : 1;
        sp.pa = block_ac_elems(sp.len, sp.rS);
        const int64_t be = block_elems(sp.len > 0 ? sp.len : 1, D, a.rank);
        int64_t off = -1;
        if (sp.len > 0) {
            if (a.slot) {
                off = a.slot[((int64_t)b * a.L + l) * a.m_cap + sp.S];
                if (off < 0) set_status(a.status, SEKV_ERR_COLD_SPAN);
            } else {
                off = ((int64_t)b * a.L + l) * a.region + a.blk_off[(int64_t)b * (a.m_cap + 1) + sp.S];
            }
        }
        sp.blk = off >= 0 ? a.arena + (off + (int64_t)kvh * be) * 2 : nullptr;
        int tc = (C::ZSLOT / 2) / (sp.rS * 2);
        tc = tc > 64 ? 64 : tc;
        sp.TC = (tc & ~7) < 8 ? 8 : (tc & ~7);
        sp.nB = (sp.rS + RB - 1) / RB;
        sp.nAC = (sp.len + sp.TC - 1) / sp.TC;
        sp.valid = true;
        return sp;
    };
    auto nslots = [](const ZSpan& sp) { return sp.blk ? 2 * sp.nB + sp.nAC : 0; };

    ZSpan cur = grab(), nxt;
    nxt.valid = false;
    nxt.blk = nullptr;
    nxt.nB = nxt.nAC = 0;
    bool i_next = false;
    int i_k = 0;
    uint32_t nis = 0, ncons = 0;
    bool zok = true;

    // slots start zeroed, so bytes past a copy are always finite
    for (int i = lane; i < C::ZNS * C::ZSLOT / 16; i += 32)
        reinterpret_cast<uint4*>(zring)[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncwarp();
    fence_proxy_async();

    auto issue = [&]() {
        if (nis - ncons < (uint32_t)C::ZNS) fence_proxy_async();
        while (nis - ncons < (uint32_t)C::ZNS) {
            if (!i_next && i_k >= nslots(cur)) {
                if (!cur.valid) break;
                nxt = grab();
                i_next = true;
                i_k = 0;
            }
            const bool sv = i_next ? nxt.valid : cur.valid;
            const char* sblk = i_next ? nxt.blk : cur.blk;
            const int snB = i_next ? nxt.nB : cur.nB, snAC = i_next ? nxt.nAC : cur.nAC;
            const int srS = i_next ? nxt.rS : cur.rS, slen = i_next ? nxt.len : cur.len;
            const int sTC = i_next ? nxt.TC : cur.TC;
            const int64_t spa = i_next ? nxt.pa : cur.pa;
            if (!sv || !sblk || i_k >= 2 * snB + snAC) break;
            const int slot = nis % C::ZNS;
            unsigned char* dst = zring + slot * C::ZSLOT;
            if (lane == 0) {
                const int k = i_k;
                if (k < snB || k >= snB + snAC) {
                    const bool isD = k >= snB;
                    const int j = isD ? k - snB - snAC : k;
                    const int r0 = j * RB;
                    const uint32_t bytes = (uint32_t)min(RB, srS - r0) * ROWB;
                    const char* src = sblk + (2 * spa + (isD ? (int64_t)srS * D : 0) + (int64_t)r0 * D) * 2;
                    mbar_arrive_expect_tx(&zb[slot], bytes);
                    bulk_g2s(dst, src, bytes, &zb[slot]);
                } else {
                    const int t0 = (k - snB) * sTC;
                    const int nt = min(sTC, slen - t0);
                    const uint32_t bytes = (uint32_t)round_up((int64_t)nt * srS * 2, 16);
                    const int64_t off = (int64_t)t0 * srS * 2;
                    mbar_arrive_expect_tx(&zb[slot], 2 * bytes);
                    bulk_g2s(dst, sblk + off, bytes, &zb[slot]);
                    bulk_g2s(dst + C::ZSLOT / 2, sblk + spa * 2 + off, bytes, &zb[slot]);
                }
            }
            ++i_k;
            ++nis;
        }
    };

    while (cur.valid && zok) {
        const int total = nslots(cur);
        const int rS = cur.rS;
        const int nig = (rS + 15) >> 4;                 // groups of 16 basis rows
        float msp[2] = {-INFINITY, -INFINITY}, lsp[2] = {0.f, 0.f};   // heads 2cq, 2cq+1
        float yacc[4][4];
#pragma unroll
        for (int ig = 0; ig < 4; ++ig) yacc[ig][0] = yacc[ig][1] = yacc[ig][2] = yacc[ig][3] = 0.f;
        for (int k = 0; k < total; ++k) {
            issue();
            const int slot = ncons % C::ZNS;
            if (!mbar_wait(&zb[slot], (ncons / C::ZNS) & 1)) {
                set_status(a.status, SEKV_ERR_TIMEOUT);
                zok = false;
                break;
            }
            const unsigned char* zs = zring + slot * C::ZSLOT;
            if (k < cur.nB) {
                // (1) u = B q for the slot's basis rows, stored transposed as hi/lo bf16
                const int r0 = k * RB;
                const int rows = min(RB, rS - r0);
                for (int g16 = 0; g16 < rows; g16 += 16) {
                    float uacc[4] = {0.f, 0.f, 0.f, 0.f};
                    const int arow = g16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        uint32_t af[4];
                        ldsm_x4(af, zs + arow * ROWB + (16 * kk + ((lane >> 4) << 3)) * 2);
                        const uint32_t bq[2] = {qa[kk][0], qa[kk][1]};
                        mma_bf16_16816(uacc, af, bq);
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int il = g16 + gid + ((e >> 1) << 3);          // row within the slot
                        const int i = r0 + il;
                        const int h = 2 * cq + (e & 1);
                        const float u = (il < rows) ? uacc[e] : 0.f;       // stale rows beyond r
                        const __nv_bfloat16 hi = __float2bfloat16_rn(u);
                        ut[h * 72 + i] = hi;
                        ut[(8 + h) * 72 + i] = __float2bfloat16_rn(u - __bfloat162float(hi));
                    }
                }
            } else if (k < cur.nB + cur.nAC) {
                // (2) scores s = A u for up to 64 tokens (four 16-token sub-chunks),
                //     span-local online softmax, y += C^T p
                __syncwarp();
                const int t0 = (k - cur.nB) * cur.TC;
                const int nt = min(cur.TC, cur.len - t0);
                const int nsc = (nt + 15) >> 4;
                const unsigned char* As = zs;
                const unsigned char* Cs = zs + C::ZSLOT / 2;
                const uint16_t* A16 = reinterpret_cast<const uint16_t*>(As);
                const uint16_t* C16 = reinterpret_cast<const uint16_t*>(Cs);
                const bool vec = (rS & 7) == 0;            // 16-byte rows: ldmatrix
                float sacc[4][4];
#pragma unroll
                for (int sc = 0; sc < 4; ++sc) {
                    sacc[sc][0] = sacc[sc][1] = sacc[sc][2] = sacc[sc][3] = 0.f;
                    if (sc < nsc) {
                        const int ts = 16 * sc;
                        for (int ks = 0; ks < nig; ++ks) {
                            uint32_t af[4];
                            if (vec) {
                                const int arow = ts + (lane & 7) + (((lane >> 3) & 1) << 3);
                                ldsm_x4(af, As + ((int64_t)arow * rS + 16 * ks + ((lane >> 4) << 3)) * 2);
                            } else {
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int t = ts + gid + ((e & 1) << 3);
                                    const int i = 16 * ks + 2 * cq + ((e >> 1) << 3);
                                    const uint32_t x0 = (t < nt && i < rS) ? A16[t * rS + i] : 0u;
                                    const uint32_t x1 = (t < nt && i + 1 < rS) ? A16[t * rS + i + 1] : 0u;
                                    af[e] = x0 | (x1 << 16);
                                }
                            }
                            const uint32_t* uh = reinterpret_cast<const uint32_t*>(ut + gid * 72 + 16 * ks + 2 * cq);
                            const uint32_t* ul = reinterpret_cast<const uint32_t*>(ut + (8 + gid) * 72 + 16 * ks + 2 * cq);
                            const uint32_t bh[2] = {uh[0], uh[4]};
                            const uint32_t bl[2] = {ul[0], ul[4]};
                            mma_bf16_16816(sacc[sc], af, bh);
                            mma_bf16_16816(sacc[sc], af, bl);
                        }
                    }
                }
                // sacc[sc][e]: token 16 sc + gid + 8 (e >> 1), head 2 cq + (e & 1)
                float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
                for (int sc = 0; sc < 4; ++sc)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int t = 16 * sc + gid + ((e >> 1) << 3);
                        const int h = 2 * cq + (e & 1);
                        const float v = (t < nt && h < G && ((cur.hm >> h) & 1u)) ? sacc[sc][e] * sl2 : -INFINITY;
                        sacc[sc][e] = v;
                        if (e & 1) mx1 = fmaxf(mx1, v); else mx0 = fmaxf(mx0, v);
                    }
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                }
                const float mn0 = fmaxf(msp[0], mx0), mn1 = fmaxf(msp[1], mx1);
                const float al0 = (mn0 == -INFINITY) ? 1.f : exp2f(msp[0] - mn0);
                const float al1 = (mn1 == -INFINITY) ? 1.f : exp2f(msp[1] - mn1);
                float ps0 = 0.f, ps1 = 0.f;
                __syncwarp();                                   // previous reads of pt are done
#pragma unroll
                for (int sc = 0; sc < 4; ++sc)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float v = sacc[sc][e];
                        const float pv = (v == -INFINITY) ? 0.f : exp2f(v - ((e & 1) ? mn1 : mn0));
                        if (e & 1) ps1 += pv; else ps0 += pv;
                        pt[(2 * cq + (e & 1)) * 72 + 16 * sc + gid + ((e >> 1) << 3)] = __float2bfloat16_rn(pv);
                    }
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    ps0 += __shfl_xor_sync(0xffffffffu, ps0, off);
                    ps1 += __shfl_xor_sync(0xffffffffu, ps1, off);
                }
                lsp[0] = fmaf(lsp[0], al0, ps0);
                lsp[1] = fmaf(lsp[1], al1, ps1);
                msp[0] = mn0;
                msp[1] = mn1;
                if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
                    for (int ig = 0; ig < 4; ++ig) {
                        yacc[ig][0] *= al0; yacc[ig][1] *= al1;
                        yacc[ig][2] *= al0; yacc[ig][3] *= al1;
                    }
                }
                __syncwarp();
#pragma unroll
                for (int sc = 0; sc < 4; ++sc) {
                    if (sc < nsc) {
                        const int ts = 16 * sc;
                        const uint32_t* pp = reinterpret_cast<const uint32_t*>(pt + gid * 72 + ts + 2 * cq);
                        const uint32_t bp[2] = {pp[0], pp[4]};
                        // this lane's tokens in the C^T fragment: ts + 2cq, +1 (k 0..7) and +8
                        const int tk = ts + 2 * cq;
                        const uint32_t m0 = (tk < nt ? 0x0000ffffu : 0u) | (tk + 1 < nt ? 0xffff0000u : 0u);
                        const uint32_t m1 = (tk + 8 < nt ? 0x0000ffffu : 0u) | (tk + 9 < nt ? 0xffff0000u : 0u);
#pragma unroll
                        for (int ig = 0; ig < 4; ++ig) {
                            if (ig < nig) {
                                uint32_t af[4];
                                if (vec) {
                                    const int mi = lane >> 3;
                                    const int trow = ts + (lane & 7) + ((mi >> 1) << 3);
                                    ldsm_x4_t(af, Cs + ((int64_t)trow * rS + 16 * ig + ((mi & 1) << 3)) * 2);
                                    af[0] &= m0; af[1] &= m0; af[2] &= m1; af[3] &= m1;
                                } else {
#pragma unroll
                                    for (int e = 0; e < 4; ++e) {
                                        const int i = 16 * ig + gid + ((e & 1) << 3);
                                        const int t = ts + 2 * cq + ((e >> 1) << 3);
                                        const uint32_t x0 = (i < rS && t < nt) ? C16[t * rS + i] : 0u;
                                        const uint32_t x1 = (i < rS && t + 1 < nt) ? C16[(t + 1) * rS + i] : 0u;
                                        af[e] = x0 | (x1 << 16);
                                    }
                                }
                                mma_bf16_16816(yacc[ig], af, bp);
                            }
                        }
                    }
                }
            } else {
                if (k == cur.nB + cur.nAC) {
                    // (3) merge: beta per zooming head, (beta y)^T to shared memory, stream state update
                    const float mh0 = __shfl_sync(0xffffffffu, mm, 4 * (2 * cq));
                    const float mh1 = __shfl_sync(0xffffffffu, mm, 4 * (2 * cq + 1));
                    const bool z0 = 2 * cq < G && ((cur.hm >> (2 * cq)) & 1u);
                    const bool z1 = 2 * cq + 1 < G && ((cur.hm >> (2 * cq + 1)) & 1u);
                    const float be0 = z0 ? exp2f(msp[0] - fmaxf(mh0, msp[0])) : 0.f;
                    const float be1 = z1 ? exp2f(msp[1] - fmaxf(mh1, msp[1])) : 0.f;
#pragma unroll
                    for (int ig = 0; ig < 4; ++ig) {
                        if (ig < nig) {
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int i = 16 * ig + gid + ((e >> 1) << 3);
                                const int h = 2 * cq + (e & 1);
                                const float v = i < rS ? yacc[ig][e] * ((e & 1) ? be1 : be0) : 0.f;
                                const __nv_bfloat16 hi = __float2bfloat16_rn(v);
                                yt[h * 72 + i] = hi;
                                yt[(8 + h) * 72 + i] = __float2bfloat16_rn(v - __bfloat162float(hi));
                            }
                        }
                    }
                    const int src = gid >> 1;
                    const float ms0 = __shfl_sync(0xffffffffu, msp[0], src), ms1 = __shfl_sync(0xffffffffu, msp[1], src);
                    const float ls0 = __shfl_sync(0xffffffffu, lsp[0], src), ls1 = __shfl_sync(0xffffffffu, lsp[1], src);
                    const float msg = (gid & 1) ? ms1 : ms0, lsg = (gid & 1) ? ls1 : ls0;
                    if (gid < G && ((cur.hm >> gid) & 1u)) {
                        const float mnew = fmaxf(mm, msg);
                        const float alpha = (mm == -INFINITY) ? 0.f : exp2f(mm - mnew);
                        const float beta = exp2f(msg - mnew);
                        lm = lm * alpha + lsg * beta;
                        mm = mnew;
#pragma unroll
                        for (int n = 0; n < D / 8; ++n) {
                            oc[n][0] *= alpha;
                            oc[n][1] *= alpha;
                        }
                    }
                    __syncwarp();
                }
                // (4) O += (beta y)^T D over the slot's basis rows
                const int r0 = (k - cur.nB - cur.nAC) * RB;
                const int rows = min(RB, rS - r0);
                for (int g16 = 0; g16 < rows; g16 += 16) {
                    const int ks = (r0 + g16) >> 4;
                    const uint32_t* yh = reinterpret_cast<const uint32_t*>(yt + gid * 72 + 16 * ks + 2 * cq);
                    const uint32_t* yl = reinterpret_cast<const uint32_t*>(yt + (8 + gid) * 72 + 16 * ks + 2 * cq);
                    const uint32_t ah[4] = {yh[0], 0u, yh[4], 0u};
                    const uint32_t al[4] = {yl[0], 0u, yl[4], 0u};
                    const int mi = lane >> 3;
                    const int drow = g16 + (lane & 7) + ((mi & 1) << 3);
                    // this lane's B rows (k): g16 + 2cq, +1 (b0) and +8 (b1); zero the stale ones
                    const int k0 = g16 + 2 * cq;
                    const uint32_t m0 = (k0 < rows ? 0x0000ffffu : 0u) | (k0 + 1 < rows ? 0xffff0000u : 0u);
                    const uint32_t m1 = (k0 + 8 < rows ? 0x0000ffffu : 0u) | (k0 + 9 < rows ? 0xffff0000u : 0u);
#pragma unroll
                    for (int qd = 0; qd < D / 16; ++qd) {
                        uint32_t vb[4];
                        ldsm_x4_t(vb, zs + drow * ROWB + (16 * qd + ((mi >> 1) << 3)) * 2);
                        const uint32_t b0[2] = {vb[0] & m0, vb[1] & m1};
                        const uint32_t b1[2] = {vb[2] & m0, vb[3] & m1};
                        mma_bf16_16816(oc[2 * qd], ah, b0);
                        mma_bf16_16816(oc[2 * qd], al, b0);
                        mma_bf16_16816(oc[2 * qd + 1], ah, b1);
                        mma_bf16_16816(oc[2 * qd + 1], al, b1);
                    }
                }
            }
            __syncwarp();
            ++ncons;
        }
        if (!zok) break;
        if (i_next) {
            cur = nxt;
            i_next = false;
            nxt.valid = false;
        } else {
            cur = grab();
            i_k = 0;
        }
    }
    while (ncons < nis) {
        if (!mbar_wait(&zb[ncons % C::ZNS], (ncons / C::ZNS) & 1)) set_status(a.status, SEKV_ERR_TIMEOUT);
        ++ncons;
    }
}

// write one partial softmax state in the dims-per-lane layout
template <int D, int G>
SEKV_DEV void store_state_lanes(const DecSmem& sm, int idx, int lane, const float (&m)[G], const float (&l)[G],
                                const float (&o)[G][D / 32]) {
    constexpr int DPL = D / 32;
    if (lane == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            sm.st_m[idx * G + h] = m[h];
            sm.st_l[idx * G + h] = l[h];
        }
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int k = 0; k < DPL; ++k) sm.st_o[(idx * G + h) * D + lane * DPL + k] = o[h][k];
}

template <int DT, int D, int G>
__global__ void __launch_bounds__((kNW + 1) * 32, DT == SEKV_BF16 ? 2 : 3)
decode_kernel(const DecArgs a, const __grid_constant__ DecMaps maps) {
    using C = DecCfg<DT, D, G>;
    constexpr int DPL = C::DPL, R = C::R, TR = C::TR, NS = C::NS;
    extern __shared__ __align__(1024) unsigned char sm_raw[];
    unsigned char* base = sm_raw + ((1024 - (smem_u32(sm_raw) & 1023)) & 1023);
    const int zwords = a.sch_max / 32;
    const DecSmem sm = carve_smem<C, G, D>(base, a.qcap, zwords);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int kvh = blockIdx.y;
    const int b = blockIdx.z / a.Lr, li = blockIdx.z % a.Lr, l = a.l0 + li;
    const int split = blockIdx.x;
    const int64_t unit = ((int64_t)b * a.L + l) * a.Hkv + kvh;            // global (b, l, kvh)
    const int64_t lunit = ((int64_t)b * a.Lr + li) * a.Hkv + kvh;         // within this launch
    const bool route_only = a.phase == SEKV_ROUTE;

    const int ab = min(a.a_count[b], a.a_cap);
    const int mb = min(a.m_count[b], a.m_cap);
    int a0 = 0, a1 = 0;
    if (!route_only) {
        const int ach = (ab + a.nsplit - 1) / a.nsplit;
        a0 = min(ab, split * ach);
        a1 = min(ab, a0 + ach);
    }
    const int sch = (((mb + a.nsplit - 1) / a.nsplit) + 31) & ~31;
    const int s0 = split * sch;
    const int s1 = min(mb, s0 + sch);
    const int nta = (a1 - a0 + TR - 1) / TR;
    const int nts = s1 > s0 ? (s1 - s0 + TR - 1) / TR : 0;
    const int ntiles = nta + nts;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], kNW);
        }
        for (int s = 0; s < kNW * C::ZNS; ++s) mbar_init(&sm.zbar[s], 1);
        *sm.zq_next = 0;
        fence_barrier_init();
    }
    for (int i = tid; i < G * zwords; i += blockDim.x) sm.zw[i] = 0u;
    __syncthreads();

    const float sl2 = a.scale * kLog2e;
    bool ok = true;

    // stream state of a consumer warp
    //   tensor-core path: lane (g = lane/4, c = lane%4) holds head g's (m, l) and the
    //   accumulator fragments oc[n][0..1] = O[g][8n + 2c .. 8n + 2c + 1]
    //   CUDA-core path:   every lane holds (m, l) of all heads and o[h][dims of lane]
    float m_run[G], l_run[G], o[G][DPL];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m_run[h] = -INFINITY;
        l_run[h] = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[h][i] = 0.f;
    }
    float m_lane = -INFINITY;
    uint32_t qa[C::MMA ? D / 16 : 1][2];      // tensor-core path: q fragments (stream and zoom)
    float oc[C::MMA ? D / 8 : 1][4];
    float mm = -INFINITY, lm = 0.f;           // tensor-core path: this lane's head
#pragma unroll
    for (int n = 0; n < (C::MMA ? D / 8 : 1); ++n) oc[n][0] = oc[n][1] = oc[n][2] = oc[n][3] = 0.f;

    if (warp == kNW) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < ntiles; ++i) {
                const int s = i % NS;
                if (i >= NS && !mbar_wait(&sm.empty[s], ((i / NS) - 1) & 1)) {
                    set_status(a.status, SEKV_ERR_TIMEOUT);
                    break;
                }
                unsigned char* st = sm.stages + (size_t)s * C::STAGE;
                if (i < nta) {
                    const int r0 = a0 + i * TR;
                    if constexpr (C::MMA) {
                        const int y = (int)(unit * a.a_cap + r0);
                        mbar_arrive_expect_tx(&sm.full[s], 2 * C::NBOX * 8192);
#pragma unroll
                        for (int h = 0; h < C::NBOX; ++h) {
                            tma_load_2d(st + h * 8192, &maps.Ka, 64 * h, y, &sm.full[s]);
                            tma_load_2d(st + C::TILE + h * 8192, &maps.Va, 64 * h, y, &sm.full[s]);
                        }
                    } else {
                        const uint32_t bytes = (uint32_t)min(TR, a1 - r0) * C::ROWB;
                        mbar_arrive_expect_tx(&sm.full[s], 2 * bytes);
                        const int64_t off = (unit * a.a_cap + r0) * C::ROWB;
                        bulk_g2s(st, a.Ka + off, bytes, &sm.full[s]);
                        bulk_g2s(st + C::TILE, a.Va + off, bytes, &sm.full[s]);
                    }
                } else {
                    const int S0 = s0 + (i - nta) * TR;
                    const int rows = min(TR, s1 - S0);
                    const uint32_t mbytes = (uint32_t)((rows + 3) & ~3) * 4;
                    if constexpr (C::MMA) {
                        const int y = (int)(unit * a.m_cap + S0);
                        mbar_arrive_expect_tx(&sm.full[s], (route_only ? 1 : 2) * C::NBOX * 8192 + 2 * mbytes);
#pragma unroll
                        for (int h = 0; h < C::NBOX; ++h) {
                            tma_load_2d(st + h * 8192, &maps.kbar, 64 * h, y, &sm.full[s]);
                            if (!route_only) tma_load_2d(st + C::TILE + h * 8192, &maps.vbar, 64 * h, y, &sm.full[s]);
                        }
                    } else {
                        const uint32_t bytes = (uint32_t)rows * C::ROWB;
                        mbar_arrive_expect_tx(&sm.full[s], (route_only ? bytes : 2 * bytes) + 2 * mbytes);
                        const int64_t off = (unit * a.m_cap + S0) * C::ROWB;
                        bulk_g2s(st, a.kbar + off, bytes, &sm.full[s]);
                        if (!route_only) bulk_g2s(st + C::TILE, a.vbar + off, bytes, &sm.full[s]);
                    }
                    bulk_g2s(st + 2 * C::TILE, a.inv_norm + unit * a.m_cap + S0, mbytes, &sm.full[s]);
                    bulk_g2s(st + 2 * C::TILE + TR * 4, a.logS + (int64_t)b * a.m_cap + S0, mbytes, &sm.full[s]);
                }
                issued = i + 1;
            }
            // drain: every issued copy has landed before the ring is reused
            for (int i = max(0, issued - NS); i < issued; ++i)
                if (!mbar_wait(&sm.full[i % NS], (i / NS) & 1)) set_status(a.status, SEKV_ERR_TIMEOUT);
        }
    } else if constexpr (C::MMA) {
        // ------------------------------------------------ consumers, tensor cores
        const int g = lane >> 2, c = lane & 3;
        const bool gv = g < G;
        const float th = gv ? a.theta[(int64_t)l * a.Hq + kvh * G + g] : INFINITY;
        // q as m16n8k16 A fragments (rows = heads, zero-padded to 16): a0, a2 per k-step
        {
            const uint32_t* qp = reinterpret_cast<const uint32_t*>(
                a.q + (((int64_t)b * a.L + l) * a.Hq + (int64_t)kvh * G + (gv ? g : 0)) * C::ROWB);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                qa[kk][0] = gv ? qp[(16 * kk + 2 * c) / 2] : 0u;
                qa[kk][1] = gv ? qp[(16 * kk + 8 + 2 * c) / 2] : 0u;
            }
        }
        int qn = 0;
        int* myq = sm.zq + warp * a.qcap;
        const int rbase = warp * R;                       // 16 rows of each tile
        for (int i = 0; i < ntiles && ok; ++i) {
            const int s = i % NS;
            if (!mbar_wait(&sm.full[s], (i / NS) & 1)) {
                set_status(a.status, SEKV_ERR_TIMEOUT);
                ok = false;
                break;
            }
            const unsigned char* st = sm.stages + (size_t)s * C::STAGE;
            const bool anchor_tile = i < nta;
            const int S0 = s0 + (i - nta) * TR;
            const int trows = anchor_tile ? min(TR, a1 - (a0 + i * TR)) : min(TR, s1 - S0);
            if (rbase < trows) {
                // ---- logits: q . K^T for the warp's 16 rows (two n-tiles of 8)
                float acc[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
                    const int row = rbase + 8 * nt + (lane & 7);
#pragma unroll
                    for (int p = 0; p < D / 32; ++p) {
                        const int chunk = (p & 1) * 4 + (lane >> 3);
                        uint32_t kb[4];
                        ldsm_x4(kb, st + (p >> 1) * 8192 + row * 128 + ((chunk ^ (row & 7)) << 4));
                        const uint32_t a0f[4] = {qa[2 * p][0], 0u, qa[2 * p][1], 0u};
                        const uint32_t a1f[4] = {qa[2 * p + 1][0], 0u, qa[2 * p + 1][1], 0u};
                        const uint32_t b0[2] = {kb[0], kb[1]};
                        const uint32_t b1[2] = {kb[2], kb[3]};
                        mma_bf16_16816(acc[nt], a0f, b0);
                        mma_bf16_16816(acc[nt], a1f, b1);
                    }
                }
                // ---- routing, zoom decisions, logits in the log2 domain
                float lg[2][2];
                if (anchor_tile) {
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int tk = rbase + 8 * nt + 2 * c + e;
                            lg[nt][e] = (gv && tk < trows) ? acc[nt][e] * sl2 : -INFINITY;
                        }
                } else {
                    const float* invn = reinterpret_cast<const float*>(st + 2 * C::TILE);
                    const float* lsv = invn + TR;
                    uint32_t zbal[2][2];
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int tk = rbase + 8 * nt + 2 * c + e;
                            const bool valid = gv && tk < trows;
                            const float x = acc[nt][e];
                            const float ls = lsv[tk];
                            const float ell = fmaf(x * invn[tk], a.scale, ls);     // Eq. (5) pre-sigmoid
                            const bool z = valid && (ell > th);                    // Eq. (9)
                            const int SL = S0 + tk;
                            if (valid && a.route_logits)
                                a.route_logits[(((int64_t)b * a.L + l) * a.Hq + kvh * G + g) * a.m_cap + SL] = ell;
                            if (z) atomicOr(&sm.zw[g * zwords + ((SL - s0) >> 5)], 1u << (SL & 31));
                            zbal[nt][e] = __ballot_sync(0xffffffffu, z);
                            lg[nt][e] = (valid && !z) ? fmaf(x, a.scale, ls) * kLog2e : -INFINITY;
                        }
                    if (!route_only) {
                        // queue every span of the warp's 16 rows that some head zooms
                        const int t = lane & 15;
                        const int tnt = t >> 3, tc = (t & 7) >> 1, te = t & 1;
                        const uint32_t zb = tnt ? (te ? zbal[1][1] : zbal[1][0]) : (te ? zbal[0][1] : zbal[0][0]);
                        uint32_t hm = 0u;
#pragma unroll
                        for (int h = 0; h < G; ++h) hm |= ((zb >> (4 * h + tc)) & 1u) << h;
                        const bool has = lane < 16 && rbase + t < trows && hm != 0u;
                        const uint32_t rows_with = __ballot_sync(0xffffffffu, has);
                        if (has) {
                            const int pos = qn + __popc(rows_with & ((1u << lane) - 1u));
                            if (pos < a.qcap) myq[pos] = (S0 + rbase + t) | (int)(hm << 24);
                        }
                        qn += __popc(rows_with);
                    }
                }
                if (!route_only) {
                    // ---- online softmax for head g over the warp's 16 rows
                    float mx = fmaxf(fmaxf(lg[0][0], lg[0][1]), fmaxf(lg[1][0], lg[1][1]));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                    const float mnew = fmaxf(mm, mx);
                    const float alpha = (mnew == -INFINITY) ? 1.f : exp2f(mm - mnew);
                    float p[2][2];
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 2; ++e) p[nt][e] = (lg[nt][e] == -INFINITY) ? 0.f : exp2f(lg[nt][e] - mnew);
                    float ps = p[0][0] + p[0][1] + p[1][0] + p[1][1];
                    ps += __shfl_xor_sync(0xffffffffu, ps, 1);
                    ps += __shfl_xor_sync(0xffffffffu, ps, 2);
                    lm = fmaf(lm, alpha, ps);
                    mm = mnew;
                    if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                        for (int n = 0; n < D / 8; ++n) {
                            oc[n][0] *= alpha;
                            oc[n][1] *= alpha;
                        }
                    }
                    // ---- O += P V (P as the A fragment: k = the 16 rows)
                    const uint32_t pa[4] = {pack_bf16(p[0][0], p[0][1]), 0u, pack_bf16(p[1][0], p[1][1]), 0u};
                    const unsigned char* vt = st + C::TILE;
                    const int mi = lane >> 3;
                    const int vrow = rbase + (lane & 7) + ((mi & 1) << 3);
#pragma unroll
                    for (int qd = 0; qd < D / 16; ++qd) {
                        const int chunk = (qd & 3) * 2 + (mi >> 1);
                        uint32_t vb[4];
                        ldsm_x4_t(vb, vt + (qd >> 2) * 8192 + vrow * 128 + ((chunk ^ (vrow & 7)) << 4));
                        const uint32_t b0[2] = {vb[0], vb[1]};
                        const uint32_t b1[2] = {vb[2], vb[3]};
                        mma_bf16_16816(oc[2 * qd], pa, b0);
                        mma_bf16_16816(oc[2 * qd + 1], pa, b1);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[s]);
        }
        if (lane == 0) sm.qcnt[warp] = ok ? min(qn, a.qcap) : 0;
    } else {
        // ------------------------------------------------ consumers, CUDA cores
        const int rL = lane / G, hL = lane % G;
        float q[G][DPL];
        {
            const char* qp = a.q + (((int64_t)b * a.L + l) * a.Hq + (int64_t)kvh * G) * C::ROWB +
                             lane * DPL * C::ESZ;
#pragma unroll
            for (int h = 0; h < G; ++h) Vec<DT, DPL>::load(qp + h * C::ROWB, q[h]);
        }
        const float th = a.theta[(int64_t)l * a.Hq + kvh * G + hL];
        float* pb = reinterpret_cast<float*>(base + 512) + warp * 32;     // per-warp tile p
        int qn = 0;
        int* myq = sm.zq + warp * a.qcap;
        const int rbase = warp * R;
        for (int i = 0; i < ntiles && ok; ++i) {
            const int s = i % NS;
            if (!mbar_wait(&sm.full[s], (i / NS) & 1)) {
                set_status(a.status, SEKV_ERR_TIMEOUT);
                ok = false;
                break;
            }
            const unsigned char* st = sm.stages + (size_t)s * C::STAGE;
            const bool anchor_tile = i < nta;
            const int S0 = s0 + (i - nta) * TR;
            const int trows = anchor_tile ? min(TR, a1 - (a0 + i * TR)) : min(TR, s1 - S0);
            float part[32];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float kk[DPL];
                if (rbase + r < trows) {
                    Vec<DT, DPL>::load(st + (rbase + r) * C::ROWB + lane * DPL * C::ESZ, kk);
                } else {
#pragma unroll
                    for (int k = 0; k < DPL; ++k) kk[k] = 0.f;
                }
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float acc = 0.f;
#pragma unroll
                    for (int k = 0; k < DPL; ++k) acc = fmaf(kk[k], q[h][k], acc);
                    part[r * G + h] = acc;
                }
            }
            const float x = transpose_reduce32(part, lane);
            const int rowL = rbase + rL;
            const bool validL = rowL < trows;
            float lg2 = -INFINITY;
            if (anchor_tile) {
                if (validL) lg2 = x * sl2;
            } else {
                const float invn = reinterpret_cast<const float*>(st + 2 * C::TILE)[rowL];
                const float ls = reinterpret_cast<const float*>(st + 2 * C::TILE + TR * 4)[rowL];
                const int SL = S0 + rowL;
                const float ell = fmaf(x * invn, a.scale, ls);      // Eq. (5) pre-sigmoid logit
                const bool z = validL && (ell > th);                // Eq. (9)
                if (validL && a.route_logits)
                    a.route_logits[(((int64_t)b * a.L + l) * a.Hq + kvh * G + hL) * a.m_cap + SL] = ell;
                if (z) atomicOr(&sm.zw[hL * zwords + ((SL - s0) >> 5)], 1u << (SL & 31));
                if (!route_only) {
                    const uint32_t zb = __ballot_sync(0xffffffffu, z);
                    const uint32_t hm = (zb >> (rL * G)) & ((1u << G) - 1u);
                    const bool head_lane = (hL == 0) && validL && hm != 0u;
                    const uint32_t rows_with = __ballot_sync(0xffffffffu, head_lane);
                    if (head_lane) {
                        const int pos = qn + __popc(rows_with & ((1u << lane) - 1u));
                        if (pos < a.qcap) myq[pos] = SL | (int)(hm << 24);
                    }
                    qn += __popc(rows_with);
                    if (validL && !z) lg2 = fmaf(x, a.scale, ls) * kLog2e;
                }
            }
            if (!route_only) {
                float mx = lg2;
#pragma unroll
                for (int off = G; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                const float m_lane_new = fmaxf(m_lane, mx);
                const float p = (lg2 == -INFINITY) ? 0.f : exp2f(lg2 - m_lane_new);
                float ps = p;
#pragma unroll
                for (int off = G; off < 32; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
                float alpha[G];
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float mnew = fmaxf(m_run[h], __shfl_sync(0xffffffffu, mx, h));
                    alpha[h] = (mnew == -INFINITY) ? 1.f : exp2f(m_run[h] - mnew);
                    l_run[h] = fmaf(l_run[h], alpha[h], __shfl_sync(0xffffffffu, ps, h));
                    m_run[h] = mnew;
                }
                m_lane = m_lane_new;
                pb[lane] = p;
                __syncwarp();
#pragma unroll
                for (int h = 0; h < G; ++h)
#pragma unroll
                    for (int k = 0; k < DPL; ++k) o[h][k] *= alpha[h];
                const unsigned char* vt = st + C::TILE;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    if (rbase + r < trows) {
                        float vv[DPL];
                        Vec<DT, DPL>::load(vt + (rbase + r) * C::ROWB + lane * DPL * C::ESZ, vv);
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float pr = pb[r * G + h];
#pragma unroll
                            for (int k = 0; k < DPL; ++k) o[h][k] = fmaf(pr, vv[k], o[h][k]);
                        }
                    }
                }
                __syncwarp();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[s]);
        }
        if (lane == 0) sm.qcnt[warp] = ok ? min(qn, a.qcap) : 0;
    }
    __syncthreads();    // the stream is done: the stage ring is free, the zoom queues are complete

    if (!route_only && warp < kNW && ok) {
        if constexpr (C::MMA) zoom_phase_mma<D, G>(a, sm, warp, lane, b, l, kvh, qa, mm, lm, oc);
        else zoom_phase<DT, D, G>(a, sm, warp, lane, b, l, kvh, m_run, l_run, o, m_lane);
    }
    __syncthreads();    // zoom slots and scratch are dead: the ring takes the partial states
    if (!route_only && warp < kNW) {
        if constexpr (C::MMA) {
            const int g = lane >> 2, c = lane & 3;
            if (g < G) {
                if (c == 0) {
                    sm.st_m[warp * G + g] = mm;
                    sm.st_l[warp * G + g] = lm;
                }
#pragma unroll
                for (int n = 0; n < D / 8; ++n) {
                    sm.st_o[(warp * G + g) * D + 8 * n + 2 * c] = oc[n][0];
                    sm.st_o[(warp * G + g) * D + 8 * n + 2 * c + 1] = oc[n][1];
                }
            }
        } else {
            store_state_lanes<D, G>(sm, warp, lane, m_run, l_run, o);
        }
    }
    __syncthreads();

    // ------------------------------------------------ zoom-mask words of this CTA
    if (a.zmask) {
        const int w0 = s0 >> 5;
        const int wend = (split == a.nsplit - 1) ? a.mw : min(a.mw, w0 + (sch >> 5));
        for (int i = tid; i < G * max(0, wend - w0); i += blockDim.x) {
            const int h = i / (wend - w0), j = i % (wend - w0);
            a.zmask[(((int64_t)b * a.L + l) * a.Hq + kvh * G + h) * a.mw + w0 + j] =
                (j < zwords) ? sm.zw[h * zwords + j] : 0u;
        }
    }
    if (route_only) return;

    // ------------------------------------------------ merge the partial states of this CTA
    for (int i = tid; i < G * D; i += blockDim.x) {
        const int h = i / D, k = i % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < C::NSTATE; ++w) M = fmaxf(M, sm.st_m[w * G + h]);
        float Ls = 0.f, Os = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < C::NSTATE; ++w) {
                const float f = exp2f(sm.st_m[w * G + h] - M);
                Ls = fmaf(sm.st_l[w * G + h], f, Ls);
                Os = fmaf(sm.st_o[(w * G + h) * D + k], f, Os);
            }
        }
        const int64_t pidx = (lunit * G + h) * a.nsplit + split;
        a.part_o[pidx * D + k] = Os;
        if (k == 0) {
            a.part_ml[pidx * 2 + 0] = M;
            a.part_ml[pidx * 2 + 1] = Ls;
        }
    }
}

// one CTA of D threads per (b, l, query head)
template <int D>
__global__ void merge_kernel(const float* part_o, const float* part_ml, float* O, float* lse, int nsplit,
                             int G, int Hkv, int L, int l0, int Lr, int Hq) {
    const int idx = blockIdx.x;
    const int hq = idx % Hq;
    const int li = (idx / Hq) % Lr;
    const int b = idx / (Hq * Lr);
    const int kvh = hq / G, h = hq % G;
    const int64_t lunit = ((int64_t)b * Lr + li) * Hkv + kvh;
    const int64_t base = (lunit * G + h) * nsplit;
    const int k = threadIdx.x;
    float M = -INFINITY;
    for (int j = 0; j < nsplit; ++j) M = fmaxf(M, part_ml[(base + j) * 2]);
    float Ls = 0.f, Os = 0.f;
    if (M != -INFINITY) {
        for (int j = 0; j < nsplit; ++j) {
            const float f = exp2f(part_ml[(base + j) * 2] - M);
            Ls = fmaf(part_ml[(base + j) * 2 + 1], f, Ls);
            Os = fmaf(part_o[(base + j) * D + k], f, Os);
        }
    }
    const int64_t out = ((int64_t)b * L + l0 + li) * Hq + hq;
    O[out * D + k] = Ls > 0.f ? Os / Ls : 0.f;
    if (k == 0) lse[out] = Ls > 0.f ? (M + log2f(Ls)) * kLn2 : -INFINITY;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static int num_sms() {
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms > 0 ? sms : 148;
}

bool decode_supported(const sekv_decode_desc& d) {
    const int G = d.Hkv > 0 ? d.Hq / d.Hkv : 0;
    return (d.d == 64 || d.d == 128) && (G == 1 || G == 2 || G == 4 || G == 8) && d.rank >= 1 &&
           d.rank <= kRMax && (d.dtype == SEKV_F32 || d.dtype == SEKV_BF16);
}

DecodePlan plan_decode(const sekv_decode_desc& d) {
    DecodePlan p{};
    const int Lr = d.l1 - d.l0;
    const int64_t units = (int64_t)d.B * Lr * d.Hkv;
    int ns = d.nsplit;
    const int max_ns = d.m_cap / 32 > 0 ? d.m_cap / 32 : 1;
    if (ns <= 0) {
        // Fill whole waves of resident CTAs (3 per SM for the bf16 / d=128 / G=4
        // variant): the smallest split count with >= 1.5 waves and >= 85% of the
        // last wave busy; otherwise the best such ratio. Splits keep >= ~128 rows.
        const double slots = 3.0 * num_sms();
        int lim = (int)((d.a_cap + d.m_cap) / 128);
        lim = lim < 1 ? 1 : (lim > max_ns ? max_ns : lim);
        if (lim > 64) lim = 64;
        int best = 1;
        double best_score = -1.0;
        for (int c = 1; c <= lim; ++c) {
            const double waves = (double)units * c / slots;
            const double eff = waves / std::ceil(waves);
            if (waves >= 1.5 && eff >= 0.85) { best = c; break; }
            const double score = eff * (waves < 2.0 ? waves / 2.0 : 1.0);
            if (score > best_score + 1e-9) { best_score = score; best = c; }
        }
        ns = best;
    }
    if (ns > max_ns) ns = max_ns;
    if (ns < 1) ns = 1;
    p.nsplit = ns;
    p.span_chunk = (int)round_up((d.m_cap + ns - 1) / ns, 32);
    p.anchor_chunk = (d.a_cap + ns - 1) / ns;
    const int G = d.Hq / d.Hkv;
    p.partial_bytes = (size_t)round_up((int64_t)units * G * ns * (d.d + 2) * 4, 256);
    return p;
}

size_t decode_workspace_bytes(const sekv_decode_desc& d) { return plan_decode(d).partial_bytes; }

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// [rows][d] bf16 viewed with 64 x 64 boxes (128-byte rows of the box) and 128-byte swizzle
static bool encode_rows(CUtensorMap* m, const void* base, int64_t rows, int d) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || !base) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    const cuuint32_t box[2] = {64, 64};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DT, int D, int G>
static cudaError_t launch_t(const sekv_decode_desc& d, const DecodePlan& p, void* partials, cudaStream_t st) {
    using C = DecCfg<DT, D, G>;
    const int Lr = d.l1 - d.l0;
    const int64_t units = (int64_t)d.B * Lr * d.Hkv;
    DecArgs a;
    a.q = (const char*)d.q;
    a.a_count = d.a_count; a.m_count = d.m_count; a.span_beg = d.span_beg; a.span_end = d.span_end;
    a.logS = d.logS; a.blk_off = d.blk_off;
    a.Ka = (const char*)d.Ka; a.Va = (const char*)d.Va; a.kbar = (const char*)d.kbar; a.vbar = (const char*)d.vbar;
    a.inv_norm = d.inv_norm; a.theta = d.theta; a.arena = (const char*)d.arena; a.slot = d.slot;
    a.zmask = d.zmask; a.route_logits = d.route_logits; a.status = d.dev_status;
    a.part_o = reinterpret_cast<float*>(partials);
    a.part_ml = a.part_o + units * G * p.nsplit * D;
    a.region = d.region_elems; a.scale = d.scale;
    a.L = d.L; a.l0 = d.l0; a.Lr = Lr; a.Hq = d.Hq; a.Hkv = d.Hkv; a.a_cap = d.a_cap; a.m_cap = d.m_cap;
    a.rank = d.rank; a.phase = d.phase; a.nsplit = p.nsplit; a.sch_max = p.span_chunk;
    a.qcap = ((p.span_chunk + C::TR - 1) / C::TR) * C::R;
    a.mw = d.m_cap / 32;
    const size_t smem = decode_smem_bytes<DT, D, G>(a.sch_max, a.qcap);
    if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<DT, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    DecMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    if (C::MMA) {
        const int64_t units_all = (int64_t)d.B * d.L * d.Hkv;
        bool ok = encode_rows(&maps.kbar, d.kbar, units_all * d.m_cap, D);
        if (d.phase != SEKV_ROUTE) {
            ok = ok && encode_rows(&maps.vbar, d.vbar, units_all * d.m_cap, D) &&
                 encode_rows(&maps.Ka, d.Ka, units_all * d.a_cap, D) &&
                 encode_rows(&maps.Va, d.Va, units_all * d.a_cap, D);
        }
        if (!ok) return cudaErrorInvalidValue;
    }
    dim3 grid(p.nsplit, d.Hkv, d.B * Lr);
    decode_kernel<DT, D, G><<<grid, (kNW + 1) * 32, smem, st>>>(a, maps);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (d.phase != SEKV_ROUTE) {
        merge_kernel<D><<<d.B * Lr * d.Hq, D, 0, st>>>(a.part_o, a.part_ml, d.O, d.lse, p.nsplit, G, d.Hkv,
                                                        d.L, d.l0, Lr, d.Hq);
        e = cudaGetLastError();
    }
    return e;
}

template <int DT, int D>
static cudaError_t launch_g(const sekv_decode_desc& d, const DecodePlan& p, void* w, cudaStream_t st) {
    switch (d.Hq / d.Hkv) {
        case 1: return launch_t<DT, D, 1>(d, p, w, st);
        case 2: return launch_t<DT, D, 2>(d, p, w, st);
        case 4: return launch_t<DT, D, 4>(d, p, w, st);
        default: return launch_t<DT, D, 8>(d, p, w, st);
    }
}

// ---------------------------------------------------------------------------
// Split-K partials for callers that pass no workspace: one static device array,
// present on every device that loads this library until the process exits.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_decode_scratch[SEKV_STATIC_SCRATCH_BYTES];

size_t decode_static_scratch_bytes() { return SEKV_STATIC_SCRATCH_BYTES; }

// Device address of g_decode_scratch on the current device. In host code the
// array's name only stands in for it, so the address is looked up once per
// device (with that device current) and cached.
void* decode_static_scratch(cudaError_t* err) {
    static std::mutex mu;
    static void* addr[256] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 256) {
        *err = e != cudaSuccess ? e : cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
        if (e != cudaSuccess || !ptr) {
            *err = e != cudaSuccess ? e : cudaErrorInvalidSymbol;
            return nullptr;
        }
        addr[dev] = ptr;
    }
    *err = cudaSuccess;
    return addr[dev];
}

cudaError_t launch_decode(const sekv_decode_desc& d, const DecodePlan& p, void* partials, cudaStream_t st) {
    if (d.dtype == SEKV_F32)
        return d.d == 64 ? launch_g<SEKV_F32, 64>(d, p, partials, st) : launch_g<SEKV_F32, 128>(d, p, partials, st);
    return d.d == 64 ? launch_g<SEKV_BF16, 64>(d, p, partials, st) : launch_g<SEKV_BF16, 128>(d, p, partials, st);
}

}  // namespace sekv
