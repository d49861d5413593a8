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
//         (mma.sync m16n8k16, the rows on M and the G query heads of the kv head
//         on N, padded to 8: GQA, one K/V read serves all G heads). The q.kbar
//         accumulator of a span row is both its routing logit and its coarse
//         attention logit. A routing pass loads key tiles only, two per stage.
//   fp32: 1-D bulk copies and CUDA-core dot products (each lane owns d/32 dims,
//         a 32-way transpose-reduce finishes the dots).
// Spans zoomed by any head of the group are queued. Phase 2 attends them without
// materialising K_S (u = B_S q, scores A_S u, y = C_S^T p, contribution y^T D_S):
//   bf16: the producer warp streams each queued span's factor pieces through one
//         CTA-wide ring; the consumer warps share every span (all four, or one
//         pair for ranks above 16), 32 tokens at a time, on the tensor cores with
//         u, p and y held in registers. With the mask given and a grid of about
//         one wave, the unit's zoomed token units are dealt evenly over its splits
//         instead.
//   fp32: each consumer warp pulls whole spans and streams them through its own
//         3-slot ring, on the CUDA cores.
// Softmax state is kept in the log2 domain; the CTA merges its warps' states, and
// the last CTA of each (b, l, kv head) to finish merges the splits by log-sum-exp
// (arrival counters; without them a second small kernel does).
#include <cuda.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "sekv_common.cuh"
#include "sekv_internal.h"

namespace sekv {

constexpr int kNW = 4;          // consumer warps per CTA
constexpr unsigned kSpanModeSpans = 64;   // zoomed spans in a CTA for whole-span pieces
constexpr int kRMax = 64;       // largest basis rank the decode accepts
constexpr size_t kDealMaskBytes = 5632;   // largest unit mask + unit table ((G + 1) x m_cap / 32 words) for dealing

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
    static constexpr int NS0 = (MMA ? 68 * 1024 : 64 * 1024) / STAGE;     // 3 CTAs / SM on the bf16 path
    static constexpr int NS = NS0 < 2 ? 2 : (NS0 > 6 ? 6 : NS0);   // ring depth
    static constexpr int YPL = kRMax * G / 32;              // y entries per lane (fp32 zoom)
    static constexpr int WSCR = MMA ? 0 : (64 * G) + 2 * kRMax * G;   // per-warp scratch floats (fp32 zoom)
    // fp32 zoom phase: per-warp ring of ZNS slots of ZSLOT bytes, carved from the stage ring
    static constexpr int ZNS = 3;
    static constexpr int ZSLOT = 4096;
    static constexpr int RB = ZSLOT / ROWB;                 // B / D rows per slot (a multiple of 8)
    static constexpr int ZBYTES = kNW * ZNS * ZSLOT;
    // tensor-core zoom phase: one CTA-wide ring of slots (ZRing below) filled by the
    // producer warp and read by all consumer warps, sized here for the largest slot
    static constexpr int ZSLOTC = 16384;
    static constexpr int RBC = ZSLOTC / ROWB;               // B / D rows per piece (a multiple of 16)
    static constexpr int ZNSC0 = (NS * STAGE) / ZSLOTC;
    static constexpr int ZNSC = ZNSC0 > 16 ? 16 : ZNSC0;
    // partial softmax states merged at the end, one per consumer warp
    static constexpr int NSTATE = kNW;
    static constexpr int SBYTES = NSTATE * (G * D + 2 * G) * 4;
    static constexpr int RING0 = NS * STAGE;
    static constexpr int ZRING = MMA ? ZNSC * ZSLOTC : ZBYTES;
    static constexpr int RING1 = ZRING > SBYTES ? ZRING : SBYTES;
    static constexpr int RING = RING0 > RING1 ? RING0 : RING1;
    static constexpr int HDR = 1024;                        // mbarriers + counters (keeps stages 1 KB aligned)
};

// The tensor-core zoom ring in the stream stages' memory: 16 KB slots (measured on
// B200 against 8 KB slots, which keep twice as many pieces in flight: the 128K
// default workload's ATTEND call was ~3 % faster with 16 KB). The variant that hands
// small spans whole to one warp needs a span's block in one slot as well.
constexpr int kMaxZSlots = 16;   // zfull / zempty barriers and piece descriptors in the header
template <class C, bool SP>
struct ZRing {
    static constexpr int SLOT = 16384;
    static constexpr int RB = SLOT / C::ROWB;               // B / D rows per piece (a multiple of 16)
    static constexpr int NS0 = C::RING0 / SLOT;
    static constexpr int NS = NS0 > kMaxZSlots ? kMaxZSlots : NS0;
    static_assert(NS * SLOT <= C::RING, "zoom ring exceeds the stage memory");
    static_assert(RB % 16 == 0, "B / D pieces must hold whole 16-row blocks");
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
    int B, L, l0, Lr, Hq, Hkv, a_cap, m_cap, rank, phase, nsplit, sch_max, qcap, mw;
    int zin;          // zoom decisions come from zmask (a capped mask) instead of l > theta
    int deal;         // zin, tensor-core path: the unit's whole mask is in shared memory and
                      // every split takes an even share of the unit's zoomed token units
    int zwords;       // zoom-mask words per head in shared memory (the split's span range)
    uint32_t polls;   // poll limit of every bounded barrier wait
    int starve;       // test hook: the producer issues no copy, so every wait runs out
    int static_ready; // the build outputs are settled: counts and first tiles are read before the dependency wait
    uint32_t* arrive; // [B][L][Hkv] arrival counters (the last CTA of a unit merges), or null
    float* O;         // [B][L][Hq][D] and [B][L][Hq]: written by the merging CTA
    float* lse;
};

// zoom bit of span S for query head hq of (b, l) in a caller-supplied (capped) mask
SEKV_DEV bool zmask_bit(const DecArgs& a, int b, int l, int hq, int S) {
    const uint32_t w = a.zmask[(((int64_t)b * a.L + l) * a.Hq + hq) * a.mw + (S >> 5)];
    return (w >> (S & 31)) & 1u;
}

// TMA descriptors of the anchor and summary stores (bf16 path), viewed as 2-D
// [rows][d] tensors with 64 x 64 boxes and 128-byte swizzle.
struct DecMaps {
    CUtensorMap Ka, Va, kbar, vbar;
};

template <int DT, int D, int G>
static size_t decode_smem_bytes(int zwords, int qcap, int deal) {
    using C = DecCfg<DT, D, G>;
    size_t s = C::HDR;
    s += (size_t)C::RING;
    s += (size_t)kNW * qcap * 4;                               // zoom queues
    s += (size_t)G * zwords * 4;                               // zoom-mask words
    s += deal ? (size_t)zwords * 4 : 0;                        // zoomed token units per word
    s += (size_t)kNW * C::WSCR * 4;                            // per-warp scratch
    s = round_up(s, 16) + (size_t)G * C::ROWB;                 // the group's query rows
    return round_up(s, 128) + 1024;                            // + alignment slack
}

// A zoomed span as the fp32 zoom pipeline sees it (warp-uniform values).
struct ZSpan {
    const char* blk;     // the span's block for this kv head
    int S;
    uint32_t hm;         // query heads of the group that zoom it
    int len, rS, nB, nAC, TC;
    int64_t pa;          // elements of the A (and of the C) section
    bool valid;
};

// One piece of the tensor-core zoom stream: what a ring slot holds. Written by
// the producer before it arms the slot's full barrier (a release), read by the
// consumers after their wait on it (an acquire).
// ZP_SPAN: a whole span's block [A | C | B | D] in one slot, handled by one warp.
// ZP_MIX: parts of one span packed into a slot, in order: the whole B (flag 1,
// at offset 0), the A and C rows of tokens [r0, r0 + cnt) (each part reserved for
// roundup(cnt, 32) tokens), the whole D (flag 2, reserved for roundup(r8, 16) rows).
// ZP_B / ZP_D: chunks of B or D rows in slots of their own (for ranks whose B or D
// takes more than half a slot).
enum : int { ZP_B = 0, ZP_D = 2, ZP_END = 3, ZP_SPAN = 4, ZP_MIX = 5 };
constexpr int kMixB = 1, kMixD = 2;
struct __align__(16) ZPiece {
    int kind;
    int first;           // B / D chunks: first chunk of its span; MIX: kMixB | kMixD flags
    int r0;              // B / D: first basis row; MIX: first token (span-local, a multiple of 32)
    int cnt;             // B / D: basis rows (a multiple of 8); MIX: tokens (may be 0)
    int len, rS;
    uint32_t hm;         // query heads of the group that zoom the span
    int rot;             // B / MIX / D: the span's 32-token unit j belongs to consumer warp
                         // (j + rot) % 4 for ranks <= 16, and to 2 (rot / 2) + (j + rot) % 2
                         // (one pair of warps per span) above; SPAN: the warp that handles
                         // the whole span
};

// shared-memory carve-up common to both paths
struct DecSmem {
    uint64_t* full;      // [NS]
    uint64_t* empty;     // [NS]
    uint64_t* zbar;      // fp32 zoom: [kNW][ZNS]
    uint64_t* zfull;     // tensor-core zoom: [ZNSC]
    uint64_t* zempty;    // tensor-core zoom: [ZNSC]
    int* qcnt;           // [kNW]
    int* zq_next;
    int* sfail;          // set when any warp gave up during the stream phase
    int* last;           // this CTA is the unit's last to finish (it merges the splits)
    ZPiece* zmeta;       // tensor-core zoom: [ZNSC]
    unsigned char* stages;
    int* zq;             // [kNW][qcap]
    uint32_t* zw;        // [G][zwords]
    int* zu;             // deal: [zwords] zoomed 32-token units of the spans of each mask word
    float* wscr;         // [kNW][WSCR]
    unsigned char* qs;   // [G][D] query rows of the kv head's group (storage dtype)
    float* st_m;         // [NSTATE][G]   (in the ring, once the zoom phase is over)
    float* st_l;         // [NSTATE][G]
    float* st_o;         // [NSTATE][G][D]
};

// header (HDR = 1024 bytes): full @0, empty @64, zbar / zfull @128, zempty @256,
// counters @384, zmeta @512 (tensor-core path; the fp32 path keeps its per-warp
// p tiles there)
template <class C, int G, int D>
SEKV_DEV DecSmem carve_smem(unsigned char* base, int qcap, int zwords, int deal) {
    DecSmem s;
    s.full = reinterpret_cast<uint64_t*>(base);
    s.empty = s.full + 8;
    s.zbar = s.full + 16;
    s.zfull = s.full + 16;
    s.zempty = s.full + 32;
    s.qcnt = reinterpret_cast<int*>(base + 384);
    s.zq_next = s.qcnt + kNW;
    s.sfail = s.zq_next + 1;
    s.last = s.sfail + 1;
    s.zmeta = reinterpret_cast<ZPiece*>(base + 512);
    s.stages = base + C::HDR;
    s.zq = reinterpret_cast<int*>(s.stages + C::RING);
    s.zw = reinterpret_cast<uint32_t*>(s.zq + kNW * qcap);
    s.zu = reinterpret_cast<int*>(s.zw + G * zwords);
    s.wscr = reinterpret_cast<float*>(s.zu + (deal ? zwords : 0));
    s.qs = reinterpret_cast<unsigned char*>(
        round_up(reinterpret_cast<uintptr_t>(s.wscr + kNW * C::WSCR), 16));
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
        int tc = (C::ZSLOT / 2) / (round8(sp.rS) * C::ESZ);
        tc = tc > 64 ? 64 : tc;
        sp.TC = (tc & ~7) < 8 ? 8 : (tc & ~7);
        sp.nB = (round8(sp.rS) + C::RB - 1) / C::RB;
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
                    const int sr8 = round8(srS);
                    const uint32_t bytes = (uint32_t)min(C::RB, sr8 - r0) * C::ROWB;
                    const char* src = sblk + (2 * spa + (isD ? (int64_t)sr8 * D : 0) + (int64_t)r0 * D) * C::ESZ;
                    mbar_arrive_expect_tx(&zb[slot], bytes);
                    bulk_g2s(dst, src, bytes, &zb[slot]);
                } else {
                    const int t0 = (k - snB) * sTC;
                    const int nt = min(sTC, slen - t0);
                    const uint32_t bytes = (uint32_t)((int64_t)round8(nt) * round8(srS) * C::ESZ);
                    const int64_t off = (int64_t)t0 * round8(srS) * C::ESZ;
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
            if (!mbar_wait_n(&zb[slot], (ncons / C::ZNS) & 1, a.polls)) {
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
                            Vec<DT, DPL>::load(zs + tile8_index(i0 + r, lane * DPL, D) * C::ESZ, kk);
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
                const int rS = cur.rS, r8 = round8(cur.rS);
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
                                const uint4 w = *reinterpret_cast<const uint4*>(As + tile8_index(t, i0, r8) * 2);
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
                                const float av = load1<DT>(As, tile8_index(t, i, r8));
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
                            acc0 = fmaf(pb[(tt + 0) * G + hL], load1<DT>(Cs, tile8_index(tt + 0, i, r8)), acc0);
                            acc1 = fmaf(pb[(tt + 1) * G + hL], load1<DT>(Cs, tile8_index(tt + 1, i, r8)), acc1);
                            acc2 = fmaf(pb[(tt + 2) * G + hL], load1<DT>(Cs, tile8_index(tt + 2, i, r8)), acc2);
                            acc3 = fmaf(pb[(tt + 3) * G + hL], load1<DT>(Cs, tile8_index(tt + 3, i, r8)), acc3);
                        }
                        for (; tt < nt; ++tt)
                            acc0 = fmaf(pb[tt * G + hL], load1<DT>(Cs, tile8_index(tt, i, r8)), acc0);
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
                    Vec<DT, DPL>::load(zs + tile8_index(r, lane * DPL, D) * C::ESZ, dv);
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
        if (!mbar_wait_n(&zb[ncons % C::ZNS], (ncons / C::ZNS) & 1, a.polls)) set_status(a.status, SEKV_ERR_TIMEOUT);
        ++ncons;
    }
}

// ---------------------------------------------------------------------------
// Phase 2 on the tensor cores (bf16). The producer warp reads the CTA's zoom
// bitmask (span order) and streams, per zoomed span, its B rows, its A/C token
// groups and its D rows through one CTA-wide ring of 16 KB slots; every consumer
// warp reads every slot. Per span, with r8 = roundup(r_S, 8) and the heads h that
// zoom it (heads on the mma N side, as on the stream path):
//   u    = B_S q        (M = basis rows, N = heads, K = d)
//   s    = A_S u        (M = tokens,     N = heads, K = r8)  -> online softmax p
//   y   += C_S^T p      (M = basis rows, N = heads, K = tokens)
//   O^T += D_S^T (beta y)  into the warp's stream accumulators
// An accumulator becomes the next product's B fragment through an 8 x 8 register
// transpose, so u, p and y never leave registers. The span's 32-token units are
// dealt round-robin to the four consumer warps (continuing across spans); a warp
// with no unit in a span skips it. u (pre-scaled by scale * log2 e) enters as a
// hi + lo bf16 pair (about 16 significant bits); p and beta*y are rounded to
// bf16 as p on the stream path.
// ---------------------------------------------------------------------------
// split v0, v1 into a hi + lo bf16x2 pair
SEKV_DEV void split_bf16x2(float v0, float v1, uint32_t& hi, uint32_t& lo) {
    hi = pack_bf16(v0, v1);
    lo = pack_bf16(v0 - bf16_lo(hi), v1 - bf16_hi(hi));
}

// hardware 2^x (ex2.approx.ftz: relative error ~2^-22; 2^-inf = 0)
SEKV_DEV float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// zoomed spans of the CTA: word w of zw[h] holds head h's bits for spans
// s0 + 32 w .. s0 + 32 w + 31; nwords words are in use. With a.deal the words are
// the unit's (s0 = 0) and this split takes an even share of the unit's zoomed
// 32-token units: the zoomed spans (any head of the group) in span order, span S
// contributing ceil(|S| / 32) units, split j the units [U j / nsplit, U (j + 1) / nsplit).
// A span cut between splits is attended in parts (each part its own u = B q and
// D projection): the parts are disjoint subsets of the one softmax's entries.
template <int D, int G, bool SP>
SEKV_DEV void zoom_produce(const DecArgs& a, const DecSmem& sm, int lane, int b, int l, int kvh, int s0, int nwords,
                           int zwords, int split) {
    using C = DecCfg<SEKV_BF16, D, G>;
    using Z = ZRing<C, SP>;
    constexpr int ZNS = Z::NS, ZSL = Z::SLOT, RBC = Z::RB;
    constexpr uint32_t FULL = 0xffffffffu;
    uint32_t np = 0;          // pieces armed
    bool good = true;
    // Shared spans: for ranks <= 16 a span's units are dealt round-robin over the four
    // consumer warps, continuing across spans. Above, u = B q and the D projection
    // (done by every warp that takes part in a span) cost more, so a span goes to one
    // of two pairs of warps, its units alternating between the pair's warps: two
    // spans in flight at once, and half the u / D work (C5, rank 32: -8 % per call;
    // at rank 16 the two forms measured within 2 %). A span goes to the pair with less
    // work queued (its units + ~4 units' worth for u and D); each pair's next span
    // continues its unit parity. Whole-span pieces rotate over the warps.
    const bool pairs = a.rank > 16;
    int owner = 0, rot = 0, pw[2] = {0, 0}, ps[2] = {0, 0};
    // Whole-span pieces (one warp per small span, no repeated u / D work) pay off
    // when the CTA has enough zoomed spans to keep the four consumer warps busy
    // with different spans; with few, sharing each span's units across the warps
    // keeps the critical path shorter.
    bool span_mode = false;
    if (SP && !a.deal) {
        unsigned nz = 0;
        for (int w = lane; w < nwords; w += 32) {
            uint32_t m = 0u;
#pragma unroll
            for (int h = 0; h < G; ++h) m |= sm.zw[h * zwords + w];
            nz += __popc(m);
        }
        span_mode = warp_sum_u(nz) >= kSpanModeSpans;
    }
    // the slots were last read through the generic proxy (stream phase)
    fence_proxy_async();
    // arm the next slot with piece pc and up to four bulk copies (lane 0 issues):
    // part k lands at byte offset off[k] of the slot
    auto emit = [&](const ZPiece& pc, int nparts, const uint32_t (&off)[4], const char* const (&src)[4],
                    const uint32_t (&bytes)[4]) {
        int okk = 1;
        if (lane == 0) {
            const int slot = (int)(np % ZNS);
            if (np >= (uint32_t)ZNS && !mbar_wait_n(&sm.zempty[slot], ((np / ZNS) - 1) & 1, a.polls)) okk = 0;
            if (okk) {
                sm.zmeta[slot] = pc;
                unsigned char* dst = sm.stages + (size_t)slot * ZSL;
                uint32_t tot = 0;
                for (int k = 0; k < nparts; ++k) tot += bytes[k];
                if (tot == 0) {
                    mbar_arrive(&sm.zfull[slot]);
                } else {
                    mbar_arrive_expect_tx(&sm.zfull[slot], tot);
                    for (int k = 0; k < nparts; ++k)
                        if (bytes[k]) {
                            // zoom-dense calls (whole-span pieces) measured faster without
                            // the evict-first policy on their many small block copies
                            if constexpr (SP) bulk_g2s(dst + off[k], src[k], bytes[k], &sm.zfull[slot]);
                            else bulk_g2s_ef(dst + off[k], src[k], bytes[k], &sm.zfull[slot], l2_evict_first());
                        }
                }
            } else {
                set_status(a.status, SEKV_ERR_TIMEOUT);
            }
        }
        okk = __shfl_sync(FULL, okk, 0);
        if (okk) ++np;
        good = good && okk;
    };
    auto emit1 = [&](const ZPiece& pc, const char* src0, uint32_t n0) {
        const uint32_t off[4] = {0u, 0u, 0u, 0u}, by[4] = {n0, 0u, 0u, 0u};
        const char* const sr[4] = {src0, nullptr, nullptr, nullptr};
        emit(pc, 1, off, sr, by);
    };
    // the pieces of tokens [tb, te) of a zoomed span of jl tokens whose Hkv blocks start
    // at element jo of the arena (tb a multiple of 32; the whole span: 0, jl)
    auto emit_span = [&](int jl, uint32_t jhm, long long jo, int tb, int te) {
        const int rS = block_rank(jl, D, a.rank), r8 = round8(rS);
        const int64_t pa = block_ac_elems(jl, rS);
        const int64_t be = 2 * pa + 2 * (int64_t)r8 * D;
        const char* blk = a.arena + ((int64_t)jo + (int64_t)kvh * be) * 2;
        ZPiece pc;
        pc.len = te - tb;
        pc.rS = rS;
        pc.hm = jhm;
        if (span_mode && tb == 0 && te == jl && be * 2 + D * 16 <= ZSL) {
            // the whole block fits one slot (with room for the D projection's
            // read of one 8-row block past D): one piece, one owner warp
            pc.rot = owner;
            pc.kind = ZP_SPAN; pc.first = 1; pc.r0 = 0; pc.cnt = jl;
            emit1(pc, blk, (uint32_t)(be * 2));
            owner = (owner + 1) & 3;
            return;
        }
        // B, then the A / C rows of the tokens, then D, packed into as few slots
        // as they fit (B or D of more than half a slot travel in chunks of their
        // own). Every part is reserved with the rows its fragment loads read:
        // tokens up to a multiple of 32, basis rows up to a multiple of 16.
        {
            const int nu = (te - tb + 31) >> 5;
            if (pairs) {
                const int pr = pw[1] < pw[0] ? 1 : 0;
                pc.rot = 2 * pr + ps[pr];
                ps[pr] = (ps[pr] + nu) & 1;
                pw[pr] += nu + 4;
            } else {
                pc.rot = rot;
                rot = (rot + nu) & 3;
            }
        }
        const uint32_t bsz = (uint32_t)r8 * D * 2;                 // bytes of B (and of D)
        const uint32_t dres = (uint32_t)((r8 + 15) & ~15) * D * 2;
        const uint32_t tokb = 4u * r8;                              // A + C bytes per token
        const bool pack = bsz <= (uint32_t)ZSL / 2;
        const char* srcB = blk + (2 * pa) * 2;
        const char* srcD = blk + (2 * pa + (int64_t)r8 * D) * 2;
        if (!pack) {
            for (int r0 = 0; r0 < r8 && good; r0 += RBC) {
                pc.kind = ZP_B; pc.first = r0 == 0; pc.r0 = r0; pc.cnt = min(RBC, r8 - r0);
                emit1(pc, srcB + (int64_t)r0 * D * 2, (uint32_t)pc.cnt * C::ROWB);
            }
        }
        bool with_b = pack;
        for (int t0 = tb; t0 < te && good;) {
            const uint32_t room = (uint32_t)ZSL - (with_b ? bsz : 0u);
            const int tmax = (int)(room / tokb) & ~31;
            const int cnt = min(tmax, te - t0);
            const uint32_t res = (uint32_t)((cnt + 31) & ~31) * r8 * 2;   // bytes reserved for A (and C)
            const bool last = t0 + cnt >= te;
            const bool with_d = pack && last && room >= 2 * res + dres;
            pc.kind = ZP_MIX; pc.first = (with_b ? kMixB : 0) | (with_d ? kMixD : 0); pc.r0 = t0 - tb; pc.cnt = cnt;
            const uint32_t oa = with_b ? bsz : 0u, ab = (uint32_t)round8(cnt) * r8 * 2;
            const uint32_t off[4] = {0u, oa, oa + res, oa + 2 * res};
            const char* const sr[4] = {srcB, blk + (int64_t)t0 * r8 * 2, blk + (pa + (int64_t)t0 * r8) * 2, srcD};
            const uint32_t by[4] = {with_b ? bsz : 0u, ab, ab, with_d ? bsz : 0u};
            emit(pc, 4, off, sr, by);
            t0 += cnt;
            with_b = false;
            if (last && pack && !with_d && good) {                 // D in a slot of its own
                pc.kind = ZP_MIX; pc.first = kMixD; pc.r0 = t0 - tb; pc.cnt = 0;
                emit1(pc, srcD, bsz);
            }
        }
        if (!pack) {
            for (int r0 = 0; r0 < r8 && good; r0 += RBC) {
                pc.kind = ZP_D; pc.first = r0 == 0; pc.r0 = r0; pc.cnt = min(RBC, r8 - r0);
                emit1(pc, srcD + (int64_t)r0 * D * 2, (uint32_t)pc.cnt * C::ROWB);
            }
        }
    };
    // span S: its length (0 when invalid) and block offset (-1 when cold); the bounds
    // and the offset are loaded together (one round trip)
    auto span_look = [&](int S, int& len, long long& off) {
        const int64_t si = (int64_t)b * a.m_cap + S;
        const int beg = a.span_beg[si], end = a.span_end[si];
        const long long o = a.slot ? a.slot[((int64_t)b * a.L + l) * a.m_cap + S]
                                   : ((int64_t)b * a.L + l) * a.region + a.blk_off[(int64_t)b * (a.m_cap + 1) + S];
        len = end - beg;
        off = -1;
        if (len < 1) {
            set_status(a.status, SEKV_ERR_INVALID_ARG);
            len = 0;
        } else {
            off = o;
            if (off < 0) set_status(a.status, SEKV_ERR_COLD_SPAN);
        }
    };
    // Walk the zoomed spans (any head of the group) in span order, up to 32 at a time:
    // visit(len, hm, off, n) gets this lane's span of the batch (len 0: none or
    // invalid; off < 0: cold) and the batch size n (warp-uniform); it returns false
    // to stop the walk.
    auto walk = [&](auto&& visit) {
        for (int w0 = 0; w0 < nwords && good; w0 += 32) {
            // lane j takes word w0 + j: spans zoomed by any head, counted and scanned
            const int wi = w0 + lane;
            uint32_t m = 0u;
            if (wi < nwords) {
#pragma unroll
                for (int h = 0; h < G; ++h) m |= sm.zw[h * zwords + wi];
            }
            const int cnt = __popc(m);
            int inc = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(FULL, inc, o);
                if (lane >= o) inc += t;
            }
            const int total = __shfl_sync(FULL, inc, 31);
            for (int e0 = 0; e0 < total && good; e0 += 32) {
                // lane j resolves entry e0 + j: its word, bit, heads and block offset
                const int e = e0 + lane;
                int k = 0;
                for (int j = 0; j < 32; ++j) k += (__shfl_sync(FULL, inc, j) <= e) ? 1 : 0;
                const int kw = k < 32 ? k : 31;
                const int inck = __shfl_sync(FULL, inc, kw), cntk = __shfl_sync(FULL, cnt, kw);
                const uint32_t mk = __shfl_sync(FULL, m, kw);
                int len = 0;
                uint32_t hm = 0u;
                long long off = -1;
                if (e < total) {
                    const int bit = (int)__fns(mk, 0u, e - (inck - cntk) + 1);
                    const int S = s0 + (w0 + kw) * 32 + bit;
#pragma unroll
                    for (int h = 0; h < G; ++h) hm |= ((sm.zw[h * zwords + w0 + kw] >> bit) & 1u) << h;
                    span_look(S, len, off);
                }
                if (!visit(len, hm, off, min(32, total - e0))) return;
            }
        }
    };
    if (!a.deal) {
        walk([&](int len, uint32_t hm, long long off, int n) {
            for (int j = 0; j < n && good; ++j) {
                const int jl = __shfl_sync(FULL, len, j);
                const uint32_t jhm = __shfl_sync(FULL, hm, j);
                const long long jo = __shfl_sync(FULL, off, j);
                if (jl >= 1 && jo >= 0) emit_span(jl, jhm, jo, 0, jl);
            }
            return true;
        });
    } else {
        // the unit's zoomed token units (the per-word table), this split's share of
        // them, and the words that hold it
        unsigned tot = 0;
        for (int w = lane; w < nwords; w += 32) tot += (unsigned)sm.zu[w];
        const long long U = (long long)warp_sum_u(tot);
        const long long lo = U * split / a.nsplit, hi = U * (split + 1) / a.nsplit;
        long long base = 0;               // units of the words before the batch
        for (int w0 = 0; w0 < nwords && good && base < hi; w0 += 32) {
            const int w = w0 + lane;
            const int u = w < nwords ? sm.zu[w] : 0;
            int inc = u;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(FULL, inc, o);
                if (lane >= o) inc += t;
            }
            const long long cw = base + inc - u;          // units before word w
            uint32_t hits = __ballot_sync(FULL, u > 0 && cw < hi && cw + u > lo);
            while (hits && good) {
                const int k = __ffs(hits) - 1;
                hits &= hits - 1u;
                const int wk = w0 + k;
                const long long cu = base + __shfl_sync(FULL, inc - u, k);
                uint32_t m = 0u;
#pragma unroll
                for (int h = 0; h < G; ++h) m |= sm.zw[h * zwords + wk];
                // lane j resolves the word's j-th zoomed span
                const int cnt = __popc(m);
                int len = 0;
                uint32_t hm = 0u;
                long long off = -1;
                if (lane < cnt) {
                    const int bit = (int)__fns(m, 0u, lane + 1);
                    const int S = s0 + wk * 32 + bit;
#pragma unroll
                    for (int h = 0; h < G; ++h) hm |= ((sm.zw[h * zwords + wk] >> bit) & 1u) << h;
                    span_look(S, len, off);
                }
                const int nu = len >= 1 ? (len + 31) >> 5 : 0;
                int ex = nu;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(FULL, ex, o);
                    if (lane >= o) ex += t;
                }
                ex -= nu;
                for (int j = 0; j < cnt && good; ++j) {
                    const long long jc = cu + __shfl_sync(FULL, ex, j);
                    if (jc >= hi) break;
                    const int jl = __shfl_sync(FULL, len, j);
                    const int jn = __shfl_sync(FULL, nu, j);
                    const uint32_t jhm = __shfl_sync(FULL, hm, j);
                    const long long jo = __shfl_sync(FULL, off, j);
                    const long long u0 = lo > jc ? lo - jc : 0, u1 = hi - jc < jn ? hi - jc : jn;
                    if (jl >= 1 && jo >= 0 && u0 < u1)
                        emit_span(jl, jhm, jo, (int)(32 * u0), (int)min((long long)jl, 32 * u1));
                }
            }
            base += __shfl_sync(FULL, inc, 31);
        }
    }
    if (good) {
        ZPiece pc;
        pc.kind = ZP_END; pc.first = 0; pc.r0 = 0; pc.cnt = 0; pc.len = 0; pc.rS = 0; pc.hm = 0u; pc.rot = 0;
        emit1(pc, nullptr, 0u);
    }
    // every copy this warp started has landed before the CTA moves on (the full
    // barrier of a slot is re-armed only by this warp, so its last phase is stable)
    if (lane == 0) {
        const uint32_t lo = np > (uint32_t)ZNS ? np - ZNS : 0u;
        for (uint32_t i = lo; i < np; ++i)
            if (!mbar_wait_n(&sm.zfull[i % ZNS], (i / ZNS) & 1, a.polls)) set_status(a.status, SEKV_ERR_TIMEOUT);
    }
}

// The table the zoom producer deals from (deal mode; producer warp): zu[w] = the
// zoomed 32-token units of the spans of mask word w (spans zoomed by any head of
// the group). The zoomed spans are gathered 32 at a time across words, so the span
// lengths cost one round of loads per 32 zoomed spans.
template <int G>
SEKV_DEV void deal_table(const DecArgs& a, const DecSmem& sm, int lane, int b, int mb, int zwords) {
    constexpr uint32_t FULL = 0xffffffffu;
    const int nwords = (mb + 31) >> 5;
    int pend = -1;           // this lane's gathered span
    int p = 0;               // lanes [0, p) hold gathered spans
    auto flush = [&]() {
        if (lane < p) {
            const int len = a.span_end[(int64_t)b * a.m_cap + pend] - a.span_beg[(int64_t)b * a.m_cap + pend];
            if (len >= 1) atomicAdd(&sm.zu[pend >> 5], (len + 31) >> 5);
        }
        p = 0;
    };
    for (int w0 = 0; w0 < nwords; w0 += 32) {
        const int wi = w0 + lane;
        uint32_t m = 0u;
        if (wi < nwords) {
#pragma unroll
            for (int h = 0; h < G; ++h) m |= sm.zw[h * zwords + wi];
        }
        const int cnt = __popc(m);
        int inc = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(FULL, inc, o);
            if (lane >= o) inc += t;
        }
        const int total = __shfl_sync(FULL, inc, 31);
        for (int done = 0; done < total;) {
            const int take = min(32 - p, total - done);
            // lane p + i takes the batch's entry done + i
            const int e = done + lane - p;
            int k = 0;
            for (int j = 0; j < 32; ++j) k += (__shfl_sync(FULL, inc, j) <= e) ? 1 : 0;
            const int kw = k < 32 ? k : 31;
            const int inck = __shfl_sync(FULL, inc, kw), cntk = __shfl_sync(FULL, cnt, kw);
            const uint32_t mk = __shfl_sync(FULL, m, kw);
            if (lane >= p && lane < p + take)
                pend = (w0 + kw) * 32 + (int)__fns(mk, 0u, e - (inck - cntk) + 1);
            p += take;
            done += take;
            if (p == 32) flush();
        }
    }
    flush();
    __syncwarp();
}

// RM: the largest basis rank this instantiation handles (16, 32 or 64), which
// sizes the u / y fragments and the unrolled basis-row loops. Lane (g, c) holds
// heads 2c, 2c+1 (the stream layout): mh, lh (partial) and the O^T columns.
template <int D, int G, int RM, bool SP>
SEKV_DEV void zoom_consume(const DecArgs& a, const DecSmem& sm, int warp, int lane, const uint32_t (&qb)[D / 16][2],
                           float (&mh)[2], float (&lh)[2], float (&oc)[D / 16][4]) {
    using C = DecCfg<SEKV_BF16, D, G>;
    using Z = ZRing<C, SP>;
    constexpr int ZNS = Z::NS, ZSL = Z::SLOT;
    constexpr int NKS = RM / 16;         // groups of 16 basis rows (m-tiles of u, y; k-steps of s, O)
    constexpr int DB = D / 8;            // column blocks of 8 in B / D rows
    constexpr uint32_t FULL = 0xffffffffu;
    const int g = lane >> 2, c = lane & 3, lj = lane >> 3, lr = lane & 7;
    const float sl2 = a.scale * kLog2e;
    uint32_t ub[NKS][4];                 // u as B fragments per k-step: hi b0, hi b1, lo b0, lo b1 (then beta y)
    float yacc[NKS][4];                  // y accumulators per 16 basis rows: (row g / g+8, heads 2c, 2c+1)
    float msp[2] = {-INFINITY, -INFINITY}, lsp[2] = {0.f, 0.f};
    bool mine = false, zh0 = false, zh1 = false;
    int nib = 1, rS = 1;
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks) {
        ub[ks][0] = ub[ks][1] = ub[ks][2] = ub[ks][3] = 0u;
        yacc[ks][0] = yacc[ks][1] = yacc[ks][2] = yacc[ks][3] = 0.f;
    }

    // a span starts: its rank, the heads of this lane that zoom it, a fresh state
    auto span_begin = [&](const ZPiece& pc) {
        rS = pc.rS;
        nib = (rS + 7) >> 3;
        zh0 = 2 * c < G && ((pc.hm >> (2 * c)) & 1u);
        zh1 = 2 * c + 1 < G && ((pc.hm >> (2 * c + 1)) & 1u);
        msp[0] = msp[1] = -INFINITY;
        lsp[0] = lsp[1] = 0.f;
#pragma unroll
        for (int ks = 0; ks < NKS; ++ks) yacc[ks][0] = yacc[ks][1] = yacc[ks][2] = yacc[ks][3] = 0.f;
    };
    // u for the basis rows [r0, r0 + cnt) of the B rows at Bp (8x8 tiles; r0 a
    // multiple of 16), 16 rows at a time; two partial sums over even / odd k-steps
    // keep the mma chains short
    auto do_u = [&](const unsigned char* Bp, int r0, int cnt) {
#pragma unroll
        for (int ks = 0; ks < NKS; ++ks) {
            if (16 * ks < r0 || 16 * ks >= r0 + cnt) continue;
            const int ib = (16 * ks - r0) >> 3;                 // local 8-row block
            const bool two = 16 * ks + 8 < r0 + cnt;
            float ua[4] = {0.f, 0.f, 0.f, 0.f}, uv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                uint32_t ba[4];
                ldsm_x4(ba, Bp + (((ib + (lj & 1)) * DB + 2 * kk + (lj >> 1)) * 64 + lr * 8) * 2);
                if (!two) ba[1] = ba[3] = 0u;
                const uint32_t qf[2] = {qb[kk][0], qb[kk][1]};
                mma_bf16_16816((kk & 1) ? uv : ua, ba, qf);
            }
            // rows i >= r_S do not exist: exact zeros (select, not multiply)
            const int i0 = 16 * ks + g;
            uint32_t h01, l01, h23, l23;
            split_bf16x2(i0 < rS ? (ua[0] + uv[0]) * sl2 : 0.f, i0 < rS ? (ua[1] + uv[1]) * sl2 : 0.f, h01, l01);
            split_bf16x2(i0 + 8 < rS ? (ua[2] + uv[2]) * sl2 : 0.f, i0 + 8 < rS ? (ua[3] + uv[3]) * sl2 : 0.f,
                         h23, l23);
            ub[ks][0] = movm_t(h01);
            ub[ks][1] = movm_t(h23);
            ub[ks][2] = movm_t(l01);
            ub[ks][3] = movm_t(l23);
        }
    };
    // the 32-token units v = v0, v0 + vstep, ... of cnt tokens whose A rows are at
    // As and C rows at Cs (8x8 tiles, r8 wide); groups at or past ceil(cnt / 8)
    // hold other bytes and are masked
    auto do_units = [&](const unsigned char* As, const unsigned char* Cs, int cnt, int v0, int vstep) {
        const int nv = (cnt + 31) >> 5;
        for (int v = v0; v < nv; v += vstep) {
            const int ngp = ((cnt + 7) >> 3) - 4 * v;           // token groups of the unit that exist
            // s = A u for the unit's 32 tokens (two m-tiles of 16)
            float sc[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                sc[mt][0] = sc[mt][1] = sc[mt][2] = sc[mt][3] = 0.f;
                if (ngp <= 2 * mt) continue;
#pragma unroll
                for (int ks = 0; ks < NKS; ++ks) {
                    if (2 * ks >= nib) continue;
                    uint32_t aa[4];
                    ldsm_x4(aa, As + (((4 * v + 2 * mt + (lj & 1)) * nib + 2 * ks + (lj >> 1)) * 64 + lr * 8) * 2);
                    if (2 * ks + 1 >= nib) aa[2] = aa[3] = 0u;
                    const uint32_t uh[2] = {ub[ks][0], ub[ks][1]}, ul[2] = {ub[ks][2], ub[ks][3]};
                    mma_bf16_16816(sc[mt], aa, uh);
                    mma_bf16_16816(sc[mt], aa, ul);
                }
            }
            // the span's online softmax for heads 2c, 2c+1 (log2 domain; u carries the scale)
            float x[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tk = 32 * v + 16 * mt + g + ((e >> 1) << 3);
                    const bool zz = (e & 1) ? zh1 : zh0;
                    x[mt][e] = (zz && tk < cnt) ? sc[mt][e] : -INFINITY;
                }
            float mx0 = fmaxf(fmaxf(x[0][0], x[0][2]), fmaxf(x[1][0], x[1][2]));
            float mx1 = fmaxf(fmaxf(x[0][1], x[0][3]), fmaxf(x[1][1], x[1][3]));
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, o));
                mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, o));
            }
            const float mn0 = fmaxf(msp[0], mx0), mn1 = fmaxf(msp[1], mx1);
            const float al0 = (mn0 == -INFINITY) ? 1.f : ex2(msp[0] - mn0);
            const float al1 = (mn1 == -INFINITY) ? 1.f : ex2(msp[1] - mn1);
            const float r0 = (mn0 == -INFINITY) ? 0.f : mn0, r1 = (mn1 == -INFINITY) ? 0.f : mn1;
            float pv[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) pv[mt][e] = ex2(x[mt][e] - ((e & 1) ? r1 : r0));
            lsp[0] = fmaf(lsp[0], al0, (pv[0][0] + pv[0][2]) + (pv[1][0] + pv[1][2]));
            lsp[1] = fmaf(lsp[1], al1, (pv[0][1] + pv[0][3]) + (pv[1][1] + pv[1][3]));
            msp[0] = mn0;
            msp[1] = mn1;
            if (__any_sync(FULL, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
                for (int ks = 0; ks < NKS; ++ks) {
                    yacc[ks][0] *= al0; yacc[ks][1] *= al1;
                    yacc[ks][2] *= al0; yacc[ks][3] *= al1;
                }
            }
            // y += C^T p: p (k = tokens, n = heads) as B fragments by transposing the
            // 8 x 8 (token, head) blocks of the score accumulators
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                if (ngp <= 2 * mt) continue;
                const bool g2 = ngp > 2 * mt + 1;                 // the m-tile's second token group exists
                const uint32_t pb[2] = {movm_t(pack_bf16(pv[mt][0], pv[mt][1])),
                                        movm_t(pack_bf16(pv[mt][2], pv[mt][3]))};
#pragma unroll
                for (int js = 0; js < NKS; ++js) {
                    if (2 * js >= nib) continue;
                    uint32_t ca[4];
                    ldsm_x4_t(ca, Cs + (((4 * v + 2 * mt + (lj >> 1)) * nib + 2 * js + (lj & 1)) * 64 + lr * 8) * 2);
                    if (!g2) ca[2] = ca[3] = 0u;
                    mma_bf16_16816(yacc[js], ca, pb);
                }
            }
        }
    };
    // merge the span's (max, partial sum) into the stream state of heads 2c, 2c+1;
    // keep (beta y) as B fragments in ub (u is dead by now)
    auto do_merge = [&]() {
        float be[2] = {0.f, 0.f};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const bool zz = hh ? zh1 : zh0;
            if (zz && msp[hh] != -INFINITY) {
                const float mnew = fmaxf(mh[hh], msp[hh]);
                const float alpha = (mh[hh] == -INFINITY) ? 0.f : ex2(mh[hh] - mnew);
                be[hh] = ex2(msp[hh] - mnew);
                lh[hh] = lh[hh] * alpha + lsp[hh] * be[hh];
                mh[hh] = mnew;
#pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    oc[mt][hh] *= alpha;
                    oc[mt][2 + hh] *= alpha;
                }
            }
        }
#pragma unroll
        for (int ks = 0; ks < NKS; ++ks) {
            const int i0 = 16 * ks + g;
            ub[ks][0] = movm_t(pack_bf16(i0 < rS ? yacc[ks][0] * be[0] : 0.f, i0 < rS ? yacc[ks][1] * be[1] : 0.f));
            ub[ks][1] = movm_t(pack_bf16(i0 + 8 < rS ? yacc[ks][2] * be[0] : 0.f,
                                         i0 + 8 < rS ? yacc[ks][3] * be[1] : 0.f));
        }
    };
    // O^T += D^T (beta y) over the basis rows [r0, r0 + cnt) of the D rows at Dp
    auto do_D = [&](const unsigned char* Dp, int r0, int cnt) {
#pragma unroll
        for (int ks = 0; ks < NKS; ++ks) {
            if (16 * ks < r0 || 16 * ks >= r0 + cnt) continue;
            const int ib = (16 * ks - r0) >> 3;
            const bool two = 16 * ks + 8 < r0 + cnt;
            const uint32_t yb[2] = {ub[ks][0], ub[ks][1]};
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt) {
                uint32_t da[4];
                ldsm_x4_t(da, Dp + (((ib + (lj >> 1)) * DB + 2 * mt + (lj & 1)) * 64 + lr * 8) * 2);
                if (!two) da[2] = da[3] = 0u;
                mma_bf16_16816(oc[mt], da, yb);
            }
        }
    };

    // does this warp take any unit of the span? (ranks above 16: the span's pair of
    // warps, units alternating within the pair; else all four warps in turn)
    constexpr bool PAIRS = RM > 16;
    constexpr int WSTEP = PAIRS ? 2 : 4;
    auto owns = [&](const ZPiece& pc) {
        if (PAIRS) return (warp >> 1) == (pc.rot >> 1) && ((pc.len + 31) >> 5) > ((warp - pc.rot) & 1);
        return ((pc.len + 31) >> 5) > ((warp - pc.rot) & 3);
    };
    for (uint32_t k = 0;; ++k) {
        const int slot = (int)(k % ZNS);
        if (!mbar_wait_n(&sm.zfull[slot], (k / ZNS) & 1, a.polls)) {
            set_status(a.status, SEKV_ERR_TIMEOUT);
            break;
        }
        ZPiece pc;
        {
            const uint4 w0 = lds_u128(&sm.zmeta[slot]), w1 = lds_u128(reinterpret_cast<const char*>(&sm.zmeta[slot]) + 16);
            pc.kind = (int)w0.x; pc.first = (int)w0.y; pc.r0 = (int)w0.z; pc.cnt = (int)w0.w;
            pc.len = (int)w1.x; pc.rS = (int)w1.y; pc.hm = w1.z; pc.rot = (int)w1.w;
        }
        if (pc.kind == ZP_END) break;
        const unsigned char* zs = sm.stages + (size_t)slot * ZSL;
        if (SP && pc.kind == ZP_SPAN) {
            // the whole block [A | C | B | D] is in the slot; one warp takes it all
            if (warp == pc.rot) {
                span_begin(pc);
                const int r8 = nib * 8;
                const int pa = round8(pc.len) * r8;              // elements of A (and of C)
                do_u(zs + 4 * pa, 0, r8);
                do_units(zs, zs + 2 * pa, pc.len, 0, 1);
                do_merge();
                do_D(zs + 4 * pa + 2 * r8 * D, 0, r8);
            }
        } else if (pc.kind == ZP_MIX) {
            const int r8 = round8(pc.rS);
            const int oa = (pc.first & kMixB) ? r8 * D * 2 : 0;
            const int res = ((pc.cnt + 31) & ~31) * r8 * 2;
            if (pc.first & kMixB) {
                span_begin(pc);
                mine = owns(pc);
                if (mine) do_u(zs, 0, r8);
            }
            if (mine && pc.cnt > 0) do_units(zs + oa, zs + oa + res, pc.cnt, (warp - pc.rot - (pc.r0 >> 5)) & (WSTEP - 1), WSTEP);
            if (mine && (pc.first & kMixD)) {
                do_merge();
                do_D(zs + oa + 2 * res, 0, r8);
            }
        } else if (pc.kind == ZP_B) {
            if (pc.first) {
                span_begin(pc);
                mine = owns(pc);
            }
            if (mine) do_u(zs, pc.r0, pc.cnt);
        } else {  // ZP_D
            if (mine) {
                if (pc.first) do_merge();
                do_D(zs, pc.r0, pc.cnt);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.zempty[slot]);
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

// The unit's last CTA merges the nsplit partial states of every head by
// log-sum-exp, in split order, with the arithmetic of merge_kernel below (so the
// two forms give the same bits): M = max_j m_j, L = sum_j l_j 2^(m_j - M),
// O = sum_j o_j 2^(m_j - M) / L, lse = (M + log2 L) ln 2. The partials of the
// other CTAs are read past L1 (they were written by other SMs). All of a thread's
// loads are issued before the factors are formed: the first PS splits' output
// quads as asynchronous copies into the free stage memory (RINGB bytes), up to KT
// more into registers, and the (m, l) pairs; only splits beyond those wait for the
// factors.
template <int D, int G, int RINGB>
SEKV_DEV void merge_unit(const DecArgs& a, const DecSmem& sm, int64_t lunit, int b, int l, int kvh, int tid) {
    constexpr int NT = (kNW + 1) * 32;
    constexpr int NQ = G * D / 4;                               // output quads of the unit
    constexpr int QPT = (NQ + NT - 1) / NT;                     // quads per thread
    constexpr int KT = 16 / QPT;                                // split quads per output quad in registers
    constexpr int KB = 16;                                      // loads per round past those
    const int ns = a.nsplit;
    const int lane = tid & 31, warp = tid >> 5;
    float* fac = reinterpret_cast<float*>(sm.stages);          // [G][ns] m_j, then 2^(m_j - M) (the ring is free)
    float* lsv = fac + G * ns;                                  // [G][ns] l_j
    float* Mh = lsv + G * ns;                                   // [G]
    float* Lh = Mh + G;                                         // [G]
    const int off = ((2 * G * ns + 2 * G) * 4 + 15) & ~15;
    const int PS = max(0, min(ns, (RINGB - off) / (NQ * 16))); // splits staged in shared memory
    unsigned char* stg = sm.stages + off;                       // [PS][NQ] quads
    const int PT = min(ns - PS, KT);                            // splits in registers
    float4 vt[QPT][KT];
#pragma unroll
    for (int qq = 0; qq < QPT; ++qq) {
        const int i = tid + qq * NT;
        if (i < NQ) {
            const float4* po = reinterpret_cast<const float4*>(a.part_o + (lunit * G + i / (D / 4)) * ns * D) + i % (D / 4);
            for (int j = 0; j < PS; ++j) cp_async16(stg + ((size_t)j * NQ + i) * 16, po + (int64_t)j * (D / 4));
#pragma unroll
            for (int k = 0; k < KT; ++k)
                vt[qq][k] = k < PT ? __ldcg(po + (int64_t)(PS + k) * (D / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    // every (head, split) pair's (m, l)
    const float2* ml = reinterpret_cast<const float2*>(a.part_ml) + lunit * G * ns;
    for (int i = tid; i < G * ns; i += NT) {
        const float2 v = __ldcg(ml + i);
        fac[i] = v.x;
        lsv[i] = v.y;
    }
    __syncthreads();
    // per head (one warp each): M, the factors, and L summed in split order
    for (int h = warp; h < G; h += kNW + 1) {
        float* fh = fac + h * ns;
        float M = -INFINITY;
        for (int j = lane; j < ns; j += 32) M = fmaxf(M, fh[j]);
        M = warp_max(M);
        for (int j = lane; j < ns; j += 32) fh[j] = (M == -INFINITY) ? 0.f : exp2f(fh[j] - M);
        __syncwarp();
        if (lane == 0) {
            float Ls = 0.f;
            if (M != -INFINITY) {
                const float* lh = lsv + h * ns;
#pragma unroll 8
                for (int j = 0; j < ns; ++j) Ls = fmaf(lh[j], fh[j], Ls);
            }
            Mh[h] = M;
            Lh[h] = Ls;
        }
    }
    __syncthreads();
    cp_async_wait_all();
    // four output dims per thread: O = sum_j o_j f_j / L, summed in split order
#pragma unroll
    for (int qq = 0; qq < QPT; ++qq) {
        const int i = tid + qq * NT;
        if (i >= NQ) continue;
        const int h = i / (D / 4), k4 = i % (D / 4);
        const float M = Mh[h], Ls = Lh[h];
        const float* fj = fac + h * ns;
        float4 os = make_float4(0.f, 0.f, 0.f, 0.f);
        if (M != -INFINITY) {
            for (int j = 0; j < PS; ++j) {
                const float4 v = *reinterpret_cast<const float4*>(stg + ((size_t)j * NQ + i) * 16);
                const float f = fj[j];
                os.x = fmaf(v.x, f, os.x);
                os.y = fmaf(v.y, f, os.y);
                os.z = fmaf(v.z, f, os.z);
                os.w = fmaf(v.w, f, os.w);
            }
#pragma unroll
            for (int k = 0; k < KT; ++k) {
                if (k < PT) {
                    const float f = fj[PS + k];
                    os.x = fmaf(vt[qq][k].x, f, os.x);
                    os.y = fmaf(vt[qq][k].y, f, os.y);
                    os.z = fmaf(vt[qq][k].z, f, os.z);
                    os.w = fmaf(vt[qq][k].w, f, os.w);
                }
            }
            const float4* po = reinterpret_cast<const float4*>(a.part_o + (lunit * G + h) * ns * D) + k4;
            for (int j0 = PS + PT; j0 < ns; j0 += KB) {
                float4 v[KB];
#pragma unroll
                for (int k = 0; k < KB; ++k)
                    v[k] = j0 + k < ns ? __ldcg(po + (int64_t)(j0 + k) * (D / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int k = 0; k < KB; ++k) {
                    if (j0 + k < ns) {
                        const float f = fj[j0 + k];
                        os.x = fmaf(v[k].x, f, os.x);
                        os.y = fmaf(v[k].y, f, os.y);
                        os.z = fmaf(v[k].z, f, os.z);
                        os.w = fmaf(v[k].w, f, os.w);
                    }
                }
            }
        }
        const int64_t out = ((int64_t)b * a.L + l) * a.Hq + kvh * G + h;
        float* o = a.O + out * D + 4 * k4;
        o[0] = Ls > 0.f ? os.x / Ls : 0.f;
        o[1] = Ls > 0.f ? os.y / Ls : 0.f;
        o[2] = Ls > 0.f ? os.z / Ls : 0.f;
        o[3] = Ls > 0.f ? os.w / Ls : 0.f;
        if (k4 == 0) a.lse[out] = Ls > 0.f ? (M + log2f(Ls)) * kLn2 : -INFINITY;
    }
}

// SP: the zoom phase may take small spans whole (rank <= 16 only; chosen by the host
// from the expected zoom count: with few zoomed spans the plain variant is faster)
template <int DT, int D, int G, int RM, bool SP>
__global__ void __launch_bounds__((kNW + 1) * 32, 3)
decode_kernel(const DecArgs a, const __grid_constant__ DecMaps maps) {
    using C = DecCfg<DT, D, G>;
    constexpr int DPL = C::DPL, R = C::R, TR = C::TR, NS = C::NS;
    // Programmatic dependent launch: the grid may be scheduled while the previous
    // kernel on the stream finishes; no input is read before that kernel has
    // completed and its writes are visible, except (static_ready: the caller
    // guarantees that nothing in flight writes them) the cache's counts and the
    // first anchor / summary tiles. Once every CTA of this grid has passed the wait,
    // the next kernel may be scheduled likewise.
    const bool pre = a.static_ready != 0;
    if (!pre) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    }
    extern __shared__ __align__(1024) unsigned char sm_raw[];
    unsigned char* base = sm_raw + ((1024 - (smem_u32(sm_raw) & 1023)) & 1023);
    const int zwords = a.zwords;
    const DecSmem sm = carve_smem<C, G, D>(base, a.qcap, zwords, a.deal);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // one CTA per (split, kv head, sequence x layer); the split index varies
    // slowest so that whole splits are dispatched in order (the zoom work of a
    // unit tends to cluster in some splits; the lighter CTAs then fill the tail)
    const int nu = a.Hkv * a.B * a.Lr;
    const int split = blockIdx.x / nu;
    const int ur = blockIdx.x % nu;
    const int kvh = ur % a.Hkv;
    const int bl = ur / a.Hkv;
    const int b = bl / a.Lr, li = bl % a.Lr, l = a.l0 + li;
    const int64_t unit = ((int64_t)b * a.L + l) * a.Hkv + kvh;            // global (b, l, kvh)
    const int64_t lunit = ((int64_t)b * a.Lr + li) * a.Hkv + kvh;         // within this launch
    const bool route_only = a.phase == SEKV_ROUTE;

    // The loads that need no count are issued together with the counts, so their
    // latencies overlap: the G query rows (held in registers until they are stored to
    // shared memory below), the consumer lanes' thresholds and, when the unit's whole
    // mask is dealt from, its mask words.
    constexpr int NT = (kNW + 1) * 32;
    constexpr int QV = G * C::ROWB / 16;                  // 16-byte pieces of the G query rows
    constexpr int QPT = (QV + NT - 1) / NT;
    const uint4* qg = reinterpret_cast<const uint4*>(a.q + (((int64_t)b * a.L + l) * a.Hq + (int64_t)kvh * G) * C::ROWB);
    uint4 qv[QPT];
    float thp[2] = {INFINITY, INFINITY};                  // heads 2c, 2c+1 of a consumer lane
    const bool zpre = C::MMA && a.zin && a.deal;          // words 0 .. zwords-1 of the unit's mask
    constexpr int ZPT = C::MMA ? (kDealMaskBytes / 4 + NT - 1) / NT : 1;
    uint32_t zv[ZPT];
    auto load_inputs = [&]() {
#pragma unroll
        for (int k = 0; k < QPT; ++k)
            if (tid + k * NT < QV) qv[k] = qg[tid + k * NT];
        if (C::MMA && warp < kNW) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                if (2 * (lane & 3) + hh < G) thp[hh] = a.theta[(int64_t)l * a.Hq + kvh * G + 2 * (lane & 3) + hh];
        }
        if (zpre) {
#pragma unroll
            for (int k = 0; k < ZPT; ++k) {
                const int i = tid + k * NT;
                zv[k] = i < G * zwords
                            ? a.zmask[(((int64_t)b * a.L + l) * a.Hq + kvh * G + i / zwords) * a.mw + i % zwords]
                            : 0u;
            }
        }
    };
    if (!pre) load_inputs();
    const int ab = min(__ldcg(a.a_count + b), a.a_cap);     // past L1: may be read before the wait
    const int mb = min(__ldcg(a.m_count + b), a.m_cap);
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

    // issue stream tile i into its ring stage (producer lane 0)
    // Ring positions: one per stage, except in a routing pass on the tensor-core path,
    // which loads key tiles only: then every stage holds two positions (key rows in
    // its K or V half, the span scalars in the first or second 512 bytes past the two
    // tiles), so twice as many tiles are in flight.
    static_assert(!C::MMA || 2 * C::TILE + 2 * C::META <= C::STAGE, "two key tiles per stage");
    const int NP = (C::MMA && route_only) ? 2 * NS : NS;
    auto pos_key = [&](int s) -> unsigned char* {
        return NP == NS ? sm.stages + (size_t)s * C::STAGE : sm.stages + (size_t)(s >> 1) * C::STAGE + (s & 1) * C::TILE;
    };
    auto pos_meta = [&](int s) -> unsigned char* {
        return NP == NS ? sm.stages + (size_t)s * C::STAGE + 2 * C::TILE
                        : sm.stages + (size_t)(s >> 1) * C::STAGE + 2 * C::TILE + (s & 1) * C::META;
    };
    auto issue_tile = [&](int i) {
        const uint64_t pol = l2_evict_first();     // rows of this unit are read once per call
        const int s = i % NP;
        unsigned char* st = pos_key(s);
        if (i < nta) {
            const int r0 = a0 + i * TR;
            if constexpr (C::MMA) {
                const int y = (int)(unit * a.a_cap + r0);
                mbar_arrive_expect_tx(&sm.full[s], 2 * C::NBOX * 8192);
#pragma unroll
                for (int h = 0; h < C::NBOX; ++h) {
                    tma_load_2d_ef(st + h * 8192, &maps.Ka, 64 * h, y, &sm.full[s], pol);
                    tma_load_2d_ef(st + C::TILE + h * 8192, &maps.Va, 64 * h, y, &sm.full[s], pol);
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
                    tma_load_2d_ef(st + h * 8192, &maps.kbar, 64 * h, y, &sm.full[s], pol);
                    if (!route_only) tma_load_2d_ef(st + C::TILE + h * 8192, &maps.vbar, 64 * h, y, &sm.full[s], pol);
                }
            } else {
                const uint32_t bytes = (uint32_t)rows * C::ROWB;
                mbar_arrive_expect_tx(&sm.full[s], (route_only ? bytes : 2 * bytes) + 2 * mbytes);
                const int64_t off = (unit * a.m_cap + S0) * C::ROWB;
                bulk_g2s(st, a.kbar + off, bytes, &sm.full[s]);
                if (!route_only) bulk_g2s(st + C::TILE, a.vbar + off, bytes, &sm.full[s]);
            }
            bulk_g2s_ef(pos_meta(s), a.inv_norm + unit * a.m_cap + S0, mbytes, &sm.full[s], pol);
            bulk_g2s(pos_meta(s) + TR * 4, a.logS + (int64_t)b * a.m_cap + S0, mbytes, &sm.full[s]);
        }
    };

    // The producer initialises the barriers and issues the first ring stages before
    // the CTA-wide barrier, so their latency overlaps the query and mask loads.
    const int early = min(NP, ntiles);
    if (tid == kNW * 32) {
        for (int s = 0; s < NP; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], kNW);
        }
        if constexpr (C::MMA) {
            for (int s = 0; s < kMaxZSlots; ++s) {
                mbar_init(&sm.zfull[s], 1);
                mbar_init(&sm.zempty[s], kNW);
            }
        } else {
            for (int s = 0; s < kNW * C::ZNS; ++s) mbar_init(&sm.zbar[s], 1);
        }
        *sm.zq_next = 0;
        *sm.sfail = 0;
        fence_barrier_init();
        if (!a.starve)
            for (int i = 0; i < early; ++i) issue_tile(i);
    }
    if (pre) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        load_inputs();
    }
    // zoom-mask words: routed in this kernel (zero here, bits or-ed in by the stream),
    // or (tensor-core path, zin) the caller's mask: the split's words, or with deal the
    // unit's, bits of spans outside them cleared
    const int zbase = a.deal ? 0 : s0;          // span of bit 0 of word 0
    const int zend = a.deal ? mb : s1;          // spans >= zend are not in the words
    if (zpre) {
#pragma unroll
        for (int k = 0; k < ZPT; ++k) {
            const int i = tid + k * NT;
            if (i < G * zwords) {
                const int S = 32 * (i % zwords);
                uint32_t v = S < zend ? zv[k] : 0u;
                if (S < zend && zend - S < 32) v &= (1u << (zend - S)) - 1u;
                sm.zw[i] = v;
            }
        }
    } else {
        for (int i = tid; i < G * zwords; i += blockDim.x) {
            uint32_t v = 0u;
            if (C::MMA && a.zin) {
                const int h = i / zwords, w = i % zwords;
                const int S = zbase + 32 * w;
                if (S < zend) {
                    v = a.zmask[(((int64_t)b * a.L + l) * a.Hq + kvh * G + h) * a.mw + (S >> 5)];
                    if (zend - S < 32) v &= (1u << (zend - S)) - 1u;
                }
            }
            sm.zw[i] = v;
        }
    }
#pragma unroll
    for (int k = 0; k < QPT; ++k)
        if (tid + k * NT < QV) reinterpret_cast<uint4*>(sm.qs)[tid + k * NT] = qv[k];
    if (C::MMA && a.deal)
        for (int w = tid; w < zwords; w += blockDim.x) sm.zu[w] = 0;
    __syncthreads();

    const float sl2 = a.scale * kLog2e;
    bool ok = true;

    // stream state of a consumer warp
    //   tensor-core path: lane (g = lane/4, c = lane%4) holds heads 2c, 2c+1: their
    //   running max mh, partial sums lh (over the lane's own rows) and the O^T
    //   accumulator fragments oc[t] = O[2c + (e & 1)][16t + g + 8 (e >> 1)]
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
    uint32_t qb[C::MMA ? D / 16 : 1][2];      // tensor-core path: q as B fragments (stream and zoom)
    float oc[C::MMA ? D / 16 : 1][4];
    float mh[2] = {-INFINITY, -INFINITY}, lh[2] = {0.f, 0.f};
#pragma unroll
    for (int n = 0; n < (C::MMA ? D / 16 : 1); ++n) oc[n][0] = oc[n][1] = oc[n][2] = oc[n][3] = 0.f;

    if (warp == kNW) {
        // ------------------------------------------------------------ producer
        // with the first stages in flight, the warp builds the table the zoom
        // producer deals from (its loads overlap the consumers' first tiles)
        if (C::MMA && a.deal) deal_table<G>(a, sm, lane, b, mb, zwords);
        int issued = 0;
        if (lane == 0) {
            issued = a.starve ? 0 : early;
            for (int i = early; i < ntiles && !a.starve; ++i) {
                const int s = i % NP;
                if (!mbar_wait_n(&sm.empty[s], ((i / NP) - 1) & 1, a.polls)) {
                    set_status(a.status, SEKV_ERR_TIMEOUT);
                    *sm.sfail = 1;
                    break;
                }
                issue_tile(i);
                issued = i + 1;
            }
        }
        if (lane == 0) {
            // drain: every issued copy has landed before the ring is reused
            for (int i = max(0, issued - NP); i < issued; ++i)
                if (!mbar_wait_n(&sm.full[i % NP], (i / NP) & 1, a.polls)) {
                    set_status(a.status, SEKV_ERR_TIMEOUT);
                    *sm.sfail = 1;
                }
        }
    } else if constexpr (C::MMA) {
        // ------------------------------------------------ consumers, tensor cores
        // Each warp owns 16 rows of every 64-row tile. S = K q^T (M = the 16 rows,
        // N = 8 query heads, K = d); online softmax per head over the rows;
        // O^T += V^T P^T (M = 16 dims, N = heads, K = the 16 rows), P^T reaching the
        // B-fragment layout through 8 x 8 register transposes. Heads >= G are zero
        // columns. The q.kbar accumulator of a span row is both its routing logit
        // and its coarse attention logit.
        constexpr uint32_t FULL = 0xffffffffu;
        const int g = lane >> 2, c = lane & 3, lj = lane >> 3, lr = lane & 7;
        const float th0 = thp[0], th1 = thp[1];
        {
            const uint32_t* qp = reinterpret_cast<const uint32_t*>(sm.qs + (g < G ? g : 0) * C::ROWB);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                qb[kk][0] = g < G ? lds_u32(qp + 8 * kk + c) : 0u;
                qb[kk][1] = g < G ? lds_u32(qp + 8 * kk + 4 + c) : 0u;
            }
        }
        const int rbase = warp * R;                       // 16 rows of each tile
        const int krow = rbase + lr + ((lj & 1) << 3);    // this lane's ldmatrix row for K
        const int vrow = rbase + lr + ((lj >> 1) << 3);   // ... and for V
        for (int i = 0; i < ntiles && ok; ++i) {
            const int s = i % NP;
            if (!mbar_wait_n(&sm.full[s], (i / NP) & 1, a.polls)) {
                set_status(a.status, SEKV_ERR_TIMEOUT);
                ok = false;
                break;
            }
            const unsigned char* st = pos_key(s);
            const bool anchor_tile = i < nta;
            const int S0 = s0 + (i - nta) * TR;
            const int trows = anchor_tile ? min(TR, a1 - (a0 + i * TR)) : min(TR, s1 - S0);
            if (rbase < trows) {
                // ---- S for the warp's 16 rows; two partial sums over even / odd k-steps
                float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int chunk = 2 * (kk & 3) + (lj >> 1);
                    uint32_t ka[4];
                    ldsm_x4(ka, st + (kk >> 2) * 8192 + krow * 128 + ((chunk ^ (krow & 7)) << 4));
                    const uint32_t qf[2] = {qb[kk][0], qb[kk][1]};
                    mma_bf16_16816((kk & 1) ? sb : sa, ka, qf);
                }
                // sc[e]: row rbase + g + 8 (e >> 1), head 2c + (e & 1)
                float lg[4];
                if (anchor_tile) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int tk = rbase + g + ((e >> 1) << 3);
                        lg[e] = (2 * c + (e & 1) < G && tk < trows) ? (sa[e] + sb[e]) * sl2 : -INFINITY;
                    }
                } else {
                    const float* invn = reinterpret_cast<const float*>(pos_meta(s));
                    const float* lsv = invn + TR;
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        const int tk = rbase + g + 8 * rr;
                        const bool rv = tk < trows;
                        const float inv = rv ? lds_f32(invn + tk) : 0.f;
                        const float ls = rv ? lds_f32(lsv + tk) : 0.f;
                        const int SL = S0 + tk;
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int e = 2 * rr + hh, h = 2 * c + hh;
                            const bool valid = rv && h < G;
                            const float x = sa[e] + sb[e];
                            const float ell = fmaf(x * inv, a.scale, ls);          // Eq. (5) pre-sigmoid
                            const int zwi = h * zwords + ((SL - zbase) >> 5);
                            const bool z = valid && (a.zin ? ((sm.zw[zwi] >> (SL & 31)) & 1u) != 0u
                                                           : (ell > (hh ? th1 : th0)));   // Eq. (9)
                            if (valid && a.route_logits)
                                a.route_logits[(((int64_t)b * a.L + l) * a.Hq + kvh * G + h) * a.m_cap + SL] = ell;
                            if (z && !a.zin) atomicOr(&sm.zw[zwi], 1u << (SL & 31));
                            lg[e] = (valid && !z) ? fmaf(x, a.scale, ls) * kLog2e : -INFINITY;
                        }
                    }
                }
                if (!route_only) {
                    // ---- online softmax of heads 2c, 2c+1 over the warp's 16 rows
                    float mx0 = fmaxf(lg[0], lg[2]), mx1 = fmaxf(lg[1], lg[3]);
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) {
                        mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, o));
                        mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, o));
                    }
                    const float mn0 = fmaxf(mh[0], mx0), mn1 = fmaxf(mh[1], mx1);
                    const float al0 = (mn0 == -INFINITY) ? 1.f : ex2(mh[0] - mn0);
                    const float al1 = (mn1 == -INFINITY) ? 1.f : ex2(mh[1] - mn1);
                    const float r0 = (mn0 == -INFINITY) ? 0.f : mn0, r1 = (mn1 == -INFINITY) ? 0.f : mn1;
                    const float p0 = ex2(lg[0] - r0), p1 = ex2(lg[1] - r1), p2 = ex2(lg[2] - r0), p3 = ex2(lg[3] - r1);
                    lh[0] = fmaf(lh[0], al0, p0 + p2);
                    lh[1] = fmaf(lh[1], al1, p1 + p3);
                    mh[0] = mn0;
                    mh[1] = mn1;
                    if (__any_sync(FULL, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
                        for (int t = 0; t < D / 16; ++t) {
                            oc[t][0] *= al0; oc[t][1] *= al1;
                            oc[t][2] *= al0; oc[t][3] *= al1;
                        }
                    }
                    // ---- O^T += V^T P^T, 16 dims at a time
                    const uint32_t pb[2] = {movm_t(pack_bf16(p0, p1)), movm_t(pack_bf16(p2, p3))};
                    const unsigned char* vt = st + C::TILE;
#pragma unroll
                    for (int t = 0; t < D / 16; ++t) {
                        const int chunk = 2 * (t & 3) + (lj & 1);
                        uint32_t va[4];
                        ldsm_x4_t(va, vt + (t >> 2) * 8192 + vrow * 128 + ((chunk ^ (vrow & 7)) << 4));
                        mma_bf16_16816(oc[t], va, pb);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[s]);
        }
        if (lane == 0 && !ok) *sm.sfail = 1;
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
            if (!mbar_wait_n(&sm.full[s], (i / NS) & 1, a.polls)) {
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
                const bool z = validL && (a.zin ? zmask_bit(a, b, l, kvh * G + hL, SL) : (ell > th));   // Eq. (9)
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

    if constexpr (C::MMA) {
        // any zoomed span in this CTA's range (the same answer in every warp)
        const int nwords = a.deal ? zwords : (s1 > s0 ? (s1 - s0 + 31) >> 5 : 0);
        bool zany = false;
        for (int i = lane; i < G * zwords; i += 32) zany = zany || sm.zw[i] != 0u;
        zany = __any_sync(0xffffffffu, zany);
        if (!route_only && zany && *sm.sfail == 0) {     // uniform over the CTA
            if (warp == kNW) zoom_produce<D, G, SP>(a, sm, lane, b, l, kvh, zbase, nwords, zwords, split);
            else zoom_consume<D, G, RM, SP>(a, sm, warp, lane, qb, mh, lh, oc);
        }
    } else {
        if (!route_only && warp < kNW && ok) zoom_phase<DT, D, G>(a, sm, warp, lane, b, l, kvh, m_run, l_run, o, m_lane);
    }
    __syncthreads();    // zoom slots are dead: the ring takes the partial states
    if (!route_only && warp < kNW) {
        if constexpr (C::MMA) {
            // the partial sums of each head column over its 8 lanes
            float l0 = lh[0], l1 = lh[1];
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                l0 += __shfl_xor_sync(0xffffffffu, l0, o);
                l1 += __shfl_xor_sync(0xffffffffu, l1, o);
            }
            const int g = lane >> 2, c = lane & 3;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int h = 2 * c + hh;
                if (h < G) {
                    if (g == 0) {
                        sm.st_m[warp * G + h] = mh[hh];
                        sm.st_l[warp * G + h] = hh ? l1 : l0;
                    }
#pragma unroll
                    for (int t = 0; t < D / 16; ++t) {
                        sm.st_o[(warp * G + h) * D + 16 * t + g] = oc[t][hh];
                        sm.st_o[(warp * G + h) * D + 16 * t + g + 8] = oc[t][2 + hh];
                    }
                }
            }
        } else {
            store_state_lanes<D, G>(sm, warp, lane, m_run, l_run, o);
        }
    }
    __syncthreads();

    // ------------------------------------------------ zoom-mask words of this CTA
    if (a.zmask && !a.zin) {
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
    if (!a.arrive) return;      // a second kernel merges the splits

    // ------------------------------------------------ the unit's last CTA merges its splits
    // One thread counts the CTA in with an acquire-release add at GPU scope after the
    // CTA barrier, so the whole CTA's partial is visible before the count and the
    // other CTAs' partials are visible to the last one after it; the last one resets
    // the counter for the next call.
    __syncthreads();
    if (tid == 0) {
        uint32_t old;
        asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(old) : "l"(a.arrive + unit) : "memory");
        const int last = old + 1u == (uint32_t)a.nsplit;
        if (last) atomicExch(&a.arrive[unit], 0u);
        *sm.last = last;
    }
    __syncthreads();
    if (!*sm.last) return;
    merge_unit<D, G, C::RING>(a, sm, lunit, b, l, kvh, tid);
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
// Zoom budget cap (SeKV blog 2.3, the paragraph under Eq. (9)): when more spans
// pass the threshold than the budget allows, keep them in descending alpha~ order
// (monotone in the routing logit); equal logits keep the lower span index. One CTA
// per (b, l, query head): an exact radix select (8 bits at a time, most
// significant first) finds the budget-th largest logit among the zoomed spans,
// then the mask keeps every larger one and the lowest-index ties up to the budget.
// ---------------------------------------------------------------------------
SEKV_DEV uint32_t order_key(float f) {       // larger float <=> larger key
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr unsigned kCapDirect = 512;   // zoomed spans ranked directly (O(n^2) per CTA)

__global__ void __launch_bounds__(256) cap_kernel(const float* logits, uint32_t* zmask, const int32_t* m_count,
                                                  int L, int l0, int Lr, int Hq, int m_cap, int budget) {
    const int idx = blockIdx.x;
    const int h = idx % Hq, li = (idx / Hq) % Lr, b = idx / (Hq * Lr);
    const int l = l0 + li;
    const int mw = m_cap / 32;
    const int m = min(m_count[b], m_cap);
    const int nw = (m + 31) >> 5;
    uint32_t* zw = zmask + (((int64_t)b * L + l) * Hq + h) * mw;
    const float* lg = logits + (((int64_t)b * L + l) * Hq + h) * m_cap;
    __shared__ unsigned hist[256];
    __shared__ unsigned red[8];
    __shared__ uint32_t s_prefix;
    __shared__ unsigned s_k;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // zoomed count
    unsigned c = 0;
    for (int w = tid; w < nw; w += blockDim.x) c += __popc(zw[w]);
    c = warp_sum_u(c);
    if (lane == 0) red[warp] = c;
    __syncthreads();
    unsigned total = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) total += red[i];
    if (total <= (unsigned)budget) return;          // uniform over the CTA
    if (total <= kCapDirect) {
        // few zoomed spans: gather them, rank each by (logit descending, index
        // ascending) against all the others, keep ranks below the budget
        __shared__ uint32_t ck[kCapDirect];
        __shared__ int cs[kCapDirect];
        __shared__ unsigned cn;
        if (tid == 0) cn = 0u;
        __syncthreads();
        for (int w = tid; w < nw; w += blockDim.x) {
            uint32_t zb = zw[w];
            while (zb) {
                const int j = __ffs(zb) - 1;
                zb &= zb - 1u;
                const unsigned pos = atomicAdd(&cn, 1u);
                ck[pos] = order_key(lg[32 * w + j]);
                cs[pos] = 32 * w + j;
            }
        }
        __syncthreads();
        const unsigned n = cn;
        for (int w = tid; w < nw; w += blockDim.x) zw[w] = 0u;
        __syncthreads();
        for (unsigned i = tid; i < n; i += blockDim.x) {
            const uint32_t ki = ck[i];
            const int si = cs[i];
            unsigned rank = 0;
            for (unsigned j = 0; j < n; ++j) rank += (ck[j] > ki) || (ck[j] == ki && cs[j] < si);
            if (rank < (unsigned)budget) atomicOr(&zw[si >> 5], 1u << (si & 31));
        }
        return;
    }
    // radix select of the budget-th largest key among the zoomed spans
    uint32_t prefix = 0u;
    unsigned k = (unsigned)budget;                   // rank (1-based) within the current prefix class
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0u;
        __syncthreads();
        for (int S = tid; S < m; S += blockDim.x) {
            if (!((zw[S >> 5] >> (S & 31)) & 1u)) continue;
            const uint32_t key = order_key(lg[S]);
            if (shift < 24 && (key >> (shift + 8)) != (prefix >> (shift + 8))) continue;
            atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        // (the zoomed keys of a head often share their top bytes: the atomics above
        // then serialise, which is why small sets take the direct path)
        __syncthreads();
        if (tid == 0) {
            unsigned cum = 0;
            int dg = 255;
            for (; dg > 0; --dg) {
                if (cum + hist[dg] >= k) break;
                cum += hist[dg];
            }
            s_prefix = prefix | ((uint32_t)dg << shift);
            s_k = k - cum;
        }
        __syncthreads();
        prefix = s_prefix;
        k = s_k;
    }
    // prefix is the budget-th largest key; keep the k lowest-index spans holding it
    if (warp != 0) return;
    unsigned carry = 0;                              // ties kept so far (span order)
    for (int w0 = 0; w0 < nw; w0 += 32) {
        const int w = w0 + lane;
        uint32_t gt = 0u, eq = 0u;
        if (w < nw) {
            const uint32_t zb = zw[w];
            for (int j = 0; j < 32; ++j) {
                if (!((zb >> j) & 1u)) continue;
                const uint32_t key = order_key(lg[32 * w + j]);
                if (key > prefix) gt |= 1u << j;
                else if (key == prefix) eq |= 1u << j;
            }
        }
        const unsigned ne = __popc(eq);
        unsigned inc = ne;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned t = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += t;
        }
        const unsigned before = carry + inc - ne;     // ties in earlier words
        uint32_t keep_eq = 0u;
        if (before < k) {
            const unsigned take = min(ne, k - before);
            keep_eq = take >= 32 ? eq : (take == 0 ? 0u : (eq & ((2u << (__fns(eq, 0u, (int)take))) - 1u)));
        }
        if (w < nw) zw[w] = gt | keep_eq;
        carry += __shfl_sync(0xffffffffu, inc, 31);
    }
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
        const double slots = 3.0 * num_sms();     // resident CTAs (3 per SM on the bf16 / d=128 variant)
        int lim = (int)((d.a_cap + d.m_cap) / 128);
        lim = lim < 1 ? 1 : (lim > max_ns ? max_ns : lim);
        if (lim > 64) lim = 64;
        if (d.rows_hint > 0) {
            // Makespan model over ns: the grid is units * ns CTAs of rows / ns rows
            // each plus a fixed cost (setup, partial write, merge; ~64 rows' worth),
            // scheduled dynamically onto the resident slots, plus half a CTA of tail.
            // A routing pass reads only the span rows' keys (about a quarter of the
            // bytes of an anchor + span row pair), so it counts a quarter of the rows,
            // and its fixed cost per CTA weighs twice as much against them (fitted on
            // a B200 at 128K: 2, 3, 4, 6 splits took 42.7, 35.9, 38.9, 40.2 us).
            const double rows = d.phase == SEKV_ROUTE ? 0.25 * d.rows_hint : (double)d.rows_hint;
            const double o = d.phase == SEKV_ROUTE ? 128.0 : 64.0;
            int best = 1;
            double best_t = 1e300;
            for (int c = 1; c <= lim; ++c) {
                const double cta = rows / c + o;
                const double t = (double)units * c / slots * cta + 0.5 * cta;
                if (t < best_t * (1.0 - 1e-9)) { best_t = t; best = c; }
            }
            ns = best;
        } else {
            // Capacities only: fill whole waves of resident CTAs: the smallest split
            // count with >= 1.5 waves and >= 85% of the last wave busy; otherwise the
            // best such ratio. Splits keep >= ~128 rows of the capacities.
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
    }
    if (ns > max_ns) ns = max_ns;
    if (ns < 1) ns = 1;
    p.nsplit = ns;
    p.span_chunk = (int)round_up((d.m_cap + ns - 1) / ns, 32);
    p.anchor_chunk = (d.a_cap + ns - 1) / ns;
    const int G = d.Hq / d.Hkv;
    p.partial_bytes = (size_t)round_up((int64_t)units * G * ns * (d.d + 2) * 4, 256);
    // routing logits for the budget cap when the caller passes no buffer
    p.logit_bytes = (d.budget > 0 && d.phase != SEKV_ATTEND && !d.route_logits)
                        ? (size_t)round_up((int64_t)d.B * d.L * d.Hq * d.m_cap * 4, 256)
                        : 0;
    return p;
}

size_t decode_workspace_bytes(const sekv_decode_desc& d) {
    const DecodePlan p = plan_decode(d);
    return p.partial_bytes + p.logit_bytes;
}

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

template <int DT, int D, int G, int RM, bool SP>
static cudaError_t launch_t(const sekv_decode_desc& d, const DecodePlan& p, void* partials, cudaStream_t st,
                            int zin) {
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
    a.B = d.B; a.L = d.L; a.l0 = d.l0; a.Lr = Lr; a.Hq = d.Hq; a.Hkv = d.Hkv; a.a_cap = d.a_cap; a.m_cap = d.m_cap;
    a.rank = d.rank; a.phase = d.phase; a.nsplit = p.nsplit; a.sch_max = p.span_chunk;
    a.qcap = C::MMA ? 0 : ((p.span_chunk + C::TR - 1) / C::TR) * C::R;   // the tensor-core path reads the bitmask
    a.mw = d.m_cap / 32;
    a.zin = zin;
    // test hook (sekv_decode_desc.test_flags bit 0): no copies and short waits
    a.starve = (d.test_flags & 1) ? 1 : 0;
    a.static_ready = d.static_ready ? 1 : 0;
    a.polls = a.starve ? 4096u : kWaitPolls;
    a.arrive = d.phase != SEKV_ROUTE ? d.arrive : nullptr;
    a.O = d.O;
    a.lse = d.lse;
    // Dealing the unit's zoom work evenly over its splits shortens the longest CTA;
    // it pays when the grid is about one wave (e.g. a call for one layer), where the
    // call lasts as long as its longest CTA. With several waves the CTAs that hold no
    // zoom work fill in around the others, and keeping zoom work with its own split
    // measured faster. It needs the zoom decisions up front (zin) and the unit's
    // whole mask beside the ring in shared memory.
    const int64_t ctas = units * p.nsplit;
    a.deal = (C::MMA && zin && ctas <= 3 * (int64_t)num_sms() && (size_t)(G + 1) * a.mw * 4 <= kDealMaskBytes) ? 1 : 0;
    a.zwords = a.deal ? a.mw : a.sch_max / 32;
    const size_t smem = decode_smem_bytes<DT, D, G>(a.zwords, a.qcap, a.deal);
    if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<DT, D, G, RM, SP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
    const int64_t nblk = (int64_t)p.nsplit * d.Hkv * d.B * Lr;
    if (nblk > 0x7fffffff) return cudaErrorInvalidConfiguration;
    dim3 grid((unsigned)nblk);
    // launched with programmatic stream serialization: its launch overlaps the end of
    // the previous kernel on the stream (the kernel waits for that kernel's writes)
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = grid;
    cfg.blockDim = dim3((kNW + 1) * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, decode_kernel<DT, D, G, RM, SP>, a, maps)) != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (d.phase != SEKV_ROUTE && !a.arrive) {
        merge_kernel<D><<<d.B * Lr * d.Hq, D, 0, st>>>(a.part_o, a.part_ml, d.O, d.lse, p.nsplit, G, d.Hkv,
                                                        d.L, d.l0, Lr, d.Hq);
        e = cudaGetLastError();
    }
    return e;
}

// the tensor-core zoom is compiled for basis ranks up to 16, 32 and 64; the
// CUDA-core path handles any rank up to 64 in one variant
template <int DT, int D, int G>
static cudaError_t launch_r(const sekv_decode_desc& d, const DecodePlan& p, void* w, cudaStream_t st, int zin) {
    if (DT == SEKV_BF16 && d.rank <= 16)
        return d.zoom_hint >= (int)kSpanModeSpans ? launch_t<DT, D, G, 16, true>(d, p, w, st, zin)
                                                   : launch_t<DT, D, G, 16, false>(d, p, w, st, zin);
    if (DT == SEKV_BF16 && d.rank <= 32) return launch_t<DT, D, G, 32, false>(d, p, w, st, zin);
    return launch_t<DT, D, G, 64, false>(d, p, w, st, zin);
}

template <int DT, int D>
static cudaError_t launch_g(const sekv_decode_desc& d, const DecodePlan& p, void* w, cudaStream_t st, int zin) {
    switch (d.Hq / d.Hkv) {
        case 1: return launch_r<DT, D, 1>(d, p, w, st, zin);
        case 2: return launch_r<DT, D, 2>(d, p, w, st, zin);
        case 4: return launch_r<DT, D, 4>(d, p, w, st, zin);
        default: return launch_r<DT, D, 8>(d, p, w, st, zin);
    }
}

static cudaError_t launch_pass(const sekv_decode_desc& d, const DecodePlan& p, void* partials, cudaStream_t st,
                               int zin) {
    if (d.dtype == SEKV_F32)
        return d.d == 64 ? launch_g<SEKV_F32, 64>(d, p, partials, st, zin)
                         : launch_g<SEKV_F32, 128>(d, p, partials, st, zin);
    return d.d == 64 ? launch_g<SEKV_BF16, 64>(d, p, partials, st, zin)
                     : launch_g<SEKV_BF16, 128>(d, p, partials, st, zin);
}

// ---------------------------------------------------------------------------
// Split-K partials for callers that pass no workspace: one static device array,
// present on every device that loads this library until the process exits.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_decode_scratch[SEKV_STATIC_SCRATCH_BYTES];

size_t decode_static_scratch_bytes() { return SEKV_STATIC_SCRATCH_BYTES; }

// Device address of g_decode_scratch on the current device. In host code the
// array's name only stands in for it, so the address is looked up with the
// device current and cached per device, together with the context it belongs
// to: after a cudaDeviceReset the device gets a new primary context (and a new
// copy of the array), which the cache notices and looks the address up again.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

static CtxGetCurrentFn ctx_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
    }
    return fn;
}

void* decode_static_scratch(cudaError_t* err) {
    static std::mutex mu;
    static void* addr[256] = {nullptr};
    static CUcontext owner[256] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 256) {
        *err = e != cudaSuccess ? e : cudaErrorInvalidDevice;
        return nullptr;
    }
    CtxGetCurrentFn cur = ctx_current_fn();
    auto current = [&]() -> CUcontext {
        CUcontext c = nullptr;
        return (cur && cur(&c) == CUDA_SUCCESS) ? c : nullptr;
    };
    std::lock_guard<std::mutex> lock(mu);
    const CUcontext ctx = current();
    if (!addr[dev] || !ctx || owner[dev] != ctx) {
        // the lookup binds the device's context if the thread has none yet
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
        if (e != cudaSuccess || !ptr) {
            *err = e != cudaSuccess ? e : cudaErrorInvalidSymbol;
            return nullptr;
        }
        addr[dev] = ptr;
        owner[dev] = current();
    }
    *err = cudaSuccess;
    return addr[dev];
}

// Without a budget: one pass (FUSED / ROUTE / ATTEND; ATTEND reads the caller's
// mask when one is given, and routes again otherwise). With a budget: ROUTE and
// FUSED run the routing pass (threshold mask + routing logits), then the cap;
// FUSED then attends with the capped mask as input. ATTEND takes the caller's
// (capped) mask as input.
cudaError_t launch_decode(const sekv_decode_desc& d, const DecodePlan& p, void* partials, cudaStream_t st) {
    const bool learned = d.route_W != nullptr;
    if (!learned && d.budget <= 0) return launch_pass(d, p, partials, st, d.phase == SEKV_ATTEND && d.zmask ? 1 : 0);
    // the attention pass takes the (capped / learned) mask as input; with learned
    // routing it must not overwrite the routing logits with identity-form ones
    sekv_decode_desc att = d;
    if (learned) att.route_logits = nullptr;
    if (d.phase == SEKV_ATTEND) return launch_pass(att, p, partials, st, 1);
    sekv_decode_desc r = d;
    r.phase = SEKV_ROUTE;
    if (d.budget > 0 && !r.route_logits)
        r.route_logits = reinterpret_cast<float*>(reinterpret_cast<char*>(partials) + p.partial_bytes);
    cudaError_t e = learned ? launch_route_learned(r, st) : launch_pass(r, p, partials, st, 0);
    if (e != cudaSuccess) return e;
    if (d.budget > 0) {
        const int Lr = d.l1 - d.l0;
        cap_kernel<<<d.B * Lr * d.Hq, 256, 0, st>>>(r.route_logits, d.zmask, d.m_count, d.L, d.l0, Lr, d.Hq,
                                                     d.m_cap, d.budget);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (d.phase == SEKV_ROUTE) return cudaSuccess;
    return launch_pass(att, p, partials, st, 1);
}

}  // namespace sekv
