// C ABI of the SeKV span-cache library: argument checks, workspace carving,
// launches, and the host side of the cold-basis fetch.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <string>
#include <vector>

#include "sekv_common.cuh"
#include "sekv_internal.h"

namespace {

thread_local std::string g_err;

sekv_status fail(sekv_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

sekv_status cuda_fail(cudaError_t e, const char* where) {
    return fail(SEKV_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int esize(int dtype) { return dtype == SEKV_F32 ? 4 : 2; }

#define SEKV_REQUIRE(cond, ...)                                   \
    do {                                                          \
        if (!(cond)) return fail(SEKV_ERR_INVALID_ARG, __VA_ARGS__); \
    } while (0)

sekv_status check_build(const sekv_build_desc* d) {
    SEKV_REQUIRE(d, "build: null descriptor");
    SEKV_REQUIRE(d->B >= 1 && d->L >= 1 && d->Hkv >= 1 && d->n >= 1, "build: B, L, Hkv, n must be >= 1");
    SEKV_REQUIRE(d->dtype == SEKV_F32 || d->dtype == SEKV_BF16, "build: dtype %d", d->dtype);
    SEKV_REQUIRE(d->steps >= 1 && d->steps <= SEKV_BUILD_ALL, "build: steps mask %d", d->steps);
    SEKV_REQUIRE(d->a_cap >= 1 && d->m_cap >= 32 && d->m_cap % 32 == 0,
                 "build: a_cap >= 1 and m_cap a positive multiple of 32 required");
    SEKV_REQUIRE(d->window >= 0, "build: window < 0");
    SEKV_REQUIRE(d->dev_status, "build: dev_status is required");
    if (d->steps & SEKV_BUILD_SCAN)
        SEKV_REQUIRE(d->H && d->a_count && d->m_count && d->anchor_pos && d->span_beg && d->span_end,
                     "build/scan: H, a_count, m_count, anchor_pos, span_beg, span_end required");
    if (d->steps & SEKV_BUILD_LAYOUT) {
        SEKV_REQUIRE(d->m_count && d->span_beg && d->span_end && d->logS && d->blk_off,
                     "build/layout: m_count, span_beg, span_end, logS, blk_off required");
        SEKV_REQUIRE(d->rank >= 1, "build/layout: rank >= 1 required");
    }
    if (d->steps & (SEKV_BUILD_SUMMARY | SEKV_BUILD_BASES)) {
        SEKV_REQUIRE(d->l0 >= 0 && d->l0 < d->l1 && d->l1 <= d->L, "build: layer range [%d, %d) of %d",
                     d->l0, d->l1, d->L);
        if (d->d != 64 && d->d != 128) return fail(SEKV_ERR_UNSUPPORTED, "build: d = %d (64 or 128)", d->d);
        SEKV_REQUIRE(d->K && d->V && aligned(d->K, 16) && aligned(d->V, 16),
                     "build: K and V must be non-null and 16-byte aligned");
    }
    if (d->steps & SEKV_BUILD_SUMMARY) {
        SEKV_REQUIRE(d->H && d->Ka && d->Va && d->kbar && d->vbar && d->inv_norm && d->anchor_pos &&
                         d->a_count && d->m_count && d->span_beg && d->span_end,
                     "build/summary: missing pointer");
        SEKV_REQUIRE(aligned(d->Ka, 16) && aligned(d->Va, 16) && aligned(d->kbar, 16) && aligned(d->vbar, 16),
                     "build/summary: Ka, Va, kbar, vbar must be 16-byte aligned");
        SEKV_REQUIRE(d->wmode >= SEKV_W_UNIFORM && d->wmode <= SEKV_W_SOFTMAX, "build: wmode %d", d->wmode);
        if (d->route_W) {
            SEKV_REQUIRE(d->kbar_r && aligned(d->route_W, 16) && aligned(d->kbar_r, 16),
                         "build/summary: route_W needs kbar_r; both 16-byte aligned");
            if (!sekv::route_summary_supported(*d))
                return fail(SEKV_ERR_UNSUPPORTED,
                            "build/summary: routing summaries for Hq=%d, Hkv=%d, dr=%d, d=%d, dtype=%d not "
                            "supported (Hq a multiple of Hkv, Hq/Hkv <= 8, dr 32 or 64, W within shared memory)",
                            d->Hq, d->Hkv, d->dr, d->d, d->dtype);
        }
    }
    if (d->steps & SEKV_BUILD_BASES) {
        SEKV_REQUIRE(d->basis_home && d->blk_off && d->m_count && d->span_beg && d->span_end,
                     "build/bases: basis_home, blk_off and the span arrays are required");
        SEKV_REQUIRE(d->rank >= 1 && d->max_sweeps >= 1, "build/bases: rank and max_sweeps >= 1");
        SEKV_REQUIRE(d->region_elems > 0 && d->region_elems % 64 == 0 && aligned(d->basis_home, 256),
                     "build/bases: region_elems a positive multiple of 64, basis_home 256-byte aligned");
        SEKV_REQUIRE(d->workspace && aligned(d->workspace, 256) &&
                         (size_t)d->workspace_bytes >= sekv::basis_workspace_bytes(*d),
                     "build/bases: workspace of %zu bytes (256-byte aligned) required",
                     sekv::basis_workspace_bytes(*d));
    }
    return SEKV_OK;
}

sekv_status check_decode(const sekv_decode_desc* d, bool with_workspace = true) {
    SEKV_REQUIRE(d, "decode: null descriptor");
    SEKV_REQUIRE(d->B >= 1 && d->L >= 1 && d->Hq >= 1 && d->Hkv >= 1 && d->Hq % d->Hkv == 0,
                 "decode: B, L, Hq, Hkv >= 1 and Hq a multiple of Hkv");
    SEKV_REQUIRE(d->l0 >= 0 && d->l0 < d->l1 && d->l1 <= d->L, "decode: layer range [%d, %d) of %d", d->l0,
                 d->l1, d->L);
    SEKV_REQUIRE(d->phase >= SEKV_FUSED && d->phase <= SEKV_ATTEND, "decode: phase %d", d->phase);
    SEKV_REQUIRE(d->a_cap >= 1 && d->m_cap >= 32 && d->m_cap % 32 == 0, "decode: a_cap >= 1, m_cap % 32 == 0");
    SEKV_REQUIRE(d->m_cap < (1 << 24), "decode: m_cap must be < 2^24");
    SEKV_REQUIRE(d->nsplit >= 0 && d->rows_hint >= 0 && d->budget >= 0 && d->zoom_hint >= 0,
                 "decode: nsplit, rows_hint, budget and zoom_hint must be >= 0");
    SEKV_REQUIRE(d->budget == 0 || d->zmask, "decode: a budget needs the zmask buffer (output of ROUTE / FUSED, "
                                             "input of ATTEND)");
    if (d->route_W) {
        SEKV_REQUIRE(d->kbar_r && d->zmask && aligned(d->kbar_r, 16),
                     "decode: learned routing (route_W) needs kbar_r (16-byte aligned) and the zmask buffer");
        if (!sekv::route_learned_supported(*d))
            return fail(SEKV_ERR_UNSUPPORTED, "decode: routing dimension dr = %d (32 or 64)", d->dr);
    }
    if (!sekv::decode_supported(*d))
        return fail(SEKV_ERR_UNSUPPORTED, "decode: d=%d, Hq/Hkv=%d, rank=%d, dtype=%d not compiled", d->d,
                    d->Hq / d->Hkv, d->rank, d->dtype);
    SEKV_REQUIRE(d->dev_status && d->q && d->a_count && d->m_count && d->span_beg && d->span_end && d->logS &&
                     d->kbar && d->inv_norm && d->theta,
                 "decode: missing input pointer");
    SEKV_REQUIRE(aligned(d->q, 16) && aligned(d->kbar, 16) && aligned(d->inv_norm, 16) && aligned(d->logS, 16),
                 "decode: q, kbar, inv_norm, logS must be 16-byte aligned");
    if (d->phase == SEKV_ROUTE) {
        SEKV_REQUIRE(d->zmask || d->route_logits, "decode/route: zmask or route_logits required");
        if (d->budget > 0 && !d->route_logits && with_workspace) {
            // the capped routing pass keeps its logits in the workspace
            const size_t need = sekv::decode_workspace_bytes(*d);
            SEKV_REQUIRE(d->workspace && aligned(d->workspace, 256) && (size_t)d->workspace_bytes >= need,
                         "decode/route: budget without route_logits needs a workspace of %zu bytes", need);
        }
    } else {
        SEKV_REQUIRE(d->Ka && d->Va && d->vbar && d->arena && d->O && d->lse,
                     "decode: Ka, Va, vbar, arena, O, lse required");
        SEKV_REQUIRE(aligned(d->Ka, 16) && aligned(d->Va, 16) && aligned(d->vbar, 16) && aligned(d->arena, 256),
                     "decode: Ka, Va, vbar 16-byte and arena 256-byte aligned");
        if (d->phase == SEKV_ATTEND) SEKV_REQUIRE(d->slot, "decode/attend: slot table required");
        if (!d->slot)
            SEKV_REQUIRE(d->blk_off && d->region_elems > 0 && d->region_elems % 64 == 0,
                         "decode: blk_off and region_elems (multiple of 64) required without a slot table");
        if (with_workspace) {
            const size_t need = sekv::decode_workspace_bytes(*d);
            SEKV_REQUIRE(d->workspace && aligned(d->workspace, 256) && (size_t)d->workspace_bytes >= need,
                         "decode: workspace of %zu bytes (256-byte aligned) required", need);
        }
    }
    return SEKV_OK;
}

}  // namespace

extern "C" {

const char* sekv_status_str(int32_t s) {
    switch (s) {
        case SEKV_OK: return "ok";
        case SEKV_ERR_INVALID_ARG: return "invalid argument";
        case SEKV_ERR_CAPACITY: return "capacity exceeded";
        case SEKV_ERR_CUDA: return "CUDA error";
        case SEKV_ERR_COLD_SPAN: return "zoomed span has no resident bases";
        case SEKV_ERR_TIMEOUT: return "bounded device wait ran out";
        case SEKV_ERR_UNSUPPORTED: return "unsupported shape";
        case SEKV_WARN_NOT_CONVERGED: return "basis eigenvector solve failed";
        default: return "unknown status";
    }
}

const char* sekv_last_error(void) { return g_err.c_str(); }

int32_t sekv_version(void) { return SEKV_VERSION; }

size_t sekv_desc_size(int32_t which) {
    switch (which) {
        case 0: return sizeof(sekv_build_desc);
        case 1: return sizeof(sekv_decode_desc);
        case 2: return sizeof(sekv_fetch_desc);
        default: return 0;
    }
}

int64_t sekv_block_elems(int32_t len, int32_t d, int32_t rank) {
    if (len < 1 || d < 1 || rank < 1) return 0;
    return sekv::block_elems(len, d, rank);
}

int64_t sekv_basis_region_bound(int32_t n, int32_t m_cap, int32_t Hkv, int32_t d, int32_t rank) {
    // per span: 2 len8 r8 + 2 r8 d with len8 <= |S| + 7 and r8 <= min(roundup(rank, 8), d)
    const int64_t r8 = std::min<int64_t>(sekv::round_up(rank, 8), d);
    const int64_t per = 2 * r8 * n + (int64_t)m_cap * (14 * r8 + 2 * r8 * d);
    return sekv::round_up((int64_t)Hkv * per, 64);
}

size_t sekv_build_workspace_bytes(const sekv_build_desc* d) {
    if (!d) return 0;
    return (d->steps & SEKV_BUILD_BASES) ? sekv::basis_workspace_bytes(*d) : 0;
}

sekv_status sekv_build_spans(const sekv_build_desc* d, sekv_stream_t stream) {
    sekv_status s = check_build(d);
    if (s != SEKV_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (d->steps & SEKV_BUILD_SCAN)
        if ((e = sekv::launch_scan(*d, st)) != cudaSuccess) return cuda_fail(e, "scan");
    if (d->steps & SEKV_BUILD_LAYOUT)
        if ((e = sekv::launch_layout(*d, (d->steps & SEKV_BUILD_BASES) != 0, st)) != cudaSuccess)
            return cuda_fail(e, "layout");
    if (d->steps & SEKV_BUILD_SUMMARY)
        if ((e = sekv::launch_summary(*d, st)) != cudaSuccess) return cuda_fail(e, "summary");
    if (d->steps & SEKV_BUILD_BASES)
        if ((e = sekv::launch_basis(*d, st)) != cudaSuccess) return cuda_fail(e, "bases");
    return SEKV_OK;
}

size_t sekv_decode_workspace_bytes(const sekv_decode_desc* d) {
    if (!d || d->Hkv < 1 || d->Hq < 1 || d->l1 <= d->l0) return 0;
    return sekv::decode_workspace_bytes(*d);
}

sekv_status sekv_decode_attn(const sekv_decode_desc* d, sekv_stream_t stream) {
    sekv_status s = check_decode(d);
    if (s != SEKV_OK) return s;
    const sekv::DecodePlan p = sekv::plan_decode(*d);
    cudaError_t e = sekv::launch_decode(*d, p, d->workspace, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "decode");
    return SEKV_OK;
}

sekv_status sekv_merge_partials(const float* O_parts, const float* lse_parts, int32_t nparts, int64_t rows,
                                int32_t d, float* O, float* lse, sekv_stream_t stream) {
    SEKV_REQUIRE(O_parts && lse_parts && O && lse, "merge: null pointer");
    SEKV_REQUIRE(nparts >= 1 && nparts <= 64 && rows >= 0 && rows < (1LL << 31) && d >= 1 && d <= 1024,
                 "merge: nparts in [1, 64], rows in [0, 2^31), d in [1, 1024]");
    cudaError_t e = sekv::launch_merge_parts(O_parts, lse_parts, nparts, rows, d, O, lse,
                                             reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "merge");
    return SEKV_OK;
}

sekv_status sekv_decode_attn_static(const sekv_decode_desc* d, sekv_stream_t stream) {
    sekv_status s = check_decode(d, false);
    if (s != SEKV_OK) return s;
    const sekv::DecodePlan p = sekv::plan_decode(*d);
    const size_t cap = sekv::decode_static_scratch_bytes();
    if (p.partial_bytes + p.logit_bytes > cap)
        return fail(SEKV_ERR_CAPACITY,
                    "decode_static: this call needs %zu bytes of split-K scratch, the static array holds %zu "
                    "(fewer layers per call, a smaller batch or nsplit, or sekv_decode_attn with a workspace)",
                    p.partial_bytes + p.logit_bytes, cap);
    cudaError_t e;
    void* scratch = sekv::decode_static_scratch(&e);
    if (!scratch) return cuda_fail(e, "decode_static: address of the static scratch");
    e = sekv::launch_decode(*d, p, scratch, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "decode_static");
    return SEKV_OK;
}

sekv_status sekv_tau_to_theta(const double* tau, float* theta, int64_t n) {
    SEKV_REQUIRE(n >= 0 && (n == 0 || (tau && theta)), "tau_to_theta: n >= 0 and non-null tau, theta required");
    for (int64_t i = 0; i < n; ++i)
        SEKV_REQUIRE(!std::isnan(tau[i]), "tau_to_theta: tau[%lld] is NaN", (long long)i);
    // sigma(l) > tau  <=>  l > ln(tau / (1 - tau)) for 0 < tau < 1 (SeKV blog 2.3, Eq. (9))
    for (int64_t i = 0; i < n; ++i) {
        const double t = tau[i];
        theta[i] = t <= 0.0 ? -INFINITY : (t >= 1.0 ? INFINITY : (float)std::log(t / (1.0 - t)));
    }
    return SEKV_OK;
}

}  // extern "C"

namespace sekv {

// Refill-mode gather (SeKV summary, workflow paragraph: the bases of the zoomed
// spans are fetched from the CPU). One CTA per (b, layer, kv head) and
// chunk: the spans zoomed by any query head of the kv head's group, in span order,
// are dealt over the unit's nch chunks; a CTA copies the kv head's block of each of
// its spans from the home (pinned host memory read through unified addressing) to
// the span's arena slot. Blocks are multiples of 128 bytes (64 elements) and start
// at multiples of 64 elements, so 16-byte vectors cover them exactly.
__global__ void __launch_bounds__(256) fetch_gather_kernel(const uint32_t* zmask, const int64_t* blk_off,
                                                           const int64_t* slot, const char* home, char* arena,
                                                           int64_t region, int L, int l0, int Lr, int Hq, int Hkv,
                                                           int m_cap, int es, int nch) {
    const int unit = blockIdx.x / nch, ch = blockIdx.x % nch;
    const int kvh = unit % Hkv, bl = unit / Hkv, b = bl / Lr, l = l0 + bl % Lr;
    const int G = Hq / Hkv, mw = m_cap / 32;
    const uint32_t* zm = zmask + (((int64_t)b * L + l) * Hq + (int64_t)kvh * G) * mw;
    const int64_t* bo = blk_off + (int64_t)b * (m_cap + 1);
    const int64_t* sl = slot + ((int64_t)b * L + l) * m_cap;
    const int64_t rbase = ((int64_t)b * L + l) * region;
    constexpr int U = 4;                                    // 16-byte vectors in flight per thread
    int rank = 0;                                           // zoomed spans passed so far
    for (int w = 0; w < mw; ++w) {
        uint32_t u = 0u;
        for (int g = 0; g < G; ++g) u |= zm[(int64_t)g * mw + w];
        for (; u; u &= u - 1u) {
            const int S = w * 32 + __ffs(u) - 1;
            if (rank++ % nch != ch) continue;
            const int64_t off = sl[S];
            if (off < 0) continue;
            const int64_t be = (bo[S + 1] - bo[S]) / Hkv;   // elements of one kv head's block
            const uint4* src = reinterpret_cast<const uint4*>(home + (rbase + bo[S] + kvh * be) * es);
            uint4* dst = reinterpret_cast<uint4*>(arena + (off + kvh * be) * es);
            const int64_t n16 = be * es / 16;
            for (int64_t i = threadIdx.x; i < n16; i += (int64_t)U * blockDim.x) {
                uint4 v[U];
#pragma unroll
                for (int k = 0; k < U; ++k) {
                    const int64_t j = i + (int64_t)k * blockDim.x;
                    v[k] = j < n16 ? src[j] : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int k = 0; k < U; ++k) {
                    const int64_t j = i + (int64_t)k * blockDim.x;
                    if (j < n16) dst[j] = v[k];
                }
            }
        }
    }
}

// Keep-mode gather: up to kGatherRuns contiguous runs (whole entries: every kv
// head's block of consecutive spans of one (b, l)) per launch, passed by value;
// nch CTAs share a run, each a contiguous share of its 16-byte vectors.
constexpr int kGatherRuns = 256;
struct GatherRuns {
    int64_t src[kGatherRuns], dst[kGatherRuns], n16[kGatherRuns];   // byte offsets / 16, vector counts
    int count;
};
__global__ void __launch_bounds__(256) run_gather_kernel(const __grid_constant__ GatherRuns gr, const char* home,
                                                         char* arena, int nch) {
    const int r = blockIdx.x / nch, ch = blockIdx.x % nch;
    if (r >= gr.count) return;
    const int64_t n = gr.n16[r], per = (n + nch - 1) / nch, i0 = ch * per, i1 = min(n, i0 + per);
    const uint4* src = reinterpret_cast<const uint4*>(home) + gr.src[r];
    uint4* dst = reinterpret_cast<uint4*>(arena) + gr.dst[r];
    constexpr int U = 4;
    for (int64_t i = i0 + threadIdx.x; i < i1; i += (int64_t)U * blockDim.x) {
        uint4 v[U];
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const int64_t j = i + (int64_t)k * blockDim.x;
            v[k] = j < i1 ? src[j] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const int64_t j = i + (int64_t)k * blockDim.x;
            if (j < i1) dst[j] = v[k];
        }
    }
}

}  // namespace sekv

namespace {

// Keep mode: the arena as a cache of span entries across calls. Entry (b, l, S)
// holds span S's Hkv blocks of layer l at [slot, slot + blk_off[S+1] - blk_off[S]).
// Misses are placed first-fit in the free gaps; when none is large enough, entries
// are evicted least recently used first (by last_use, then (b, l, S)) among those
// that neither this call nor the calls of this step or the previous one needed:
// an ATTEND of those steps may still be reading them. Nothing is changed on the
// host or the device unless every miss finds room.
struct KeepPlan {
    struct Copy { int64_t src, dst, width; int b, l; };
    std::vector<int64_t> hit;                           // slot-table indices of the hits
    std::vector<Copy> copies;
    std::vector<std::pair<int64_t, int64_t>> evict;     // (index into the slot table, unused)
    std::vector<std::pair<int64_t, int64_t>> place;     // (index into the slot table, slot)
    std::vector<uint8_t> dirty;                         // per layer: slot rows to upload
    int64_t hits = 0, spans = 0, bytes_elems = 0, used = 0;
    int64_t top = -1;                                   // end of the highest entry after the plan
};

bool plan_keep(const sekv_fetch_desc* d, KeepPlan& kp) {
    const int mw = d->m_cap / 32;
    const int64_t step = d->step;
    auto idx = [&](int b, int l, int S) { return ((int64_t)b * d->L + l) * d->m_cap + S; };
    auto size_of = [&](int b, int S) {
        const int64_t* bo = d->blk_off_host + (int64_t)b * (d->m_cap + 1);
        return bo[S + 1] - bo[S];
    };
    // spans this call needs: any head of (b, l) zooms them (rows of [l0, l1) only)
    const int Lr = d->l1 - d->l0;
    std::vector<uint32_t> needw((size_t)d->B * Lr * mw, 0u);
    int64_t misses = 0, need = 0;                     // spans to place and their elements
    struct Miss { int b, l, S; };
    std::vector<Miss> miss;                             // in (b, l, S) order
    for (int b = 0; b < d->B; ++b) {
        const int m = d->m_count_host[b] < d->m_cap ? d->m_count_host[b] : d->m_cap;
        for (int l = d->l0; l < d->l1; ++l) {
            uint32_t* uni = needw.data() + ((size_t)b * Lr + (l - d->l0)) * mw;
            const uint32_t* zm = d->zmask_host + ((int64_t)b * d->L + l) * d->Hq * mw;
            for (int h = 0; h < d->Hq; ++h)
                for (int w = 0; w < mw; ++w) uni[w] |= zm[h * mw + w];
            if (m < d->m_cap) {                                   // bits of spans >= m_count are ignored
                for (int w = m >> 5; w < mw; ++w) uni[w] &= (w == (m >> 5)) ? ((1u << (m & 31)) - 1u) : 0u;
            }
            for (int w = 0; w < mw; ++w)
                for (uint32_t bits = uni[w]; bits; bits &= bits - 1u) {
                    const int S = (w << 5) + __builtin_ctz(bits);
                    if (d->slot_host[idx(b, l, S)] >= 0) {
                        kp.hit.push_back(idx(b, l, S));
                    } else {
                        ++misses;
                        need += size_of(b, S);
                        miss.push_back({b, l, S});
                    }
                }
        }
    }
    auto needed = [&](int b, int l, int S) {
        if (l < d->l0 || l >= d->l1) return false;
        return ((needw[((size_t)b * Lr + (l - d->l0)) * mw + (S >> 5)] >> (S & 31)) & 1u) != 0u;
    };
    kp.hits = (int64_t)kp.hit.size();
    kp.dirty.assign(d->L, 0);
    if (misses == 0) {                                    // nothing to place: no scan of the arena
        kp.used = d->arena_used ? *d->arena_used : 0;
        return true;
    }
    // Fast path: the end of the highest resident entry, and the misses placed one
    // after another above it when they fit there (nothing is evicted then; only when
    // they do not fit are the gaps searched and entries evicted).
    {
        int64_t top = 0, held = 0;
        if (d->arena_top) {
            top = *d->arena_top;                          // the caller keeps it with the slot table
            held = d->arena_used ? *d->arena_used : 0;
        } else {
            for (int b = 0; b < d->B; ++b) {
                const int m = d->m_count_host[b] < d->m_cap ? d->m_count_host[b] : d->m_cap;
                const int64_t* bo = d->blk_off_host + (int64_t)b * (d->m_cap + 1);
                for (int l = 0; l < d->L; ++l) {
                    const int64_t* sl = d->slot_host + idx(b, l, 0);
                    for (int S = 0; S < m; ++S) {         // branch-free: vectorises
                        const int64_t sz = bo[S + 1] - bo[S];
                        const bool r = sl[S] >= 0;
                        top = std::max(top, r ? sl[S] + sz : 0);
                        held += r ? sz : 0;
                    }
                }
            }
        }
        if (top >= 0 && top + need <= d->arena_elems) {
            kp.used = held;
            for (size_t i = 0; i < miss.size();) {
                const int b = miss[i].b, l = miss[i].l, Sa = miss[i].S;
                size_t j = i + 1;                        // a run of consecutive missing spans
                while (j < miss.size() && miss[j].b == b && miss[j].l == l && miss[j].S == Sa + (int)(j - i)) ++j;
                const int Se = Sa + (int)(j - i);
                const int64_t* bo = d->blk_off_host + (int64_t)b * (d->m_cap + 1);
                const int64_t width = bo[Se] - bo[Sa];
                const int64_t src = ((int64_t)b * d->L + l) * d->region_elems + bo[Sa];
                for (int t = Sa; t < Se; ++t) kp.place.push_back({idx(b, l, t), top + (bo[t] - bo[Sa])});
                kp.copies.push_back({src, top, width, b, l});
                top += width;
                kp.spans += Se - Sa;
                kp.bytes_elems += width;
                kp.used += width;
                kp.dirty[l] = 1;
                i = j;
            }
            kp.top = top;
            return true;
        }
    }
    // resident entries: the occupied intervals and the eviction candidates
    struct Ent { int64_t last, off, size, id; int b, l; };
    std::vector<Ent> occ, cand;
    for (int b = 0; b < d->B; ++b) {
        const int m = d->m_count_host[b] < d->m_cap ? d->m_count_host[b] : d->m_cap;
        for (int l = 0; l < d->L; ++l)
            for (int S = 0; S < m; ++S) {
                const int64_t i = idx(b, l, S), off = d->slot_host[i];
                if (off < 0) continue;
                const Ent e{d->last_use[i], off, size_of(b, S), i, b, l};
                occ.push_back(e);
                if (!needed(b, l, S) && e.last < step - 1) cand.push_back(e);
            }
    }
    std::sort(occ.begin(), occ.end(), [](const Ent& x, const Ent& y) { return x.off < y.off; });
    std::sort(cand.begin(), cand.end(), [](const Ent& x, const Ent& y) {
        return x.last != y.last ? x.last < y.last : x.id < y.id;
    });
    std::map<int64_t, int64_t> gaps;                    // offset -> elements
    int64_t cur = 0;
    for (const Ent& e : occ) {
        if (e.off > cur) gaps[cur] = e.off - cur;
        cur = std::max(cur, e.off + e.size);
        kp.used += e.size;
    }
    if (d->arena_elems > cur) gaps[cur] = d->arena_elems - cur;
    auto release = [&](int64_t off, int64_t size) {
        auto nx = gaps.lower_bound(off);
        if (nx != gaps.end() && nx->first == off + size) {
            size += nx->second;
            nx = gaps.erase(nx);
        }
        if (nx != gaps.begin()) {
            auto pv = std::prev(nx);
            if (pv->first + pv->second == off) {
                pv->second += size;
                return;
            }
        }
        gaps[off] = size;
    };
    size_t next_victim = 0;
    std::vector<char> gone((size_t)d->B * d->L * d->m_cap, 0);   // evicted by this plan
    int64_t top = 0;                                   // end of the highest entry after the plan
    auto alloc = [&](int64_t size) -> int64_t {
        for (;;) {
            for (auto it = gaps.begin(); it != gaps.end(); ++it) {
                if (it->second < size) continue;
                const int64_t off = it->first, rest = it->second - size;
                gaps.erase(it);
                if (rest > 0) gaps[off + size] = rest;
                return off;
            }
            if (next_victim >= cand.size()) return -1;
            const Ent& v = cand[next_victim++];
            gone[v.id] = 1;
            kp.evict.push_back({v.id, 0});
            kp.dirty[v.l] = 1;
            kp.used -= v.size;
            release(v.off, v.size);
        }
    };
    for (int b = 0; b < d->B; ++b) {
        const int m = d->m_count_host[b] < d->m_cap ? d->m_count_host[b] : d->m_cap;
        const int64_t* bo = d->blk_off_host + (int64_t)b * (d->m_cap + 1);
        for (int l = d->l0; l < d->l1; ++l) {
            int S = 0;
            while (S < m) {
                const int64_t i = idx(b, l, S);
                if (!needed(b, l, S) || d->slot_host[i] >= 0) { ++S; continue; }
                const int Sa = S;                        // a run of consecutive misses
                while (S < m && needed(b, l, S) && d->slot_host[idx(b, l, S)] < 0) ++S;
                const int64_t width = bo[S] - bo[Sa];
                const int64_t src = ((int64_t)b * d->L + l) * d->region_elems + bo[Sa];
                int64_t off = alloc(width);
                if (off >= 0) {
                    for (int t = Sa; t < S; ++t) kp.place.push_back({idx(b, l, t), off + (bo[t] - bo[Sa])});
                    kp.copies.push_back({src, off, width, b, l});
                    top = std::max(top, off + width);
                } else {
                    // no room for the whole run: place its spans one by one
                    for (int t = Sa; t < S; ++t) {
                        const int64_t w1 = bo[t + 1] - bo[t];
                        const int64_t o1 = alloc(w1);
                        if (o1 < 0) return false;
                        kp.place.push_back({idx(b, l, t), o1});
                        kp.copies.push_back({src + (bo[t] - bo[Sa]), o1, w1, b, l});
                        top = std::max(top, o1 + w1);
                    }
                }
                kp.spans += S - Sa;
                kp.bytes_elems += width;
                kp.used += width;
                kp.dirty[l] = 1;
            }
        }
    }
    for (const Ent& e : occ)
        if (!gone[e.id]) top = std::max(top, e.off + e.size);
    kp.top = top;
    return true;
}

}  // namespace

extern "C" {

// The home's device address when the device can read it (pinned or registered host
// memory through unified addressing, or device memory), else null.
static const char* device_home(const void* home) {
    cudaPointerAttributes pa;
    if (cudaPointerGetAttributes(&pa, home) != cudaSuccess) {
        (void)cudaGetLastError();                       // an unregistered host pointer: not an error here
        return nullptr;
    }
    if (pa.type == cudaMemoryTypeHost && pa.devicePointer) return reinterpret_cast<const char*>(pa.devicePointer);
    if (pa.type == cudaMemoryTypeDevice || pa.type == cudaMemoryTypeManaged) return reinterpret_cast<const char*>(home);
    return nullptr;
}

sekv_status sekv_fetch_bases(const sekv_fetch_desc* d, sekv_stream_t compute, sekv_stream_t copy,
                             sekv_event_t done) {
    SEKV_REQUIRE(d, "fetch: null descriptor");
    SEKV_REQUIRE(d->zmask_dev && d->zmask_host && d->m_count_host && d->blk_off_host && d->home && d->arena &&
                     d->slot_dev && d->slot_host && done,
                 "fetch: missing pointer or event");
    SEKV_REQUIRE(d->B >= 1 && d->L >= 1 && d->Hq >= 1 && d->Hkv >= 1 && d->l0 >= 0 && d->l0 < d->l1 &&
                     d->l1 <= d->L && d->m_cap >= 32 && d->m_cap % 32 == 0 && d->region_elems > 0 &&
                     d->arena_elems >= 0 && (d->dtype == SEKV_F32 || d->dtype == SEKV_BF16),
                 "fetch: bad shape");
    SEKV_REQUIRE(d->keep == 0 || (d->keep == 1 && d->last_use && d->step >= 0),
                 "fetch: keep must be 0 or 1, and keep mode needs last_use and a step >= 0");
    SEKV_REQUIRE(!d->route_done || d->keep == 1,
                 "fetch: route_done (a fetch that overlaps earlier ATTEND calls) needs keep mode: a refill "
                 "would overwrite bases those calls may still read");
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(compute);
    cudaStream_t xs = reinterpret_cast<cudaStream_t>(copy);
    cudaEvent_t ev = reinterpret_cast<cudaEvent_t>(done);
    const int mw = d->m_cap / 32, Lr = d->l1 - d->l0;
    const int64_t es = esize(d->dtype);
    cudaError_t e;
    // the previous call's slot upload must be finished before the mirror is rewritten
    if ((e = cudaEventSynchronize(ev)) != cudaSuccess) return cuda_fail(e, "fetch: previous done event");
    // the routing result: after route_done on the copy stream (the compute stream may
    // already hold later work), else on the compute stream after all its work
    cudaStream_t rs = cs;
    if (d->route_done) {
        if ((e = cudaStreamWaitEvent(xs, reinterpret_cast<cudaEvent_t>(d->route_done), 0)) != cudaSuccess)
            return cuda_fail(e, "fetch: wait for route_done");
        rs = xs;
    }
    for (int b = 0; b < d->B; ++b) {
        const int64_t w0 = ((int64_t)b * d->L + d->l0) * d->Hq * mw;
        if ((e = cudaMemcpyAsync(d->zmask_host + w0, d->zmask_dev + w0, sizeof(uint32_t) * Lr * d->Hq * mw,
                                 cudaMemcpyDeviceToHost, rs)) != cudaSuccess)
            return cuda_fail(e, "fetch: zmask readback");
    }
    // the host needs the routing result; without route_done this also orders the
    // copies after the previous step's ATTEND (which ran earlier on `compute`)
    if ((e = cudaStreamSynchronize(rs)) != cudaSuccess) return cuda_fail(e, "fetch: routing result");
    const char* home = reinterpret_cast<const char*>(d->home);
    char* arena = reinterpret_cast<char*>(d->arena);

    if (d->keep == 1) {
        KeepPlan kp;
        if (!plan_keep(d, kp)) {
            if ((e = cudaEventRecord(ev, xs)) != cudaSuccess) return cuda_fail(e, "fetch: record");
            return fail(SEKV_ERR_CAPACITY,
                        "fetch: the zoomed bases that are not resident do not fit the arena of %lld elements "
                        "even after evicting every span this step and the previous one do not need",
                        (long long)d->arena_elems);
        }
        for (const auto& v : kp.evict) d->slot_host[v.first] = -1;
        for (const auto& p : kp.place) {
            d->slot_host[p.first] = p.second;
            d->last_use[p.first] = d->step;
        }
        for (const int64_t i : kp.hit) d->last_use[i] = d->step;     // hits are stamped too
        // the placed runs: by a gather kernel when the device can read the home (no
        // fixed cost per run), else one copy-engine copy each
        const char* hd = kp.copies.empty() ? nullptr : device_home(d->home);
        if (hd) {
            int dev = 0, sms = 148;
            if (cudaGetDevice(&dev) != cudaSuccess ||
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
                sms = 148;
            for (size_t c0 = 0; c0 < kp.copies.size(); c0 += sekv::kGatherRuns) {
                sekv::GatherRuns gr;
                gr.count = (int)std::min<size_t>(sekv::kGatherRuns, kp.copies.size() - c0);
                for (int k = 0; k < gr.count; ++k) {
                    const auto& c = kp.copies[c0 + k];
                    gr.src[k] = c.src * es / 16;
                    gr.dst[k] = c.dst * es / 16;
                    gr.n16[k] = c.width * es / 16;
                }
                const int nch = std::max(1, std::min(16, (4 * sms + gr.count - 1) / gr.count));
                sekv::run_gather_kernel<<<gr.count * nch, 256, 0, xs>>>(gr, hd, arena, nch);
                if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "fetch: gather");
            }
        } else {
            for (const auto& c : kp.copies)
                if ((e = cudaMemcpyAsync(arena + c.dst * es, home + c.src * es, c.width * es, cudaMemcpyHostToDevice,
                                         xs)) != cudaSuccess)
                    return cuda_fail(e, "fetch: basis copy");
        }
        // the slot rows of the layers that changed: one copy per sequence over the
        // range from the first to the last such layer (the copy engine's fixed cost
        // per copy outweighs the few unchanged rows in between)
        int lf = d->L, ll = -1;
        for (int l = 0; l < d->L; ++l)
            if (kp.dirty[l]) {
                lf = std::min(lf, l);
                ll = l;
            }
        for (int b = 0; b < d->B && ll >= lf; ++b) {
            const int64_t o = ((int64_t)b * d->L + lf) * d->m_cap;
            if ((e = cudaMemcpyAsync(d->slot_dev + o, d->slot_host + o, sizeof(int64_t) * d->m_cap * (ll - lf + 1),
                                     cudaMemcpyHostToDevice, xs)) != cudaSuccess)
                return cuda_fail(e, "fetch: slot upload");
        }
        if (d->stats) {
            d->stats[0] = kp.bytes_elems * es;
            d->stats[1] = kp.spans;
            d->stats[2] = (int64_t)kp.copies.size();
            d->stats[3] = kp.hits;
            d->stats[4] = (int64_t)kp.evict.size();
        }
        if (d->arena_used) *d->arena_used = kp.used;
        if (d->arena_top && kp.top >= 0) *d->arena_top = kp.top;
        if ((e = cudaEventRecord(ev, xs)) != cudaSuccess) return cuda_fail(e, "fetch: record");
        return SEKV_OK;
    }

    // Refill mode. A span's blocks sit at the same offset blk_off[b][S] of every
    // layer's region, so a run of consecutive spans zoomed in a run of consecutive
    // layers is one pitched rectangle of the home: width = the spans' blocks,
    // height = the layers, source pitch = the region. The copy engine pays a fixed
    // cost per copy (a few microseconds), so one rectangle per (span run, layer run)
    // instead of one copy per (span run, layer) is what keeps the fetch near the
    // PCIe rate.
    struct Rect { int64_t src, dst, width, height; };
    std::vector<Rect> rects;
    std::vector<uint32_t> uni;
    std::vector<uint64_t> lmask;
    int dev = 0, max_pitch = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&max_pitch, cudaDevAttrMaxPitch, dev) != cudaSuccess)
        max_pitch = 0;
    const bool pitched = (int64_t)max_pitch >= d->region_elems * es;
    int64_t end = 0, spans = 0;
    for (int b = 0; b < d->B; ++b) {
        const int m = d->m_count_host[b] < d->m_cap ? d->m_count_host[b] : d->m_cap;
        const int64_t* bo = d->blk_off_host + (int64_t)b * (d->m_cap + 1);
        for (int l = d->l0; l < d->l1; ++l) {
            int64_t* sl = d->slot_host + ((int64_t)b * d->L + l) * d->m_cap;
            for (int S = 0; S < d->m_cap; ++S) sl[S] = -1;
        }
        // layers in chunks of 64: lmask[S] bit j = span S zoomed (by any head) in layer lc + j
        for (int lc = d->l0; lc < d->l1; lc += 64) {
            const int nl = d->l1 - lc < 64 ? d->l1 - lc : 64;
            lmask.assign(m, 0ull);
            uni.assign(mw, 0u);
            for (int j = 0; j < nl; ++j) {
                std::fill(uni.begin(), uni.end(), 0u);
                const uint32_t* zm = d->zmask_host + ((int64_t)b * d->L + lc + j) * d->Hq * mw;
                for (int h = 0; h < d->Hq; ++h)
                    for (int w = 0; w < mw; ++w) uni[w] |= zm[h * mw + w];
                for (int S = 0; S < m; ++S)
                    if ((uni[S >> 5] >> (S & 31)) & 1u) lmask[S] |= 1ull << j;
            }
            int S = 0;
            while (S < m) {
                if (!lmask[S]) { ++S; continue; }
                const int Sa = S;
                const uint64_t mk = lmask[S];
                while (S < m && lmask[S] == mk) ++S;      // spans [Sa, S) share the layer set
                const int64_t width = bo[S] - bo[Sa];
                spans += (int64_t)(S - Sa) * __builtin_popcountll(mk);
                int j = 0;
                while (j < nl) {
                    if (!((mk >> j) & 1ull)) { ++j; continue; }
                    const int ja = j;
                    while (j < nl && ((mk >> j) & 1ull)) ++j;   // layers [lc + ja, lc + j)
                    const int hgt = j - ja;
                    for (int q = 0; q < hgt; ++q) {
                        int64_t* sl = d->slot_host + ((int64_t)b * d->L + lc + ja + q) * d->m_cap;
                        for (int t = Sa; t < S; ++t) sl[t] = end + (int64_t)q * width + (bo[t] - bo[Sa]);
                    }
                    const int64_t src = ((int64_t)b * d->L + lc + ja) * d->region_elems + bo[Sa];
                    if (pitched) {
                        rects.push_back({src, end, width, hgt});
                    } else {
                        for (int q = 0; q < hgt; ++q)
                            rects.push_back({src + (int64_t)q * d->region_elems, end + (int64_t)q * width, width, 1});
                    }
                    end += (int64_t)hgt * width;
                }
            }
        }
    }
    if (d->stats) {
        d->stats[0] = 0;
        for (const Rect& r : rects) d->stats[0] += r.width * r.height * es;
        d->stats[1] = spans;
        d->stats[2] = (int64_t)rects.size();
        d->stats[3] = 0;
        d->stats[4] = 0;
    }
    if (end > d->arena_elems) {
        // nothing is copied and the device slot table stays as it was
        if ((e = cudaEventRecord(ev, xs)) != cudaSuccess) return cuda_fail(e, "fetch: record");
        return fail(SEKV_ERR_CAPACITY, "fetch: zoomed bases need %lld elements, arena holds %lld",
                    (long long)end, (long long)d->arena_elems);
    }
    if (d->arena_used) *d->arena_used = end;
    // With the device block offsets and a home the device can address, one gather
    // kernel moves only the kv-head blocks the kv groups zoom (the copy engine would
    // move every zoomed span's Hkv blocks, and pays a fixed cost per copy).
    const char* home_dev = d->blk_off_dev ? device_home(d->home) : nullptr;
    if (home_dev) {
        for (int b = 0; b < d->B; ++b) {
            const int64_t o = ((int64_t)b * d->L + d->l0) * d->m_cap;
            if ((e = cudaMemcpyAsync(d->slot_dev + o, d->slot_host + o, sizeof(int64_t) * Lr * d->m_cap,
                                     cudaMemcpyHostToDevice, xs)) != cudaSuccess)
                return cuda_fail(e, "fetch: slot upload");
        }
        const int G = d->Hq / d->Hkv;
        int64_t blocks = 0, bytes = 0;
        for (int b = 0; b < d->B; ++b) {
            const int64_t* bo = d->blk_off_host + (int64_t)b * (d->m_cap + 1);
            for (int l = d->l0; l < d->l1; ++l)
                for (int kvh = 0; kvh < d->Hkv; ++kvh) {
                    const uint32_t* zm = d->zmask_host + (((int64_t)b * d->L + l) * d->Hq + (int64_t)kvh * G) * mw;
                    const int64_t* sl = d->slot_host + ((int64_t)b * d->L + l) * d->m_cap;
                    for (int w = 0; w < mw; ++w) {
                        uint32_t u = 0u;
                        for (int g = 0; g < G; ++g) u |= zm[(int64_t)g * mw + w];
                        for (; u; u &= u - 1u) {
                            const int S = (w << 5) + __builtin_ctz(u);
                            if (sl[S] < 0) continue;
                            ++blocks;
                            bytes += (bo[S + 1] - bo[S]) / d->Hkv * es;
                        }
                    }
                }
        }
        if (d->stats) {
            d->stats[0] = bytes;
            d->stats[2] = blocks;
        }
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            sms = 148;
        const int64_t units = (int64_t)d->B * Lr * d->Hkv;
        const int nch = (int)std::max<int64_t>(1, std::min<int64_t>(32, (8 * (int64_t)sms + units - 1) / units));
        if (units * nch > 0x7fffffff) return fail(SEKV_ERR_INVALID_ARG, "fetch: too many (b, layer, kv head) units");
        sekv::fetch_gather_kernel<<<(unsigned)(units * nch), 256, 0, xs>>>(
            d->zmask_dev, d->blk_off_dev, d->slot_dev, home_dev, arena, d->region_elems, d->L, d->l0, Lr, d->Hq,
            d->Hkv, d->m_cap, (int)es, nch);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "fetch: gather");
        if ((e = cudaEventRecord(ev, xs)) != cudaSuccess) return cuda_fail(e, "fetch: record");
        return SEKV_OK;
    }
    for (const Rect& r : rects) {
        if (r.height == 1)
            e = cudaMemcpyAsync(arena + r.dst * es, home + r.src * es, r.width * es, cudaMemcpyHostToDevice, xs);
        else
            e = cudaMemcpy2DAsync(arena + r.dst * es, r.width * es, home + r.src * es, d->region_elems * es,
                                  r.width * es, r.height, cudaMemcpyHostToDevice, xs);
        if (e != cudaSuccess) return cuda_fail(e, "fetch: basis copy");
    }
    for (int b = 0; b < d->B; ++b) {
        const int64_t o = ((int64_t)b * d->L + d->l0) * d->m_cap;
        if ((e = cudaMemcpyAsync(d->slot_dev + o, d->slot_host + o, sizeof(int64_t) * Lr * d->m_cap,
                                 cudaMemcpyHostToDevice, xs)) != cudaSuccess)
            return cuda_fail(e, "fetch: slot upload");
    }
    if ((e = cudaEventRecord(ev, xs)) != cudaSuccess) return cuda_fail(e, "fetch: record");
    return SEKV_OK;
}

}  // extern "C"
