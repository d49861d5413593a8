// K-b: anchor gather and per-span weighted-mean key/value.
//
// SeKV blog walkthrough, section 2.1 (anchors kept at full resolution) and
// section 2.2 (Eq. (2) surprisal weights; weighted means kbar_S, vbar_S kept in
// the original key/value space for the coarse entries of non-expanded spans);
// SeKV summary page, workflow paragraph (kbar_S = sum w_t K_t / sum w_t).
// With the identity routing projection Eq. (3)'s routing summary is kbar / ||kbar||:
// the kernel stores 1/||stored kbar|| beside it. With a learned projection W^(l,h)
// (route_W) it also writes the dr-dimensional routing summaries per query head.
//
// Both kernels are HBM-bound single passes: every K/V row of the layer range is
// read exactly once (anchor rows by the gather, span rows by the means).
#include "sekv_common.cuh"
#include "sekv_internal.h"

namespace sekv {

constexpr int kGatherThreads = 256;
constexpr int kGatherRows = 64;        // anchor rows per CTA
constexpr int kMeanWarps = 8;          // spans per CTA (one warp each)

// grid: (ceil(a_cap / kGatherRows), Hkv, B * Lr)
__global__ void __launch_bounds__(kGatherThreads)
gather_anchors_kernel(const char* __restrict__ K, const char* __restrict__ V, char* Ka, char* Va,
                      const int32_t* a_count, const int32_t* anchor_pos, int L, int l0, int Lr,
                      int Hkv, int n, int a_cap, int row_bytes, int32_t* status) {
    const int kvh = blockIdx.y;
    const int b = blockIdx.z / Lr, l = l0 + blockIdx.z % Lr;
    const int a = min(a_count[b], a_cap);
    const int r0 = blockIdx.x * kGatherRows;
    if (r0 >= a) return;
    const int rows = min(kGatherRows, a - r0);
    const int64_t unit = ((int64_t)b * L + l) * Hkv + kvh;
    const char* srcK = K + unit * n * row_bytes;
    const char* srcV = V + unit * n * row_bytes;
    char* dstK = Ka + (unit * a_cap + r0) * row_bytes;
    char* dstV = Va + (unit * a_cap + r0) * row_bytes;
    const int vec = row_bytes / 16;
    for (int i = threadIdx.x; i < rows * vec; i += blockDim.x) {
        const int r = i / vec, c = i % vec;
        const int pos = anchor_pos[(int64_t)b * a_cap + r0 + r];
        if (pos < 0 || pos >= n) {            // caller-supplied segmentation out of range
            set_status(status, SEKV_ERR_INVALID_ARG);
            continue;
        }
        const uint4 k = *reinterpret_cast<const uint4*>(srcK + (int64_t)pos * row_bytes + c * 16);
        const uint4 v = *reinterpret_cast<const uint4*>(srcV + (int64_t)pos * row_bytes + c * 16);
        *reinterpret_cast<uint4*>(dstK + (int64_t)r * row_bytes + c * 16) = k;
        *reinterpret_cast<uint4*>(dstV + (int64_t)r * row_bytes + c * 16) = v;
    }
}

// Learned-form routing summaries (SeKV blog 2.2 Eq. (3)): per query head h of the
// kv head, y = sum_t w_t W^(l,h) K_t = (sum_t w_t) W^(l,h) kbar_S, stored as
// y / ||y||. The positive weight sum cancels, so y is formed from the warp's
// unrounded fp32 mean. W of the CTA's G query heads is staged once per CTA in
// shared memory (storage dtype) with rows padded by 4 elements, which makes the
// 4-element row reads of 8 (fp32) or 16 (bf16) lanes at a time conflict-free;
// lane j owns routing output j (and j + 32 when dr = 64).
struct RouteSum {
    const void* W;      // [L][Hq][dr][D] storage dtype, or null
    void* out;          // [B][L][Hq][m_cap][dr] storage dtype
    int Hq, G, dr;
};

constexpr int kRoutePad = 4;     // elements of padding per staged W row
constexpr int kRouteGMax = 8;    // query heads per kv head

template <int DT, int D>
__host__ __device__ inline size_t route_stage_bytes(int G, int dr) {
    return (size_t)G * dr * (D + kRoutePad) * Elt<DT>::bytes;
}

// grid: (chunks, Hkv, B * Lr); warp w of chunk c handles spans c*kMeanWarps + w,
// then every gridDim.x*kMeanWarps-th span after it. One warp per span; each lane
// owns DPL = d/32 consecutive dimensions of the means.
template <int DT, int DPL, bool RT>
__global__ void __launch_bounds__(kMeanWarps * 32)
span_means_kernel(const void* __restrict__ K, const void* __restrict__ V, const float* __restrict__ H,
                  void* kbar, void* vbar, float* inv_norm, const int32_t* m_count,
                  const int32_t* span_beg, const int32_t* span_end, int L, int l0, int Lr, int Hkv,
                  int n, int m_cap, int wmode, RouteSum rt, int32_t* status) {
    constexpr int D = DPL * 32;
    constexpr int WS = D + kRoutePad;
    using E = Elt<DT>;
    extern __shared__ __align__(16) unsigned char sm_route[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int kvh = blockIdx.y;
    const int b = blockIdx.z / Lr, l = l0 + blockIdx.z % Lr;
    const int m = min(m_count[b], m_cap);
    float* ks = nullptr;
    if constexpr (RT) {
        // stage W^(l, h) of the kv head's G query heads, row-padded
        const int rows = rt.G * rt.dr;
        const char* src = reinterpret_cast<const char*>(rt.W) +
                          ((int64_t)l * rt.Hq + (int64_t)kvh * rt.G) * rt.dr * D * E::bytes;
        for (int i = threadIdx.x; i < rows * (D / 4); i += blockDim.x) {
            const int row = i / (D / 4), c = (i % (D / 4)) * 4;
            unsigned char* dst = sm_route + ((int64_t)row * WS + c) * E::bytes;
            const char* s4 = src + ((int64_t)row * D + c) * E::bytes;
            if (DT == SEKV_F32) *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(s4);
            else *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(s4);
        }
        ks = reinterpret_cast<float*>(sm_route + route_stage_bytes<DT, D>(rt.G, rt.dr)) + warp * D;
        __syncthreads();
    }
    const float* h = H + (int64_t)b * n;
    const int64_t unit = ((int64_t)b * L + l) * Hkv + kvh;
    const char* Kr = reinterpret_cast<const char*>(K) + (unit * n) * D * E::bytes + lane * DPL * E::bytes;
    const char* Vr = reinterpret_cast<const char*>(V) + (unit * n) * D * E::bytes + lane * DPL * E::bytes;

    for (int S = blockIdx.x * kMeanWarps + warp; S < m; S += gridDim.x * kMeanWarps) {
        const int beg = span_beg[(int64_t)b * m_cap + S], end = span_end[(int64_t)b * m_cap + S];
        if (beg < 0 || end > n || end <= beg) {
            if (lane == 0) set_status(status, SEKV_ERR_INVALID_ARG);
            continue;
        }
        // weight mode resolution (Eq. (2) falls back to uniform when sum H = 0)
        int mode = wmode;
        float hmax = 0.f;
        if (mode != SEKV_W_UNIFORM) {
            float acc = (mode == SEKV_W_SURPRISAL) ? 0.f : -INFINITY;
            for (int t = beg + lane; t < end; t += 32)
                acc = (mode == SEKV_W_SURPRISAL) ? acc + h[t] : fmaxf(acc, h[t]);
            if (mode == SEKV_W_SURPRISAL) {
                if (warp_sum(acc) == 0.f) mode = SEKV_W_UNIFORM;
            } else {
                hmax = warp_max(acc);
            }
        }
        float ak[DPL], av[DPL];
#pragma unroll
        for (int i = 0; i < DPL; ++i) ak[i] = av[i] = 0.f;
        float wsum = 0.f;
        int t = beg;
        for (; t + 4 <= end; t += 4) {
            float kk[4][DPL], vv[4][DPL], w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                Vec<DT, DPL>::load(Kr + (int64_t)(t + u) * D * E::bytes, kk[u]);
                Vec<DT, DPL>::load(Vr + (int64_t)(t + u) * D * E::bytes, vv[u]);
                const float hv = h[t + u];
                w[u] = (mode == SEKV_W_UNIFORM) ? 1.f : (mode == SEKV_W_SURPRISAL) ? hv : expf(hv - hmax);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                wsum += w[u];
#pragma unroll
                for (int i = 0; i < DPL; ++i) {
                    ak[i] = fmaf(w[u], kk[u][i], ak[i]);
                    av[i] = fmaf(w[u], vv[u][i], av[i]);
                }
            }
        }
        for (; t < end; ++t) {
            float kk[DPL], vv[DPL];
            Vec<DT, DPL>::load(Kr + (int64_t)t * D * E::bytes, kk);
            Vec<DT, DPL>::load(Vr + (int64_t)t * D * E::bytes, vv);
            const float hv = h[t];
            const float w = (mode == SEKV_W_UNIFORM) ? 1.f : (mode == SEKV_W_SURPRISAL) ? hv : expf(hv - hmax);
            wsum += w;
#pragma unroll
            for (int i = 0; i < DPL; ++i) {
                ak[i] = fmaf(w, kk[i], ak[i]);
                av[i] = fmaf(w, vv[i], av[i]);
            }
        }
        const int64_t row = (unit * m_cap + S) * D + lane * DPL;
        float nrm = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) {
            const float km = ak[i] / wsum;
            const float k = round_storage<DT>(km);
            store1<DT>(kbar, row + i, k);
            store1<DT>(vbar, row + i, av[i] / wsum);
            nrm = fmaf(k, k, nrm);
            if constexpr (RT) ks[lane * DPL + i] = km;
        }
        nrm = warp_sum(nrm);
        if (lane == 0) inv_norm[unit * m_cap + S] = nrm > 0.f ? 1.0f / sqrtf(nrm) : 0.f;
        if constexpr (RT) {
            __syncwarp();
            const int DRW = rt.dr >> 5;        // outputs per lane: 1 or 2
            float y[kRouteGMax][2];
#pragma unroll
            for (int g = 0; g < kRouteGMax; ++g) y[g][0] = y[g][1] = 0.f;
            for (int i0 = 0; i0 < D; i0 += 4) {
                float kv[4];
#pragma unroll
                for (int v = 0; v < 4; ++v) kv[v] = ks[i0 + v];
#pragma unroll
                for (int g = 0; g < kRouteGMax; ++g) {
                    if (g >= rt.G) break;
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        if (jj >= DRW) break;
                        float wv[4];
                        Vec<DT, 4>::load(sm_route + ((int64_t)(g * rt.dr + jj * 32 + lane) * WS + i0) * E::bytes, wv);
#pragma unroll
                        for (int v = 0; v < 4; ++v) y[g][jj] = fmaf(wv[v], kv[v], y[g][jj]);
                    }
                }
            }
#pragma unroll
            for (int g = 0; g < kRouteGMax; ++g) {
                if (g >= rt.G) break;
                float n2 = 0.f;
#pragma unroll
                for (int jj = 0; jj < 2; ++jj)
                    if (jj < DRW) n2 = fmaf(y[g][jj], y[g][jj], n2);
                n2 = warp_sum(n2);
                const float inv = n2 > 0.f ? 1.0f / sqrtf(n2) : 0.f;
                const int64_t orow = ((((int64_t)b * L + l) * rt.Hq + (int64_t)kvh * rt.G + g) * m_cap + S) * rt.dr;
#pragma unroll
                for (int jj = 0; jj < 2; ++jj)
                    if (jj < DRW) store1<DT>(rt.out, orow + jj * 32 + lane, y[g][jj] * inv);
            }
            __syncwarp();
        }
    }
}

// shared memory of the routing-summary variant (W of G heads + one mean per warp)
static size_t route_summary_smem(int dtype, int d, int G, int dr) {
    const size_t w = (size_t)G * dr * (d + kRoutePad) * (dtype == SEKV_F32 ? 4 : 2);
    return w + (size_t)kMeanWarps * d * 4;
}

bool route_summary_supported(const sekv_build_desc& d) {
    if (d.Hkv < 1 || d.Hq < d.Hkv || d.Hq % d.Hkv) return false;
    const int G = d.Hq / d.Hkv;
    if (G > kRouteGMax || (d.dr != 32 && d.dr != 64)) return false;
    return route_summary_smem(d.dtype, d.d, G, d.dr) <= 200 * 1024;
}

cudaError_t launch_summary(const sekv_build_desc& d, cudaStream_t st) {
    const int Lr = d.l1 - d.l0;
    const int esz = d.dtype == SEKV_F32 ? 4 : 2;
    dim3 gg((d.a_cap + kGatherRows - 1) / kGatherRows, d.Hkv, d.B * Lr);
    gather_anchors_kernel<<<gg, kGatherThreads, 0, st>>>(
        (const char*)d.K, (const char*)d.V, (char*)d.Ka, (char*)d.Va, d.a_count, d.anchor_pos, d.L,
        d.l0, Lr, d.Hkv, d.n, d.a_cap, d.d * esz, d.dev_status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int chunks = (d.m_cap + kMeanWarps - 1) / kMeanWarps;
    RouteSum rt{d.route_W, d.kbar_r, d.Hq, d.Hkv > 0 && d.Hq >= d.Hkv ? d.Hq / d.Hkv : 1, d.dr};
    if (!d.route_W) {
        dim3 gm(chunks, d.Hkv, d.B * Lr);
#define SEKV_MEANS(DT, DPL)                                                                        \
        span_means_kernel<DT, DPL, false><<<gm, kMeanWarps * 32, 0, st>>>(                         \
            d.K, d.V, d.H, d.kbar, d.vbar, d.inv_norm, d.m_count, d.span_beg, d.span_end, d.L, d.l0, \
            Lr, d.Hkv, d.n, d.m_cap, d.wmode, rt, d.dev_status)
        if (d.dtype == SEKV_F32) {
            if (d.d == 64) SEKV_MEANS(SEKV_F32, 2); else SEKV_MEANS(SEKV_F32, 4);
        } else {
            if (d.d == 64) SEKV_MEANS(SEKV_BF16, 2); else SEKV_MEANS(SEKV_BF16, 4);
        }
#undef SEKV_MEANS
        return cudaGetLastError();
    }
    // routing variant: fewer, longer-lived CTAs so each staged W serves many spans
    const int gx = chunks < 16 ? chunks : 16;
    dim3 gm(gx, d.Hkv, d.B * Lr);
    const size_t smem = route_summary_smem(d.dtype, d.d, rt.G, d.dr);
#define SEKV_MEANS_RT(DT, DPL)                                                                     \
    do {                                                                                           \
        e = cudaFuncSetAttribute(span_means_kernel<DT, DPL, true>,                                 \
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);          \
        if (e != cudaSuccess) return e;                                                            \
        span_means_kernel<DT, DPL, true><<<gm, kMeanWarps * 32, smem, st>>>(                       \
            d.K, d.V, d.H, d.kbar, d.vbar, d.inv_norm, d.m_count, d.span_beg, d.span_end, d.L, d.l0, \
            Lr, d.Hkv, d.n, d.m_cap, d.wmode, rt, d.dev_status);                                   \
    } while (0)
    if (d.dtype == SEKV_F32) {
        if (d.d == 64) SEKV_MEANS_RT(SEKV_F32, 2); else SEKV_MEANS_RT(SEKV_F32, 4);
    } else {
        if (d.d == 64) SEKV_MEANS_RT(SEKV_BF16, 2); else SEKV_MEANS_RT(SEKV_BF16, 4);
    }
#undef SEKV_MEANS_RT
    return cudaGetLastError();
}

}  // namespace sekv
