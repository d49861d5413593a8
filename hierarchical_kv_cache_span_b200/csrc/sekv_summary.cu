// K-b: anchor gather and per-span weighted-mean key/value.
//
// SeKV blog walkthrough, section 2.1 (anchors kept at full resolution) and
// section 2.2 (Eq. (2) surprisal weights; weighted means kbar_S, vbar_S kept in
// the original key/value space for the coarse entries of non-expanded spans);
// SeKV summary page, workflow paragraph (kbar_S = sum w_t K_t / sum w_t).
// The routing projection is the identity here, so Eq. (3)'s routing summary is
// kbar / ||kbar||: the kernel stores 1/||stored kbar|| beside it.
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

// grid: (ceil(m_cap / kMeanWarps), Hkv, B * Lr); one warp per span, each lane owns
// DPL = d/32 consecutive dimensions.
template <int DT, int DPL>
__global__ void __launch_bounds__(kMeanWarps * 32)
span_means_kernel(const void* __restrict__ K, const void* __restrict__ V, const float* __restrict__ H,
                  void* kbar, void* vbar, float* inv_norm, const int32_t* m_count,
                  const int32_t* span_beg, const int32_t* span_end, int L, int l0, int Lr, int Hkv,
                  int n, int m_cap, int wmode, int32_t* status) {
    constexpr int D = DPL * 32;
    using E = Elt<DT>;
    const int lane = threadIdx.x & 31;
    const int S = blockIdx.x * kMeanWarps + (threadIdx.x >> 5);
    const int kvh = blockIdx.y;
    const int b = blockIdx.z / Lr, l = l0 + blockIdx.z % Lr;
    if (S >= min(m_count[b], m_cap)) return;
    const int beg = span_beg[(int64_t)b * m_cap + S], end = span_end[(int64_t)b * m_cap + S];
    if (beg < 0 || end > n || end <= beg) {
        if (lane == 0) set_status(status, SEKV_ERR_INVALID_ARG);
        return;
    }
    const float* h = H + (int64_t)b * n;
    const int64_t unit = ((int64_t)b * L + l) * Hkv + kvh;
    const char* Kr = reinterpret_cast<const char*>(K) + (unit * n) * D * E::bytes + lane * DPL * E::bytes;
    const char* Vr = reinterpret_cast<const char*>(V) + (unit * n) * D * E::bytes + lane * DPL * E::bytes;

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
        const float k = round_storage<DT>(ak[i] / wsum);
        store1<DT>(kbar, row + i, k);
        store1<DT>(vbar, row + i, av[i] / wsum);
        nrm = fmaf(k, k, nrm);
    }
    nrm = warp_sum(nrm);
    if (lane == 0) inv_norm[unit * m_cap + S] = nrm > 0.f ? 1.0f / sqrtf(nrm) : 0.f;
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
    dim3 gm((d.m_cap + kMeanWarps - 1) / kMeanWarps, d.Hkv, d.B * Lr);
#define SEKV_MEANS(DT, DPL)                                                                        \
    span_means_kernel<DT, DPL><<<gm, kMeanWarps * 32, 0, st>>>(                                    \
        d.K, d.V, d.H, d.kbar, d.vbar, d.inv_norm, d.m_count, d.span_beg, d.span_end, d.L, d.l0, Lr, \
        d.Hkv, d.n, d.m_cap, d.wmode, d.dev_status)
    if (d.dtype == SEKV_F32) {
        if (d.d == 64) SEKV_MEANS(SEKV_F32, 2); else SEKV_MEANS(SEKV_F32, 4);
    } else {
        if (d.d == 64) SEKV_MEANS(SEKV_BF16, 2); else SEKV_MEANS(SEKV_BF16, 4);
    }
#undef SEKV_MEANS
    return cudaGetLastError();
}

}  // namespace sekv
