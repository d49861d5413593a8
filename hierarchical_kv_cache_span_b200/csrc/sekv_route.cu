// Learned-form routing pass (Stage 1 with a routing projection).
//
// SeKV blog walkthrough, section 2.3: the current query is projected into the
// routing space and compared with every span's routing summary (Eq. (3), built
// by the summary step), Eq. (5):
//     l_S = (W^(l,h) q_h) . kbar_r_S / sqrt(d') + log|S|,
// and Eq. (9) zooms span S iff sigma(l_S) > tau, i.e. l_S > theta = ln(tau/(1-tau)).
// The same W^(l,h) projects the query and the keys (the plainest reading of
// "the query projected into the routing space").
//
// One CTA per (b, l, query head): q~ = W q (dr x d, fp32) into shared memory, then
// one thread per span streams the dr-element summary rows (HBM-bound: dr * 2
// bytes per span and head in bf16), the next row loaded before the current one
// is used; zoom bits are formed by warp ballots, 32 spans per mask word. Words
// past the last span are written as zero so the mask is fully defined.
#include <math.h>

#include "sekv_common.cuh"
#include "sekv_internal.h"

namespace sekv {

constexpr int kRouteThreads = 256;

template <int DT, int DR>
struct RouteRow {
    static constexpr int bytes = DR * Elt<DT>::bytes;
    static constexpr int vecs = bytes / 16;
    uint4 v[vecs];
    SEKV_DEV void load(const char* p) {
#pragma unroll
        for (int i = 0; i < vecs; ++i) v[i] = __ldg(reinterpret_cast<const uint4*>(p) + i);
    }
    SEKV_DEV float dot(const float* qt) const {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < vecs; ++i) {
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (DT == SEKV_F32) {
                    acc = fmaf(__uint_as_float(w[k]), qt[i * 4 + k], acc);
                } else {
                    acc = fmaf(bf16_lo(w[k]), qt[i * 8 + 2 * k], acc);
                    acc = fmaf(bf16_hi(w[k]), qt[i * 8 + 2 * k + 1], acc);
                }
            }
        }
        return acc;
    }
};

template <int DT, int DR>
__global__ void __launch_bounds__(kRouteThreads)
route_learned_kernel(const void* __restrict__ q, const void* __restrict__ W, const void* __restrict__ kbar_r,
                     const float* __restrict__ logS, const float* __restrict__ theta, const int32_t* m_count,
                     uint32_t* zmask, float* logits, int L, int l0, int Lr, int Hq, int d, int m_cap,
                     float rscale) {
    using E = Elt<DT>;
    __shared__ float qt[DR];
    const int idx = blockIdx.x;
    const int h = idx % Hq, li = (idx / Hq) % Lr, b = idx / (Hq * Lr);
    const int l = l0 + li;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int m = min(m_count[b], m_cap);
    const int64_t head = ((int64_t)b * L + l) * Hq + h;
    const char* rows = reinterpret_cast<const char*>(kbar_r) + head * m_cap * (int64_t)RouteRow<DT, DR>::bytes;

    // first row in flight before the projection
    RouteRow<DT, DR> cur;
    if (tid < m) cur.load(rows + (int64_t)tid * RouteRow<DT, DR>::bytes);

    // q~ = W^(l,h) q_h: TPJ threads per output, strided over the d inputs
    constexpr int TPJ = kRouteThreads / DR;
    {
        const int j = tid / TPJ, p = tid % TPJ;
        const int64_t wrow = (((int64_t)l * Hq + h) * DR + j) * d;
        const int64_t qrow = head * d;
        float acc = 0.f;
        for (int i = p; i < d; i += TPJ) acc = fmaf(load1<DT>(W, wrow + i), load1<DT>(q, qrow + i), acc);
#pragma unroll
        for (int o = TPJ / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (p == 0) qt[j] = acc;
    }
    __syncthreads();
    const float th = theta[(int64_t)l * Hq + h];
    uint32_t* zw = zmask + head * (m_cap / 32);
    float* lg = logits ? logits + head * m_cap : nullptr;
    const int mw32 = (m + 31) & ~31;
    for (int S0 = 0; S0 < mw32; S0 += kRouteThreads) {
        const int S = S0 + tid;
        const bool valid = S < m;
        RouteRow<DT, DR> nxt;
        if (S + kRouteThreads < m) nxt.load(rows + (int64_t)(S + kRouteThreads) * RouteRow<DT, DR>::bytes);
        bool z = false;
        if (valid) {
            const float ell = cur.dot(qt) * rscale + logS[(int64_t)b * m_cap + S];   // Eq. (5)
            z = ell > th;                                                           // Eq. (9)
            if (lg) lg[S] = ell;
        }
        const uint32_t bits = __ballot_sync(0xffffffffu, z);
        if (lane == 0 && S0 + warp * 32 < mw32) zw[(S0 >> 5) + warp] = bits;
        cur = nxt;
    }
    for (int w = (mw32 >> 5) + tid; w < m_cap / 32; w += kRouteThreads) zw[w] = 0u;
}

bool route_learned_supported(const sekv_decode_desc& d) {
    return (d.dr == 32 || d.dr == 64) && d.d % 32 == 0 && d.Hq >= 1;
}

cudaError_t launch_route_learned(const sekv_decode_desc& d, cudaStream_t st) {
    const int Lr = d.l1 - d.l0;
    const unsigned grid = (unsigned)(d.B * Lr * d.Hq);
    if (grid == 0) return cudaSuccess;
    const float rscale = (float)(1.0 / sqrt((double)d.dr));
#define SEKV_ROUTE_L(DT, DR)                                                                        \
    route_learned_kernel<DT, DR><<<grid, kRouteThreads, 0, st>>>(d.q, d.route_W, d.kbar_r, d.logS, d.theta, \
                                                                 d.m_count, d.zmask, d.route_logits, d.L, \
                                                                 d.l0, Lr, d.Hq, d.d, d.m_cap, rscale)
    if (d.dtype == SEKV_F32) {
        if (d.dr == 32) SEKV_ROUTE_L(SEKV_F32, 32); else SEKV_ROUTE_L(SEKV_F32, 64);
    } else {
        if (d.dr == 32) SEKV_ROUTE_L(SEKV_BF16, 32); else SEKV_ROUTE_L(SEKV_BF16, 64);
    }
#undef SEKV_ROUTE_L
    return cudaGetLastError();
}

}  // namespace sekv
