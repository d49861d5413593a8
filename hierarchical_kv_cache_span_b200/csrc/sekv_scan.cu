// K-a: surprisal boundary scan and span layout.
//
// SeKV blog walkthrough, section 2.1: H_t = -log p(x_t | x_<t) (Eq. (1)); a span
// boundary wherever H_t > mu + alpha*sigma with mu, sigma the mean and std of the
// in-context surprisal; boundary tokens are kept as full-resolution anchors.
// Fig. 2 adds the local window. Spans are the maximal runs of non-anchor tokens.
//
// One CTA per sequence (1024 threads, a contiguous chunk of positions each):
// fp64 two-pass mean / population variance with a fixed reduction tree (so the
// threshold is deterministic), then an in-CTA exclusive scan of three counters
// (anchors, span starts, span ends) compacts positions. No inter-CTA waits.
#include "sekv_common.cuh"
#include "sekv_internal.h"

namespace sekv {

constexpr int kScanThreads = 1024;

__device__ double block_sum_f64(double v, double* red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) red[wid] = v;
    __syncthreads();
    if (wid == 0) {
        v = (lane < (int)(blockDim.x >> 5)) ? red[lane] : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[0] = v;
    }
    __syncthreads();
    double r = red[0];
    __syncthreads();
    return r;
}

// exclusive scan of an int64 per thread; returns the prefix, *total = block sum
__device__ int64_t block_exscan_i64(int64_t v, int64_t* buf, int64_t* total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    __syncthreads();
    if (lane == 31) buf[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int64_t w = (lane < nw) ? buf[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int64_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        buf[lane] = w;   // inclusive over warps
    }
    __syncthreads();
    int64_t warp_base = wid ? buf[wid - 1] : 0;
    *total = buf[nw - 1];
    __syncthreads();
    return warp_base + x - v;
}

__global__ void __launch_bounds__(kScanThreads)
scan_kernel(const float* __restrict__ H, int n, double alpha, int window, int a_cap, int m_cap,
            int32_t* a_count, int32_t* m_count, int32_t* anchor_pos, int32_t* span_beg,
            int32_t* span_end, double* stats, int32_t* status) {
    __shared__ double red[32];
    __shared__ int64_t sbuf[32];
    const int b = blockIdx.x;
    const float* h = H + (int64_t)b * n;
    const int tid = threadIdx.x;
    const int chunk = (n + kScanThreads - 1) / kScanThreads;
    const int t0 = min(n, tid * chunk), t1 = min(n, t0 + chunk);

    double s = 0.0;
    for (int t = t0; t < t1; ++t) s += (double)h[t];
    const double mu = block_sum_f64(s, red) / (double)n;
    double v = 0.0;
    for (int t = t0; t < t1; ++t) {
        double dd = (double)h[t] - mu;
        v += dd * dd;
    }
    const double sigma = sqrt(block_sum_f64(v, red) / (double)n);
    const double thr = mu + alpha * sigma;
    const int wstart = n - window;   // positions >= wstart are window anchors
    auto is_anchor = [&](int t) -> bool { return (double)h[t] > thr || t >= wstart; };

    // counts: anchors, span starts, span ends (packed 21 bits each is too tight
    // for n = 2^17, so three scans of a packed pair + one)
    int na = 0, ns = 0, ne = 0;
    bool prev = (t0 > 0) ? is_anchor(t0 - 1) : true;
    for (int t = t0; t < t1; ++t) {
        const bool a = is_anchor(t);
        if (a) {
            ++na;
        } else {
            if (prev) ++ns;
            const bool next = (t + 1 < n) ? is_anchor(t + 1) : true;
            if (next) ++ne;
        }
        prev = a;
    }
    int64_t tot_a, tot_s, tot_e;
    // pack anchors (low 32 bits) and starts (high 32 bits) in one scan; ends in a second
    const int64_t packed = (int64_t)na | ((int64_t)ns << 32);
    int64_t tot_p;
    const int64_t pre_p = block_exscan_i64(packed, sbuf, &tot_p);
    const int64_t pre_e = block_exscan_i64((int64_t)ne, sbuf, &tot_e);
    tot_a = tot_p & 0xffffffffLL;
    tot_s = tot_p >> 32;
    int ia = (int)(pre_p & 0xffffffffLL), is = (int)(pre_p >> 32), ie = (int)pre_e;

    prev = (t0 > 0) ? is_anchor(t0 - 1) : true;
    for (int t = t0; t < t1; ++t) {
        const bool a = is_anchor(t);
        if (a) {
            if (ia < a_cap) anchor_pos[(int64_t)b * a_cap + ia] = t;
            ++ia;
        } else {
            if (prev) {
                if (is < m_cap) span_beg[(int64_t)b * m_cap + is] = t;
                ++is;
            }
            const bool next = (t + 1 < n) ? is_anchor(t + 1) : true;
            if (next) {
                if (ie < m_cap) span_end[(int64_t)b * m_cap + ie] = t + 1;
                ++ie;
            }
        }
        prev = a;
    }
    if (tid == 0) {
        a_count[b] = (int32_t)(tot_a < a_cap ? tot_a : (int64_t)a_cap);
        m_count[b] = (int32_t)(tot_s < m_cap ? tot_s : (int64_t)m_cap);
        if (tot_a > a_cap || tot_s > m_cap) set_status(status, SEKV_ERR_CAPACITY);
        if (stats) {
            stats[b * 3 + 0] = mu;
            stats[b * 3 + 1] = sigma;
            stats[b * 3 + 2] = thr;
        }
    }
}

// logS and the basis block offsets of every span of sequence b.
__global__ void __launch_bounds__(kScanThreads)
layout_kernel(const int32_t* m_count, const int32_t* span_beg, const int32_t* span_end, int m_cap,
              int Hkv, int d, int rank, int64_t region_elems, float* logS, int64_t* blk_off,
              int32_t* status) {
    __shared__ int64_t sbuf[32];
    const int b = blockIdx.x;
    const int m = min(m_count[b], m_cap);
    int64_t carry = 0;
    for (int base = 0; base < m; base += kScanThreads) {
        const int S = base + threadIdx.x;
        int64_t e = 0;
        if (S < m) {
            const int len = span_end[(int64_t)b * m_cap + S] - span_beg[(int64_t)b * m_cap + S];
            if (len <= 0) set_status(status, SEKV_ERR_INVALID_ARG);
            const int l = len > 0 ? len : 1;
            e = (int64_t)Hkv * block_elems(l, d, rank);
            logS[(int64_t)b * m_cap + S] = (float)log((double)l);
        }
        int64_t tot;
        const int64_t pre = block_exscan_i64(e, sbuf, &tot);
        if (S < m) blk_off[(int64_t)b * (m_cap + 1) + S] = carry + pre;
        carry += tot;
    }
    if (threadIdx.x == 0) {
        blk_off[(int64_t)b * (m_cap + 1) + m] = carry;
        if (region_elems >= 0 && carry > region_elems) set_status(status, SEKV_ERR_CAPACITY);
    }
}

cudaError_t launch_scan(const sekv_build_desc& d, cudaStream_t st) {
    scan_kernel<<<d.B, kScanThreads, 0, st>>>(d.H, d.n, d.alpha, d.window, d.a_cap, d.m_cap,
                                              d.a_count, d.m_count, d.anchor_pos, d.span_beg,
                                              d.span_end, d.stats, d.dev_status);
    return cudaGetLastError();
}

cudaError_t launch_layout(const sekv_build_desc& d, bool check_region, cudaStream_t st) {
    layout_kernel<<<d.B, kScanThreads, 0, st>>>(d.m_count, d.span_beg, d.span_end, d.m_cap, d.Hkv,
                                                d.d, d.rank, check_region ? d.region_elems : -1,
                                                d.logS, d.blk_off, d.dev_status);
    return cudaGetLastError();
}

}  // namespace sekv
