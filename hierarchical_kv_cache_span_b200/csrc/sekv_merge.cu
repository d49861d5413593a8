// Log-sum-exp merge of decode results over disjoint parts of one logit list.
//
// SeKV summary, workflow paragraph (Stage 2): anchors, coarse span entries and the
// reconstructed tokens of zoomed spans share ONE softmax. A partition of that
// list (the context split across ranks) therefore recombines exactly:
//   M = max_p lse_p,  w_p = exp(lse_p - M),
//   O = sum_p w_p O_p / sum_p w_p,  lse = M + log sum_p w_p.
// lse is the natural-log value sekv_decode_attn writes. A part with lse = -inf
// has no entries for that row and weighs nothing; a row with no entries in any
// part gets O = 0 and lse = -inf, as sekv_decode_attn writes for an empty list.
//
// One CTA per row: the nparts (<= 64) weights are computed once into shared
// memory, then the d outputs are read coalesced across the CTA's threads.
#include <math.h>

#include "sekv_common.cuh"
#include "sekv_internal.h"

namespace sekv {

constexpr int kMergeMaxParts = 64;

__global__ void merge_parts_kernel(const float* O_parts, const float* lse_parts, int nparts, int64_t rows, int d,
                                   float* O, float* lse) {
    const int64_t row = blockIdx.x;
    __shared__ float w[kMergeMaxParts];
    __shared__ float s_inv;
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        float l0 = lane < nparts ? lse_parts[(int64_t)lane * rows + row] : -INFINITY;
        float l1 = lane + 32 < nparts ? lse_parts[(int64_t)(lane + 32) * rows + row] : -INFINITY;
        float M = fmaxf(l0, l1);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float w0 = M == -INFINITY ? 0.f : expf(l0 - M);
        const float w1 = M == -INFINITY ? 0.f : expf(l1 - M);
        w[lane] = w0;
        w[lane + 32] = w1;
        float Ls = w0 + w1;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
        if (lane == 0) {
            s_inv = Ls > 0.f ? 1.f / Ls : 0.f;
            lse[row] = Ls > 0.f ? M + logf(Ls) : -INFINITY;
        }
    }
    __syncthreads();
    const float inv = s_inv;
    for (int k = threadIdx.x; k < d; k += blockDim.x) {
        float o = 0.f;
        for (int p = 0; p < nparts; ++p)
            if (w[p] != 0.f) o = fmaf(w[p], O_parts[((int64_t)p * rows + row) * d + k], o);
        O[row * d + k] = o * inv;
    }
}

cudaError_t launch_merge_parts(const float* O_parts, const float* lse_parts, int nparts, int64_t rows, int d,
                               float* O, float* lse, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if (nparts < 1 || nparts > kMergeMaxParts) return cudaErrorInvalidValue;
    const int threads = d <= 128 ? 128 : (d > 1024 ? 1024 : ((d + 31) / 32) * 32);
    merge_parts_kernel<<<(unsigned)rows, threads, 0, st>>>(O_parts, lse_parts, nparts, rows, d, O, lse);
    return cudaGetLastError();
}

}  // namespace sekv
