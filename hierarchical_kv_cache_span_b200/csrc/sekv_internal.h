// Host-side launchers shared between the kernel files and the C ABI layer.
#pragma once

#include <cuda_runtime.h>

#include "../../include/sekv.h"

namespace sekv {

cudaError_t launch_scan(const sekv_build_desc& d, cudaStream_t st);
cudaError_t launch_layout(const sekv_build_desc& d, bool check_region, cudaStream_t st);
cudaError_t launch_summary(const sekv_build_desc& d, cudaStream_t st);
bool route_summary_supported(const sekv_build_desc& d);   // route_W shapes the summary step handles

// basis build: workspace layout and launch
size_t basis_workspace_bytes(const sekv_build_desc& d);
cudaError_t launch_basis(const sekv_build_desc& d, cudaStream_t st);

// decode
struct DecodePlan {
    int nsplit;        // CTAs per (b, l, kv head)
    int span_chunk;    // spans per split (multiple of 32)
    int anchor_chunk;  // anchors per split
    size_t partial_bytes;
    size_t logit_bytes;  // routing logits kept for the budget cap (after the partials)
};
DecodePlan plan_decode(const sekv_decode_desc& d);
size_t decode_workspace_bytes(const sekv_decode_desc& d);
bool decode_supported(const sekv_decode_desc& d);
cudaError_t launch_decode(const sekv_decode_desc& d, const DecodePlan& p, void* partials, cudaStream_t st);
// learned-form routing pass (zoom mask + optional logits); defined with its kernel
cudaError_t launch_route_learned(const sekv_decode_desc& d, cudaStream_t st);
bool route_learned_supported(const sekv_decode_desc& d);
cudaError_t launch_merge_parts(const float* O_parts, const float* lse_parts, int nparts, int64_t rows, int d,
                               float* O, float* lse, cudaStream_t st);
size_t decode_static_scratch_bytes();
void* decode_static_scratch(cudaError_t* err);

}  // namespace sekv
