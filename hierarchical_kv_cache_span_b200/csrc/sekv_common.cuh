// Device-side helpers shared by the SeKV kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sekv.h"

#define SEKV_DEV __device__ __forceinline__

namespace sekv {

constexpr int kWarp = 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------------------
// element types: DT 0 = float, 1 = bfloat16
// ---------------------------------------------------------------------------
template <int DT> struct Elt;
template <> struct Elt<SEKV_F32> {
    using T = float;
    static constexpr int bytes = 4;
};
template <> struct Elt<SEKV_BF16> {
    using T = __nv_bfloat16;
    static constexpr int bytes = 2;
};

SEKV_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
SEKV_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// load N (2 or 4) consecutive elements starting at p (aligned to N elements) as floats
template <int DT, int N> struct Vec;
template <> struct Vec<SEKV_F32, 4> {
    SEKV_DEV static void load(const void* p, float* v) {
        float4 x = *reinterpret_cast<const float4*>(p);
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    }
};
template <> struct Vec<SEKV_F32, 2> {
    SEKV_DEV static void load(const void* p, float* v) {
        float2 x = *reinterpret_cast<const float2*>(p);
        v[0] = x.x; v[1] = x.y;
    }
};
template <> struct Vec<SEKV_BF16, 4> {
    SEKV_DEV static void load(const void* p, float* v) {
        uint2 x = *reinterpret_cast<const uint2*>(p);
        v[0] = bf16_lo(x.x); v[1] = bf16_hi(x.x); v[2] = bf16_lo(x.y); v[3] = bf16_hi(x.y);
    }
};
template <> struct Vec<SEKV_BF16, 2> {
    SEKV_DEV static void load(const void* p, float* v) {
        uint32_t x = *reinterpret_cast<const uint32_t*>(p);
        v[0] = bf16_lo(x); v[1] = bf16_hi(x);
    }
};

template <int DT> SEKV_DEV float load1(const void* p, int64_t i);
template <> SEKV_DEV float load1<SEKV_F32>(const void* p, int64_t i) {
    return reinterpret_cast<const float*>(p)[i];
}
template <> SEKV_DEV float load1<SEKV_BF16>(const void* p, int64_t i) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
}

template <int DT> SEKV_DEV void store1(void* p, int64_t i, float v);
template <> SEKV_DEV void store1<SEKV_F32>(void* p, int64_t i, float v) {
    reinterpret_cast<float*>(p)[i] = v;
}
template <> SEKV_DEV void store1<SEKV_BF16>(void* p, int64_t i, float v) {
    reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
}
// value after a round trip through the storage type
template <int DT> SEKV_DEV float round_storage(float v);
template <> SEKV_DEV float round_storage<SEKV_F32>(float v) { return v; }
template <> SEKV_DEV float round_storage<SEKV_BF16>(float v) {
    return __bfloat162float(__float2bfloat16_rn(v));
}

// ---------------------------------------------------------------------------
// status: first error wins
// ---------------------------------------------------------------------------
SEKV_DEV void set_status(int32_t* st, int code) {
    if (st) atomicCAS(st, 0, code);
}

// ---------------------------------------------------------------------------
// basis block layout (must match sekv_block_elems on the host)
//   block = [ A | C | B | D ], every factor stored 8x8-blocked: an R x W matrix
//   (R, W padded with zeros to multiples of 8) is a row-major grid of 8 x 8 tiles,
//   each tile 64 contiguous elements, row-major inside. A and C are len8 x r8,
//   B and D are r8 x d, with len8 = roundup(|S|, 8), r8 = roundup(rS, 8).
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }
__host__ __device__ __forceinline__ int block_rank(int len, int d, int rank) {
    int r = rank < len ? rank : len;
    return r < d ? r : d;
}
__host__ __device__ __forceinline__ int round8(int x) { return (x + 7) & ~7; }
// elements of the A (and of the C) section
__host__ __device__ __forceinline__ int64_t block_ac_elems(int len, int rS) {
    return (int64_t)round8(len) * round8(rS);
}
__host__ __device__ __forceinline__ int64_t block_elems(int len, int d, int rank) {
    const int rS = block_rank(len, d, rank);
    return 2 * block_ac_elems(len, rS) + 2 * (int64_t)round8(rS) * d;
}
// position of element (r, c) of an 8x8-blocked matrix whose padded width is w8
__host__ __device__ __forceinline__ int64_t tile8_index(int64_t r, int c, int w8) {
    return ((r >> 3) * (w8 >> 3) + (c >> 3)) * 64 + ((r & 7) << 3) + (c & 7);
}

// ---------------------------------------------------------------------------
// mbarrier + bulk copy (1-D, global -> this CTA's shared memory)
// ---------------------------------------------------------------------------
SEKV_DEV uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

SEKV_DEV void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
SEKV_DEV void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
SEKV_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\t"
                 "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
SEKV_DEV void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\t"
                 "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
                 ::"r"(smem_u32(bar)) : "memory");
}
SEKV_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}
// Bounded wait: gives up after ~2^22 polls with back-off (far above any
// legitimate wait, well under a second of wall time).
constexpr uint32_t kWaitPolls = 1u << 22;
SEKV_DEV bool mbar_wait_n(uint64_t* bar, uint32_t parity, uint32_t polls) {
    for (uint32_t i = 0; i < polls; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if (i > 64) __nanosleep(64);
    }
    return false;
}
SEKV_DEV bool mbar_wait(uint64_t* bar, uint32_t parity) { return mbar_wait_n(bar, parity, kWaitPolls); }
SEKV_DEV void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst_smem)), "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
// 16 bytes global -> this thread's shared memory, cached in L2 only (both addresses
// 16-byte aligned); visible to the issuing thread after cp_async_wait_all()
SEKV_DEV void cp_async16(void* dst_smem, const void* src_gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem) : "memory");
}
SEKV_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// ---------------------------------------------------------------------------
// warp-level tensor-core helpers (ldmatrix + mma.sync m16n8k16 bf16 -> fp32)
// ---------------------------------------------------------------------------
// transpose an 8 x 8 bf16 matrix held as one mma fragment register per lane
// (lane l holds row l/4, columns 2(l%4), 2(l%4)+1; the result holds the transpose)
SEKV_DEV uint32_t movm_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// explicit shared-memory loads (a generic load of shared memory is slower)
SEKV_DEV uint32_t lds_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)));
    return v;
}
SEKV_DEV uint4 lds_u128(const void* p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(smem_u32(p)));
    return v;
}
SEKV_DEV float lds_f32(const void* p) { return __uint_as_float(lds_u32(p)); }

SEKV_DEV void ldsm_x4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_u32(p)));
}
SEKV_DEV void ldsm_x2(uint32_t (&r)[2], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1]) : "r"(smem_u32(p)));
}
SEKV_DEV void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_u32(p)));
}
SEKV_DEV void ldsm_x2_t(uint32_t (&r)[2], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1]) : "r"(smem_u32(p)));
}
SEKV_DEV void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

SEKV_DEV uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// 2-D tensor-map bulk copy (TMA) global -> this CTA's shared memory
SEKV_DEV void tma_load_2d(void* dst_smem, const void* tmap, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst_smem)), "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar)) : "memory");
}
SEKV_DEV void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// L2 policy for data read once per call (streamed rows, zoomed bases): evicted first,
// so the small data every CTA reads (queries, masks, span bounds, the code) stays
SEKV_DEV uint64_t l2_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
SEKV_DEV void tma_load_2d_ef(void* dst_smem, const void* tmap, int x, int y, uint64_t* bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;"
        ::"r"(smem_u32(dst_smem)), "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(pol) : "memory");
}
SEKV_DEV void bulk_g2s_ef(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        ::"r"(smem_u32(dst_smem)), "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar)), "l"(pol) : "memory");
}

// ---------------------------------------------------------------------------
// warp helpers
// ---------------------------------------------------------------------------
SEKV_DEV unsigned warp_sum_u(unsigned v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
SEKV_DEV float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
SEKV_DEV float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Transpose-reduce: every lane holds 32 partial sums v[0..31]; afterwards lane L
// holds the warp-wide sum of index L. 31 shuffles for 32 reductions.
SEKV_DEV float transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const bool up = lane & 16;
        float send = up ? v[i] : v[i + 16];
        float keep = up ? v[i + 16] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const bool up = lane & 8;
        float send = up ? v[i] : v[i + 8];
        float keep = up ? v[i + 8] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool up = lane & 4;
        float send = up ? v[i] : v[i + 4];
        float keep = up ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool up = lane & 2;
        float send = up ? v[i] : v[i + 2];
        float keep = up ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    {
        const bool up = lane & 1;
        float send = up ? v[0] : v[1];
        float keep = up ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
    }
    return v[0];
}

}  // namespace sekv
