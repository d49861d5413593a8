// K-c: batched per-span rank-r bases.
//
// SeKV blog walkthrough, section 2.2, Eq. (6)-(8): each span's key matrix (and
// value matrix) is stored as a truncated SVD, K_S ~ sum_{i<=R} m_i sigma_i u_i v_i^T;
// with the rank gate m_i = 1 for i <= r this is the rank-r truncation; a caller-
// supplied gate scales component i (row i of the stored B or D factor).
//
// Per (sequence, layer, kv head, span, K-or-V) problem with X = the span's rows
// (|S| x d) and N = min(|S|, d):
//   |S| <= d: G = X X^T (N x N), top-rS eigenvectors U_r, A = U_r, B = U_r^T X
//   |S| >  d: G = X^T X (N x N), top-rS eigenvectors V_r, A = X V_r, B = V_r^T
// so A B is the projection of X on its top-rS singular subspace (Eckart-Young).
// The symmetric eigenproblem is solved by the parallel cyclic Jacobi method
// (round-robin pairing, N/2 disjoint rotations per round) in shared memory, fp32.
// The Gram contraction runs on the tensor cores (mma.sync m16n8k16 bf16 -> fp32)
// for bf16 inputs and on the FMA pipes for fp32 inputs.
//
// Problems are bucketed by N (<= 32, <= 64, <= 128) so each bucket gets a
// shared-memory footprint and CTA size that fit it; each bucket is a persistent
// launch that pulls work items from an atomic counter.
#include "sekv_common.cuh"
#include "sekv_internal.h"

namespace sekv {

constexpr int kBuckets = 3;
constexpr int kChunkRows = 32;    // rows of X staged per step when |S| > d

struct BasisWork {
    int* bucket_count;   // [kBuckets]
    int* work_next;      // [kBuckets]
    int2* list;          // [kBuckets][B * m_cap]  (b, S)
};

static size_t list_cap(const sekv_build_desc& d) { return (size_t)d.B * d.m_cap; }

size_t basis_workspace_bytes(const sekv_build_desc& d) {
    return 256 + round_up(sizeof(int2) * kBuckets * list_cap(d), 256);
}

static BasisWork carve(const sekv_build_desc& d) {
    BasisWork w;
    char* p = reinterpret_cast<char*>(d.workspace);
    w.bucket_count = reinterpret_cast<int*>(p);
    w.work_next = reinterpret_cast<int*>(p + 64);
    w.list = reinterpret_cast<int2*>(p + 256);
    return w;
}

__global__ void classify_kernel(const int32_t* m_count, const int32_t* span_beg, const int32_t* span_end,
                                int m_cap, int dmodel, BasisWork w, size_t cap) {
    const int b = blockIdx.x;
    const int m = min(m_count[b], m_cap);
    for (int S = threadIdx.x; S < m; S += blockDim.x) {
        const int len = span_end[(int64_t)b * m_cap + S] - span_beg[(int64_t)b * m_cap + S];
        const int N = min(len, dmodel);
        const int bk = N <= 32 ? 0 : (N <= 64 ? 1 : 2);
        const int idx = atomicAdd(&w.bucket_count[bk], 1);
        w.list[(size_t)bk * cap + idx] = make_int2(b, S);
    }
}

struct BasisArgs {
    const int32_t* m_count;
    const void* K;
    const void* V;
    const int32_t* span_beg;
    const int32_t* span_end;
    const int64_t* blk_off;
    void* home;
    int32_t* status;
    const float* gate;   // null or [B][L][Hkv][m_cap][2][rank] rank gate m_{S,i} (Eq. (6))
    int64_t region;
    int L, l0, Lr, Hkv, n, d, m_cap, rank, max_sweeps;
};

// ---------------------------------------------------------------------------
// Gram on tensor cores: C[i][j] = sum_k P[i][k] Q[j][k] for bf16 row-major P, Q in
// shared memory (ldb elements per row, 16-byte aligned rows), M, N multiples of 16,
// Kdim a multiple of 16. Each warp takes 16x8 output tiles; fp32 accumulate.
// ---------------------------------------------------------------------------
// G (+)= X X^T over rows [0, M) of Xb (M x Kdim, row stride ldb elements).
SEKV_DEV void gram_rows_mma(float* G, int ldg, const __nv_bfloat16* Xb, int ldb, int M, int Kdim,
                            bool accumulate) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int tm = M / 16, tn = M / 8;
    for (int t = wid; t < tm * tn; t += nw) {
        const int i0 = (t / tn) * 16, j0 = (t % tn) * 8;
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k0 = 0; k0 < Kdim; k0 += 16) {
            uint32_t a[4], bb[2];
            // A fragment: rows i0..i0+15, cols k0..k0+15 (row-major)
            ldsm_x4(a, Xb + (size_t)(i0 + (lane & 15)) * ldb + k0 + ((lane >> 4) << 3));
            // B fragment (k x n, "col"): n = rows j0..j0+7 of X, k contiguous
            ldsm_x2(bb, Xb + (size_t)(j0 + (lane & 7)) * ldb + k0 + (((lane >> 3) & 1) << 3));
            mma_bf16_16816(c, a, bb);
        }
        const int r = i0 + (lane >> 2), cc = j0 + ((lane & 3) << 1);
        float* g0 = G + (size_t)r * ldg + cc;
        float* g1 = G + (size_t)(r + 8) * ldg + cc;
        if (accumulate) {
            g0[0] += c[0]; g0[1] += c[1]; g1[0] += c[2]; g1[1] += c[3];
        } else {
            g0[0] = c[0]; g0[1] = c[1]; g1[0] = c[2]; g1[1] = c[3];
        }
    }
}

// G (+)= Xc^T Xc for a chunk Xc (Krows x M, row stride ldb), Krows multiple of 16.
SEKV_DEV void gram_cols_mma(float* G, int ldg, const __nv_bfloat16* Xb, int ldb, int M, int Krows,
                            bool accumulate) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int tm = M / 16, tn = M / 8;
    for (int t = wid; t < tm * tn; t += nw) {
        const int i0 = (t / tn) * 16, j0 = (t % tn) * 8;
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k0 = 0; k0 < Krows; k0 += 16) {
            uint32_t a[4], bb[2];
            // A[i][k] = Xc[k][i]: transposed load of the 16x16 block (k0.., i0..)
            {
                const int mi = lane >> 3, rr = lane & 7;     // matrix index, row in matrix
                // matrices: 0:(k0..+7, i0..+7) 1:(k0..+7, i0+8..) 2:(k0+8.., i0..) 3:(k0+8.., i0+8..)
                // ldmatrix.trans of [k][i] tiles yields A-fragment order a0:(i0-7,k0-7) a1:(i8-15,k0-7)
                // a2:(i0-7,k8-15) a3:(i8-15,k8-15)
                const int kk = k0 + rr + ((mi >> 1) << 3);
                const int ii = i0 + ((mi & 1) << 3);
                ldsm_x4_t(a, Xb + (size_t)kk * ldb + ii);
            }
            // B[k][j] = Xc[k][j] ("col" operand wants k contiguous per n -> transposed load)
            {
                const int mi = (lane >> 3) & 1, rr = lane & 7;
                ldsm_x2_t(bb, Xb + (size_t)(k0 + rr + (mi << 3)) * ldb + j0);
            }
            mma_bf16_16816(c, a, bb);
        }
        const int r = i0 + (lane >> 2), cc = j0 + ((lane & 3) << 1);
        float* g0 = G + (size_t)r * ldg + cc;
        float* g1 = G + (size_t)(r + 8) * ldg + cc;
        if (accumulate) {
            g0[0] += c[0]; g0[1] += c[1]; g1[0] += c[2]; g1[1] += c[3];
        } else {
            g0[0] = c[0]; g0[1] = c[1]; g1[0] = c[2]; g1[1] = c[3];
        }
    }
}

// ---------------------------------------------------------------------------
// parallel cyclic Jacobi on the symmetric Ne x Ne matrix G (Ne even); Vm <- eigenvectors
// returns true when ||off||_F^2 <= tol2 * ||diag||_F^2
// ---------------------------------------------------------------------------
SEKV_DEV bool jacobi(float* G, float* Vm, int ld, int Ne, int max_sweeps, int* rp, int* rq, float* rc,
                     float* rs, float* red, float tol2) {
    const int tid = threadIdx.x, T = blockDim.x;
    const int half = Ne >> 1;
    for (int i = tid; i < Ne * Ne; i += T) Vm[(i / Ne) * ld + (i % Ne)] = (i / Ne == i % Ne) ? 1.f : 0.f;
    bool converged = false;
    for (int sweep = 0; sweep <= max_sweeps; ++sweep) {
        // convergence test
        float off = 0.f, dia = 0.f;
        for (int i = tid; i < Ne * Ne; i += T) {
            const int r = i / Ne, c = i % Ne;
            const float g = G[r * ld + c];
            if (r == c) dia = fmaf(g, g, dia); else off = fmaf(g, g, off);
        }
        off = warp_sum(off);
        dia = warp_sum(dia);
        if ((tid & 31) == 0) { red[2 * (tid >> 5)] = off; red[2 * (tid >> 5) + 1] = dia; }
        __syncthreads();
        float o = 0.f, dd = 0.f;
        for (int w = 0; w < (T >> 5); ++w) { o += red[2 * w]; dd += red[2 * w + 1]; }
        __syncthreads();
        if (o <= tol2 * dd) { converged = true; break; }
        if (sweep == max_sweeps) break;
        for (int rho = 0; rho < Ne - 1; ++rho) {
            if (tid < half) {
                const int k = tid;
                auto pos = [&](int i) { return i == 0 ? 0 : 1 + (i - 1 + rho) % (Ne - 1); };
                int p = pos(k), q = pos(Ne - 1 - k);
                if (p > q) { int t = p; p = q; q = t; }
                const float app = G[p * ld + p], aqq = G[q * ld + q], apq = G[p * ld + q];
                float c = 1.f, s = 0.f;
                if (fabsf(apq) > 1e-30f && fabsf(apq) > 1e-9f * sqrtf(fabsf(app * aqq))) {
                    const float zeta = (aqq - app) / (2.f * apq);
                    float t;
                    if (fabsf(zeta) > 1e15f) {
                        t = 0.5f / zeta;
                    } else {
                        t = 1.f / (fabsf(zeta) + sqrtf(fmaf(zeta, zeta, 1.f)));
                        if (zeta < 0.f) t = -t;
                    }
                    c = rsqrtf(fmaf(t, t, 1.f));
                    s = t * c;
                }
                rp[k] = p; rq[k] = q; rc[k] = c; rs[k] = s;
            }
            __syncthreads();
            // columns of G and of Vm: [x_p, x_q] <- [c x_p - s x_q, s x_p + c x_q]
            for (int i = tid; i < Ne * half; i += T) {
                const int r = i % Ne, k = i / Ne;
                const int p = rp[k], q = rq[k];
                const float c = rc[k], s = rs[k];
                float* g = G + r * ld;
                const float gp = g[p], gq = g[q];
                g[p] = c * gp - s * gq;
                g[q] = s * gp + c * gq;
                float* v = Vm + r * ld;
                const float vp = v[p], vq = v[q];
                v[p] = c * vp - s * vq;
                v[q] = s * vp + c * vq;
            }
            __syncthreads();
            // rows of G: [G_p., G_q.] <- [c G_p. - s G_q., s G_p. + c G_q.]
            for (int i = tid; i < Ne * half; i += T) {
                const int j = i % Ne, k = i / Ne;
                const int p = rp[k], q = rq[k];
                const float c = rc[k], s = rs[k];
                const float gp = G[p * ld + j], gq = G[q * ld + j];
                float np = c * gp - s * gq, nq = s * gp + c * gq;
                if (j == q) np = 0.f;      // the annihilated pair
                if (j == p) nq = 0.f;
                G[p * ld + j] = np;
                G[q * ld + j] = nq;
            }
            __syncthreads();
        }
    }
    return converged;
}

template <int DT, int NB>
__global__ void __launch_bounds__(NB * 4)
basis_kernel(BasisArgs a, BasisWork w, int bucket, size_t cap) {
    using E = Elt<DT>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int tid = threadIdx.x, T = blockDim.x;
    const int d = a.d;
    const int ld = NB + 1;           // fp32 G / Vm row stride
    // X staging: fp32 rows (stride d+1) for fp32 inputs, bf16 rows (stride d+8,
    // 16-byte aligned for ldmatrix) for bf16 inputs; bf16 values are exact in fp32.
    const int ldx = (DT == SEKV_BF16) ? d + 8 : d + 1;
    const int xrows = NB > kChunkRows ? NB : kChunkRows;
    float* G = reinterpret_cast<float*>(smem_raw);
    float* Vm = G + NB * ld;
    float* X = Vm + NB * ld;
    __nv_bfloat16* Xb = reinterpret_cast<__nv_bfloat16*>(X);
    auto xs = [&](int r, int c) -> float {
        return (DT == SEKV_BF16) ? __bfloat162float(Xb[r * ldx + c]) : X[r * ldx + c];
    };
    auto xput = [&](int r, int c, float v) {
        if (DT == SEKV_BF16) Xb[r * ldx + c] = __float2bfloat16_rn(v); else X[r * ldx + c] = v;
    };
    int* rp = reinterpret_cast<int*>(smem_raw + round_up((size_t)2 * NB * ld * 4 +
                                                          (size_t)xrows * ldx * (DT == SEKV_BF16 ? 2 : 4), 16));
    int* rq = rp + NB / 2;
    float* rc = reinterpret_cast<float*>(rq + NB / 2);
    float* rs = rc + NB / 2;
    float* red = rs + NB / 2;        // 2 * 32 floats
    int* sel = reinterpret_cast<int*>(red + 64);
    __shared__ int item_s;

    const int per_entry = a.Lr * a.Hkv * 2;
    const int total = w.bucket_count[bucket] * per_entry;
    for (;;) {
        if (tid == 0) item_s = atomicAdd(&w.work_next[bucket], 1);
        __syncthreads();
        const int item = item_s;
        __syncthreads();
        if (item >= total) break;
        const int2 bs = w.list[(size_t)bucket * cap + item / per_entry];
        const int rest = item % per_entry;
        const int which = rest & 1;                 // 0: keys -> (A, B); 1: values -> (C, D)
        const int kvh = (rest >> 1) % a.Hkv;
        const int l = a.l0 + (rest >> 1) / a.Hkv;
        const int b = bs.x, S = bs.y;
        const int beg = a.span_beg[(int64_t)b * a.m_cap + S];
        const int len = a.span_end[(int64_t)b * a.m_cap + S] - beg;
        const int64_t region_used = a.blk_off[(int64_t)b * (a.m_cap + 1) + min(a.m_count[b], a.m_cap)];
        if (beg < 0 || len < 1 || beg + len > a.n || region_used > a.region) {
            if (tid == 0) set_status(a.status, (region_used > a.region) ? SEKV_ERR_CAPACITY : SEKV_ERR_INVALID_ARG);
            continue;   // uniform across the CTA: the loop head re-synchronises
        }
        const int N = min(len, d);
        const int Ne = N + (N & 1);
        const int rS = block_rank(len, d, a.rank);
        const int r8 = round8(rS);
        const int64_t pa = block_ac_elems(len, rS);
        const bool rows_form = len <= d;            // G = X X^T
        // rank gate of component j (descending singular value), folded into row j of B / D
        const float* gate = a.gate ? a.gate + (((((int64_t)b * a.L + l) * a.Hkv + kvh) * a.m_cap + S) * 2 + which) *
                                                  (int64_t)a.rank
                                   : nullptr;
        const char* src = reinterpret_cast<const char*>(which ? a.V : a.K) +
                          ((((int64_t)b * a.L + l) * a.Hkv + kvh) * a.n + beg) * (int64_t)d * E::bytes;
        char* blk = reinterpret_cast<char*>(a.home) +
                    (((int64_t)b * a.L + l) * a.region + a.blk_off[(int64_t)b * (a.m_cap + 1) + S] +
                     (int64_t)kvh * block_elems(len, d, a.rank)) * E::bytes;
        char* fac_row = blk + (which ? pa : 0) * E::bytes;              // A or C: len8 x r8, 8x8-blocked
        char* fac_col = blk + (2 * pa + (which ? (int64_t)r8 * d : 0)) * E::bytes;  // B or D: r8 x d, 8x8-blocked

        // ---- Gram ---------------------------------------------------------------
        const int Mp = (N + 15) & ~15;              // padded for the MMA tiles
        for (int i = tid; i < Mp * ld; i += T) G[i] = 0.f;
        if (rows_form) {
            for (int i = tid; i < Mp * d; i += T) {
                const int r = i / d, c = i % d;
                xput(r, c, r < len ? load1<DT>(src, (int64_t)r * d + c) : 0.f);
            }
            __syncthreads();
            if (DT == SEKV_BF16) {
                gram_rows_mma(G, ld, Xb, ldx, Mp, d, false);
            } else {
                for (int i = tid; i < N * N; i += T) {
                    const int r = i / N, c = i % N;
                    float acc = 0.f;
                    for (int k = 0; k < d; ++k) acc = fmaf(X[r * ldx + k], X[c * ldx + k], acc);
                    G[r * ld + c] = acc;
                }
            }
        } else {
            __syncthreads();
            for (int t0 = 0; t0 < len; t0 += kChunkRows) {
                const int rows = min(kChunkRows, len - t0);
                for (int i = tid; i < kChunkRows * d; i += T) {
                    const int r = i / d, c = i % d;
                    xput(r, c, r < rows ? load1<DT>(src, (int64_t)(t0 + r) * d + c) : 0.f);
                }
                __syncthreads();
                if (DT == SEKV_BF16) {
                    gram_cols_mma(G, ld, Xb, ldx, Mp, kChunkRows, true);
                } else {
                    for (int i = tid; i < N * N; i += T) {
                        const int r = i / N, c = i % N;
                        float acc = G[r * ld + c];
                        for (int k = 0; k < rows; ++k) acc = fmaf(X[k * ldx + r], X[k * ldx + c], acc);
                        G[r * ld + c] = acc;
                    }
                }
                __syncthreads();
            }
        }
        __syncthreads();
        // zero the padding row/column of odd N
        if (Ne > N) {
            for (int i = tid; i < Ne; i += T) { G[N * ld + i] = 0.f; G[i * ld + N] = 0.f; }
        }
        __syncthreads();

        // ---- eigenvectors ---------------------------------------------------------
        bool conv = true;
        // bf16 factors (precision 2^-9): stop at ||off|| <= 1e-5 ||diag|| (fp32 rounding
        // leaves ~1e-7 per element, so a much tighter test is never met, and with
        // quadratic convergence the eigenvectors are then far more accurate than the
        // factors are stored); fp32 factors keep the strict test (max_sweeps bounds it)
        const float tol2 = (DT == SEKV_BF16) ? 1e-10f : 1e-12f;
        if (Ne >= 2) conv = jacobi(G, Vm, ld, Ne, a.max_sweeps, rp, rq, rc, rs, red, tol2);
        else if (tid == 0) Vm[0] = 1.f;
        __syncthreads();
        if (!conv && tid == 0) set_status(a.status, SEKV_WARN_NOT_CONVERGED);
        // top-rS by descending eigenvalue (ties: lower index first), over the real N
        for (int i = tid; i < N; i += T) {
            const float li = G[i * ld + i];
            int rank = 0;
            for (int j = 0; j < N; ++j) {
                const float lj = G[j * ld + j];
                rank += (lj > li) || (lj == li && j < i);
            }
            if (rank < rS) sel[rank] = i;
        }
        __syncthreads();

        // ---- factors ----------------------------------------------------------------
        if (rows_form) {
            // A[t][j] = U[t][sel j];  B[j][k] = sum_t U[t][sel j] X[t][k]
            for (int i = tid; i < len * rS; i += T) {
                const int t = i / rS, j = i % rS;
                store1<DT>(fac_row, tile8_index(t, j, r8), Vm[t * ld + sel[j]]);
            }
            for (int i = tid; i < rS * d; i += T) {
                const int j = i / d, k = i % d;
                const int cj = sel[j];
                float acc = 0.f;
                for (int t = 0; t < len; ++t) acc = fmaf(Vm[t * ld + cj], xs(t, k), acc);
                store1<DT>(fac_col, tile8_index(j, k, d), gate ? acc * gate[j] : acc);
            }
        } else {
            // B[j][k] = V[k][sel j];  A[t][j] = sum_k X[t][k] V[k][sel j]
            for (int i = tid; i < rS * d; i += T) {
                const int j = i / d, k = i % d;
                const float v = Vm[k * ld + sel[j]];
                store1<DT>(fac_col, tile8_index(j, k, d), gate ? v * gate[j] : v);
            }
            for (int t0 = 0; t0 < len; t0 += kChunkRows) {
                const int rows = min(kChunkRows, len - t0);
                __syncthreads();
                for (int i = tid; i < rows * d; i += T) {
                    const int r = i / d, c = i % d;
                    xput(r, c, load1<DT>(src, (int64_t)(t0 + r) * d + c));
                }
                __syncthreads();
                for (int i = tid; i < rows * rS; i += T) {
                    const int r = i / rS, j = i % rS;
                    const int cj = sel[j];
                    float acc = 0.f;
                    for (int k = 0; k < d; ++k) acc = fmaf(xs(r, k), Vm[k * ld + cj], acc);
                    store1<DT>(fac_row, tile8_index(t0 + r, j, r8), acc);
                }
            }
        }
        // zero the padding (token rows >= |S|, columns >= rS of A / C; rows >= rS of
        // B / D) so the block is fully defined
        const int len8 = round8(len);
        for (int i = tid; i < len8 * r8; i += T) {
            const int t = i / r8, j = i % r8;
            if (t >= len || j >= rS) store1<DT>(fac_row, tile8_index(t, j, r8), 0.f);
        }
        for (int i = rS * d + tid; i < r8 * d; i += T) store1<DT>(fac_col, tile8_index(i / d, i % d, d), 0.f);
        __syncthreads();
    }
}

template <int DT, int NB>
static size_t basis_smem(int d) {
    const int xrows = NB > kChunkRows ? NB : kChunkRows;
    size_t s = 2 * (size_t)NB * (NB + 1) * 4;              // G, Vm
    s += (DT == SEKV_BF16) ? (size_t)xrows * (d + 8) * 2   // X bf16
                           : (size_t)xrows * (d + 1) * 4;  // X fp32
    s = round_up(s, 16);
    s += 4 * (size_t)(NB / 2) * 4;                         // rp, rq, rc, rs
    s += 64 * 4 + (size_t)NB * 4;                          // red, sel
    return round_up(s, 16);
}

template <int DT, int NB>
static cudaError_t launch_bucket(const BasisArgs& a, const BasisWork& w, int bucket, size_t cap,
                                 cudaStream_t st) {
    const size_t smem = basis_smem<DT, NB>(a.d);
    cudaError_t e = cudaFuncSetAttribute(basis_kernel<DT, NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, basis_kernel<DT, NB>, NB * 4, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    basis_kernel<DT, NB><<<sms * per_sm, NB * 4, smem, st>>>(a, w, bucket, cap);
    return cudaGetLastError();
}

cudaError_t launch_basis(const sekv_build_desc& d, cudaStream_t st) {
    BasisWork w = carve(d);
    const size_t cap = list_cap(d);
    cudaError_t e = cudaMemsetAsync(d.workspace, 0, 256, st);
    if (e != cudaSuccess) return e;
    classify_kernel<<<d.B, 256, 0, st>>>(d.m_count, d.span_beg, d.span_end, d.m_cap, d.d, w, cap);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    BasisArgs a{d.m_count, d.K, d.V, d.span_beg, d.span_end, d.blk_off, d.basis_home, d.dev_status, d.rank_gate,
                d.region_elems,
                d.L, d.l0, d.l1 - d.l0, d.Hkv, d.n, d.d, d.m_cap, d.rank, d.max_sweeps};
    if (d.dtype == SEKV_F32) {
        if ((e = launch_bucket<SEKV_F32, 32>(a, w, 0, cap, st)) != cudaSuccess) return e;
        if ((e = launch_bucket<SEKV_F32, 64>(a, w, 1, cap, st)) != cudaSuccess) return e;
        if (d.d > 64) e = launch_bucket<SEKV_F32, 128>(a, w, 2, cap, st);
    } else {
        if ((e = launch_bucket<SEKV_BF16, 32>(a, w, 0, cap, st)) != cudaSuccess) return e;
        if ((e = launch_bucket<SEKV_BF16, 64>(a, w, 1, cap, st)) != cudaSuccess) return e;
        if (d.d > 64) e = launch_bucket<SEKV_BF16, 128>(a, w, 2, cap, st);
    }
    return e;
}

}  // namespace sekv
