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
//
// Only the top rS of the N eigenpairs are needed, so the symmetric eigenproblem is
// solved the way a selected-eigenvector solver does it rather than by a full
// diagonalisation (whose cost is ~N^3 per sweep over many sweeps):
//   1. Householder tridiagonalisation G = Q T Q^T in shared memory (N - 2
//      reflectors; each step is a symmetric matrix-vector product and a rank-2
//      update of the trailing block);
//   2. the rS largest eigenvalues of T by multisection on Sturm counts (several
//      threads probe one eigenvalue's bracket at once);
//   3. their eigenvectors by inverse iteration on T - lambda I (one thread per
//      eigenvalue, pseudo-random start vectors), then modified Gram-Schmidt twice in
//      descending eigenvalue order, so that vectors of clustered eigenvalues come
//      out orthonormal and span their cluster;
//   4. back-transformation by the reflectors (u = Q z), one warp per vector.
// T is scaled to unit norm before steps 2-3 (eigenvectors do not change).
// The Gram contraction runs on the tensor cores (mma.sync m16n8k16 bf16 -> fp32)
// for bf16 inputs and on the FMA pipes for fp32 inputs.
//
// Problems are bucketed by N (<= 32, <= 64, <= 128) so each bucket gets a
// shared-memory footprint and CTA size that fit it; each bucket is a persistent
// launch that pulls work items from an atomic counter.
#include <cfloat>

#include "sekv_common.cuh"
#include "sekv_internal.h"

namespace sekv {

constexpr int kBuckets = 3;
constexpr int kChunkRows = 32;    // rows of X staged per step when |S| > d
constexpr int kInvIters = 3;      // inverse-iteration steps per eigenvector
constexpr float kBig = 1e20f;     // rescaling threshold of the tridiagonal solves
constexpr float kSmall = 1e-20f;

struct BasisWork {
    int* bucket_count;   // [kBuckets]
    int* work_next;      // [kBuckets]
    int* failures;       // [2]: eigenvectors restarted after a failed solve; vectors lost in Gram-Schmidt
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
    w.failures = reinterpret_cast<int*>(p + 128);
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
    int L, l0, Lr, Hkv, n, d, m_cap, rank;
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
// Householder tridiagonalisation of the symmetric N x N matrix in G (row stride
// ld, full storage). Afterwards dg[0..N-1] holds the diagonal of T, eo[0..N-2] its
// off-diagonal, and reflector k (k = 0 .. N-3), H_k = I - tk[k] v v^T acting on
// coordinates k+1 .. N-1, is stored with v in row k of G at columns k+1 .. N-1
// (v[k+1] = 1), so that G = Q T Q^T with Q = H_0 H_1 ... H_{N-3}.
// Scratch: pv[ld] (the vector p), red[>= 64].
// ---------------------------------------------------------------------------
SEKV_DEV void tridiagonalize(float* G, int ld, int N, float* dg, float* eo, float* tk, float* pv, float* red) {
    const int tid = threadIdx.x, T = blockDim.x, lane = tid & 31, wid = tid >> 5;
    // column c, partition part: the symmetric product splits each column's sum over R parts
    const int R = T / ld >= 1 ? T / ld : 1;
    float* part = red + 64;      // [R][ld] partial column sums (caller sized)
    for (int k = 0; k + 2 < N; ++k) {
        const int m = N - k - 1;              // trailing block: coordinates k+1 .. N-1
        float* row = G + (size_t)k * ld;
        // (a) reflector of x = row k, columns k+1 .. N-1 (warp 0)
        if (wid == 0) {
            float s = 0.f;
            for (int i = k + 2 + lane; i < N; i += 32) s = fmaf(row[i], row[i], s);
            s = warp_sum(s);
            const float alpha = row[k + 1];
            float tau = 0.f, beta = alpha, scl = 0.f;
            if (s > 0.f) {
                const float nrm = sqrtf(fmaf(alpha, alpha, s));
                beta = alpha >= 0.f ? -nrm : nrm;
                tau = (beta - alpha) / beta;
                scl = 1.f / (alpha - beta);
            }
            for (int i = k + 2 + lane; i < N; i += 32) row[i] *= scl;   // tau = 0: v = e1, tail unused
            if (lane == 0) {
                row[k + 1] = 1.f;
                dg[k] = row[k];
                eo[k] = beta;
                tk[k] = tau;
            }
        }
        __syncthreads();
        const float tau = tk[k];
        if (tau != 0.f) {
            // (b) p = tau A v over the trailing block (A symmetric: column sums, conflict-free rows)
            {
                const int c = tid % ld, pr = tid / ld;
                if (pr < R && c < m) {
                    const int i = k + 1 + c;
                    const int per = (m + R - 1) / R;
                    const int j0 = pr * per, j1 = min(m, j0 + per);
                    float acc = 0.f;
                    for (int j = j0; j < j1; ++j) acc = fmaf(G[(size_t)(k + 1 + j) * ld + i], row[k + 1 + j], acc);
                    part[pr * ld + c] = acc;
                }
            }
            __syncthreads();
            // (c) p, and p . v
            float dot = 0.f;
            for (int c = tid; c < m; c += T) {
                float p = 0.f;
                for (int r = 0; r < R; ++r) p += part[r * ld + c];
                p *= tau;
                pv[c] = p;
                dot = fmaf(p, row[k + 1 + c], dot);
            }
            dot = warp_sum(dot);
            if (lane == 0) red[wid] = dot;
            __syncthreads();
            float pvd = 0.f;
            for (int w = 0; w < (T >> 5); ++w) pvd += red[w];
            const float Kc = 0.5f * tau * pvd;
            // (d) A -= v w^T + w v^T with w = p - Kc v
            {
                const int c = tid % ld, r0 = tid / ld;
                if (c < m) {
                    const float vj = row[k + 1 + c];
                    const float wj = pv[c] - Kc * vj;
                    for (int r = r0; r < m; r += R) {
                        const float vi = row[k + 1 + r];
                        const float wi = pv[r] - Kc * vi;
                        float* g = G + (size_t)(k + 1 + r) * ld + (k + 1 + c);
                        *g = fmaf(-vi, wj, fmaf(-wi, vj, *g));
                    }
                }
            }
        }
        __syncthreads();
    }
    if (tid == 0) {
        if (N >= 2) {
            dg[N - 2] = G[(size_t)(N - 2) * ld + N - 2];
            eo[N - 2] = G[(size_t)(N - 2) * ld + N - 1];
        }
        dg[N - 1] = G[(size_t)(N - 1) * ld + N - 1];
    }
    __syncthreads();
}

// number of eigenvalues of T (diagonal dg, squared off-diagonal e2) below x
// (Sturm count of the LDL^T pivots; a pivot smaller than pivmin counts as -pivmin)
SEKV_DEV int sturm_count(const float* dg, const float* e2, int N, float x, float pivmin) {
    float q = dg[0] - x;
    if (fabsf(q) < pivmin) q = -pivmin;
    int c = q < 0.f;
    for (int i = 1; i < N; ++i) {
        q = (dg[i] - x) - __fdividef(e2[i - 1], q);
        if (fabsf(q) < pivmin) q = -pivmin;
        c += q < 0.f;
    }
    return c;
}

// deterministic start vectors for inverse iteration: a hash of (vector, row) in [-1, 1)
SEKV_DEV float start_entry(int j, int i) {
    uint32_t h = (uint32_t)(j * 0x9E3779B1u) ^ (uint32_t)(i * 0x85EBCA77u) ^ 0x27D4EB2Fu;
    h ^= h >> 15; h *= 0x2C1B3C6Du; h ^= h >> 12; h *= 0x297A2D39u; h ^= h >> 15;
    return (float)(h >> 8) * (2.f / 16777216.f) - 1.f;
}

// ---------------------------------------------------------------------------
// The rS largest eigenpairs of the tridiagonal T (dg, eo; N x N), eigenvectors
// written to Z[j][0..N-1] (row stride ldz) in descending eigenvalue order, j < rS.
// Scratch: Dw[rS][ldz] (pivots of the solves), e2[N], lam[rS], red[>= 64].
// Returns false (uniform over the CTA) when a solve produced no usable vector.
// ---------------------------------------------------------------------------
SEKV_DEV bool top_eigvecs_tridiag(float* dg, float* eo, float* e2, int N, int rS, float* Z, int ldz, float* Dw,
                                  float* lam, float* red, int* lost, int* failures) {
    const int tid = threadIdx.x, T = blockDim.x, lane = tid & 31, wid = tid >> 5, nw = T >> 5;
    // Gershgorin bound of ||T||; scale T to unit norm
    float tn = 0.f;
    for (int i = tid; i < N; i += T) {
        const float el = i > 0 ? fabsf(eo[i - 1]) : 0.f, er = i + 1 < N ? fabsf(eo[i]) : 0.f;
        tn = fmaxf(tn, fabsf(dg[i]) + el + er);
    }
    tn = warp_max(tn);
    if (lane == 0) red[wid] = tn;
    __syncthreads();
    tn = 0.f;
    for (int w = 0; w < nw; ++w) tn = fmaxf(tn, red[w]);
    __syncthreads();
    if (!(tn > 0.f) || !isfinite(tn)) {
        // T = 0: every vector is an eigenvector; take the coordinate axes
        for (int i = tid; i < rS * ldz; i += T) Z[i] = ((i % ldz) == (i / ldz)) ? 1.f : 0.f;
        __syncthreads();
        return isfinite(tn);
    }
    const float inv = 1.f / tn;
    for (int i = tid; i < N; i += T) {
        dg[i] *= inv;
        if (i + 1 < N) {
            eo[i] *= inv;
            e2[i] = eo[i] * eo[i];
        }
    }
    __syncthreads();
    // ---- multisection: S threads per eigenvalue (S a power of two, <= 8)
    const float pivmin = 1e-30f;
    int S = 8;
    while (S > 1 && S * rS > T) S >>= 1;
    const int groups = T / S;
    const int g = tid / S, s = tid % S;
    const float tol = 4.f * FLT_EPSILON;
    for (int j0 = 0; j0 < rS; j0 += groups) {
        const int j = j0 + g;
        const int k = N - 1 - (j < rS ? j : rS - 1);    // ascending index of the j-th largest
        float lo = -1.f - 2.f * tol, hi = 1.f + 2.f * tol;    // contains every eigenvalue of the scaled T
        // every lane of the warp runs the same iterations (the shuffles below need
        // them all); a finished bracket only keeps shrinking
        for (int it = 0; it < 64 && __any_sync(0xffffffffu, hi - lo > tol); ++it) {
            const float x = lo + (float)(s + 1) * ((hi - lo) / (float)(S + 1));
            const int c = sturm_count(dg, e2, N, x, pivmin);
            // the largest probe with count <= k is the new lo, the smallest with count > k the new hi
            float nlo = (c <= k) ? x : -INFINITY, nhi = (c > k) ? x : INFINITY;
            for (int o = 1; o < S; o <<= 1) {
                nlo = fmaxf(nlo, __shfl_xor_sync(0xffffffffu, nlo, o));
                nhi = fminf(nhi, __shfl_xor_sync(0xffffffffu, nhi, o));
            }
            lo = fmaxf(lo, nlo);
            hi = fminf(hi, nhi);
        }
        if (j < rS && s == 0) lam[j] = 0.5f * (lo + hi);
    }
    __syncthreads();
    // ---- block inverse iteration: every step solves (T - lam_j I) x_j = z_j for all j
    // in parallel (one thread per eigenvalue, LDL^T recurrence; a pivot below eps,
    // with |T| = 1, is set to +-eps, i.e. the shift moves by at most eps, which
    // inverse iteration tolerates) and then orthonormalises the block by modified
    // Gram-Schmidt in descending eigenvalue order. The orthonormalisation inside the
    // iteration makes the vectors of eigenvalues closer than the bisection
    // tolerance converge to different directions of their cluster instead of all to
    // the same one.
    // modified Gram-Schmidt over the block: vector j is final after step j - 1; warp w
    // updates vectors j + 1 + w, j + 1 + w + nw, ...; a vector that vanishes is flagged
    auto mgs = [&]() {
        for (int j = 0; j < rS; ++j) {
            const float* zj = Z + (size_t)j * ldz;
            if (j == 0 && wid == 0) {                  // vector 0 only needs normalising
                float nn = 0.f;
                for (int i = lane; i < N; i += 32) nn = fmaf(zj[i], zj[i], nn);
                nn = warp_sum(nn);
                const float r = nn > 1e-30f ? rsqrtf(nn) : 0.f;
                if (r == 0.f && lane == 0) {
                    *lost = 1;
                    if (failures) atomicAdd(&failures[1], 1);
                }
                for (int i = lane; i < N; i += 32) Z[i] *= r;
            }
            __syncthreads();
            for (int kv = j + 1 + wid; kv < rS; kv += nw) {
                float* zk = Z + (size_t)kv * ldz;
                float dt = 0.f;
                for (int i = lane; i < N; i += 32) dt = fmaf(zj[i], zk[i], dt);
                dt = warp_sum(dt);
                float nn = 0.f;
                for (int i = lane; i < N; i += 32) {
                    const float v = fmaf(-dt, zj[i], zk[i]);
                    zk[i] = v;
                    nn = fmaf(v, v, nn);
                }
                if (kv == j + 1) {                     // normalise the next vector here
                    nn = warp_sum(nn);
                    const float r = nn > 1e-30f ? rsqrtf(nn) : 0.f;
                    if (r == 0.f && lane == 0) {       // dependent vectors: reported
                        *lost = 1;
                        if (failures) atomicAdd(&failures[1], 1);
                    }
                    for (int i = lane; i < N; i += 32) zk[i] *= r;
                }
            }
        }
        __syncthreads();
    };
    bool good = true;
    if (tid < rS) {
        float* z = Z + (size_t)tid * ldz;
        float nrm = 0.f;
        for (int i = 0; i < N; ++i) {
            z[i] = start_entry(tid, i);
            nrm = fmaf(z[i], z[i], nrm);
        }
        const float r = rsqrtf(nrm);
        for (int i = 0; i < N; ++i) z[i] *= r;
    }
    __syncthreads();
    for (int it = 0; it < kInvIters; ++it) {
        if (tid < rS) {
            const int j = tid;
            float* z = Z + (size_t)j * ldz;
            float* D = Dw + (size_t)j * ldz;
            const float lj = lam[j];
            const float pv = FLT_EPSILON;
            // forward: D_i and y = L^{-1} (rs * z). The unpivoted elimination can grow
            // by up to 1/eps per step; when |y| passes kBig, the partial solution and
            // the multiplier of the remaining right-hand side are scaled down together,
            // which scales the whole system and keeps it exact.
            float rs = 1.f;
            float Dp = dg[0] - lj;
            if (fabsf(Dp) < pv) Dp = Dp < 0.f ? -pv : pv;
            D[0] = Dp;
            float y = z[0];
            for (int i = 1; i < N; ++i) {
                const float l = __fdividef(eo[i - 1], Dp);
                float Dn = (dg[i] - lj) - l * eo[i - 1];
                if (fabsf(Dn) < pv) Dn = Dn < 0.f ? -pv : pv;
                y = fmaf(-l, y, z[i] * rs);
                if (fabsf(y) > kBig) {
                    for (int k = 0; k < i; ++k) z[k] *= kSmall;
                    y *= kSmall;
                    rs *= kSmall;
                }
                z[i] = y;
                D[i] = Dn;
                Dp = Dn;
            }
            // backward: x_i = (y_i - e_i x_{i+1}) / D_i, rescaled the same way (the
            // x found so far and the y still to use)
            float x = __fdividef(z[N - 1], D[N - 1]);
            if (fabsf(x) > kBig) {
                for (int k = 0; k < N - 1; ++k) z[k] *= kSmall;
                x *= kSmall;
            }
            z[N - 1] = x;
            float mx = fabsf(x);
            for (int i = N - 2; i >= 0; --i) {
                x = __fdividef(fmaf(-eo[i], x, z[i]), D[i]);
                if (fabsf(x) > kBig) {
                    for (int k = 0; k < N; ++k)
                        if (k != i) z[k] *= kSmall;
                    x *= kSmall;
                    mx *= kSmall;
                }
                z[i] = x;
                mx = fmaxf(mx, fabsf(x));
            }
            // scale by the largest entry (no overflow in the later norms)
            const float im = mx > 0.f && isfinite(mx) ? 1.f / mx : 0.f;
            bool finite = im > 0.f;
            for (int i = 0; i < N; ++i) {
                z[i] *= im;
                finite = finite && isfinite(z[i]);
            }
            if (!finite) {
                if (failures) atomicAdd(&failures[0], 1);
                for (int i = 0; i < N; ++i) z[i] = start_entry(j + 977, i);     // restart from another vector
                good = false;
            }
        }
        __syncthreads();
        mgs();
    }
    mgs();                                             // a second pass: orthogonal to rounding
    good = __syncthreads_and(good);
    return good && *lost == 0;
}

// u = Q z for the rS vectors in Z (row stride ldz), with the reflectors stored by
// tridiagonalize in G; one warp per vector, no block barrier inside
SEKV_DEV void back_transform(const float* G, int ld, const float* tk, int N, int rS, float* Z, int ldz) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int j = wid; j < rS; j += nw) {
        float* z = Z + (size_t)j * ldz;
        for (int k = N - 3; k >= 0; --k) {
            const float tau = tk[k];
            if (tau == 0.f) continue;
            const float* v = G + (size_t)k * ld;
            float s = 0.f;
            for (int i = k + 1 + lane; i < N; i += 32) s = fmaf(v[i], z[i], s);
            s = warp_sum(s) * tau;
            for (int i = k + 1 + lane; i < N; i += 32) z[i] = fmaf(-s, v[i], z[i]);
            __syncwarp();
        }
    }
    __syncthreads();
}

// threads per CTA of a bucket
template <int NB> struct BasisThreads { static constexpr int value = NB >= 128 ? 256 : (NB >= 64 ? 128 : 64); };

// shared-memory carve-up (bytes), shared by the kernel and its launcher:
//   [ G: NB x NB fp32 | XA | small arrays ]
// XA holds X for the Gram (|S| <= d: up to NB rows; |S| > d: 32-row chunks), then,
// during the eigensolve, the solve pivots at offset 0 and the vectors at z_off. In
// the factor stage X is streamed again in 32-row chunks from the start of G, which
// may run past G into the (dead) pivots but stops before z_off.
struct BasisSmem {
    size_t g, xa, z_off, small, total;
    int ldx, ldz, rsmax, R;
};

template <int DT, int NB>
__host__ __device__ inline BasisSmem basis_smem_layout(int d, int rank) {
    BasisSmem s;
    constexpr int T = BasisThreads<NB>::value;
    const int esz = DT == SEKV_BF16 ? 2 : 4;
    s.rsmax = rank < NB ? rank : NB;
    s.ldx = (DT == SEKV_BF16) ? d + 8 : d + 1;
    s.ldz = NB + 1;
    s.R = T / NB >= 1 ? T / NB : 1;
    const int xrows = NB > kChunkRows ? NB : kChunkRows;
    s.g = (size_t)NB * NB * 4;
    const size_t xbytes = (size_t)xrows * s.ldx * esz;
    const size_t chunk = (size_t)kChunkRows * s.ldx * esz;
    const size_t zbytes = (size_t)s.rsmax * s.ldz * 4;
    const size_t past_g = chunk > s.g ? chunk - s.g : 0;
    s.z_off = round_up(zbytes > past_g ? zbytes : past_g, 16);
    const size_t need = s.z_off + zbytes;
    s.xa = round_up(xbytes > need ? xbytes : need, 16);
    // dg, eo, e2, tk, pv: 5 x NB floats; lam: rsmax; red: 64 + R * NB floats
    s.small = round_up((size_t)(5 * NB + s.rsmax + 64 + s.R * NB) * 4, 16);
    s.total = s.g + s.xa + s.small;
    return s;
}

// Stage rows [0, fill) of a row-padded copy of X in shared memory (row stride ldx
// elements): rows < rows come from src (row stride d elements), the rest are zero.
// bf16 rows move as 16-byte vectors (d and ldx are multiples of 8, rows of X are
// 16-byte aligned); fp32 element by element.
template <int DT>
SEKV_DEV void stage_rows(void* dst, int ldx, const char* src, int d, int rows, int fill) {
    const int tid = threadIdx.x, T = blockDim.x;
    if constexpr (DT == SEKV_BF16) {
        const int vpr = d / 8;                                       // 16-byte vectors per row
        for (int i = tid; i < fill * vpr; i += T) {
            const int r = i / vpr, c = (i % vpr) * 8;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (r < rows) v = *reinterpret_cast<const uint4*>(src + ((int64_t)r * d + c) * 2);
            *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(dst) + (size_t)r * ldx + c) = v;
        }
    } else {
        for (int i = tid; i < fill * d; i += T) {
            const int r = i / d, c = i % d;
            reinterpret_cast<float*>(dst)[(size_t)r * ldx + c] = r < rows ? load1<DT>(src, (int64_t)r * d + c) : 0.f;
        }
    }
}

template <int DT, int NB>
__global__ void __launch_bounds__(BasisThreads<NB>::value, NB >= 128 ? 2 : 4)
basis_kernel(BasisArgs a, BasisWork w, int bucket, size_t cap) {
    using E = Elt<DT>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int tid = threadIdx.x, T = blockDim.x;
    const int d = a.d;
    constexpr int ld = NB;                          // fp32 G row stride
    const BasisSmem L = basis_smem_layout<DT, NB>(d, a.rank);
    const int ldx = L.ldx, ldz = L.ldz;
    float* G = reinterpret_cast<float*>(smem_raw);
    unsigned char* xa = smem_raw + L.g;
    float* X = reinterpret_cast<float*>(xa);
    __nv_bfloat16* Xb = reinterpret_cast<__nv_bfloat16*>(xa);
    float* Dw = reinterpret_cast<float*>(xa);                  // solve pivots
    float* Z = reinterpret_cast<float*>(xa + L.z_off);         // eigenvectors
    float* dg = reinterpret_cast<float*>(smem_raw + L.g + L.xa);
    float* eo = dg + NB;
    float* e2 = eo + NB;
    float* tk = e2 + NB;
    float* pv = tk + NB;
    float* lam = pv + NB;
    float* red = lam + L.rsmax;                    // 64 + R * NB floats
    __shared__ int item_s, lost_s;

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
            stage_rows<DT>(xa, ldx, src, d, len, Mp);
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
                stage_rows<DT>(xa, ldx, src + (int64_t)t0 * d * E::bytes, d, rows, kChunkRows);
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

        // ---- top-rS eigenvectors of G ------------------------------------------
        if (tid == 0) lost_s = 0;
        tridiagonalize(G, ld, N, dg, eo, tk, pv, red);
        const bool good = top_eigvecs_tridiag(dg, eo, e2, N, rS, Z, ldz, Dw, lam, red, &lost_s, w.failures);
        if (!good && tid == 0) set_status(a.status, SEKV_WARN_NOT_CONVERGED);
        back_transform(G, ld, tk, N, rS, Z, ldz);

        // ---- factors ----------------------------------------------------------------
        // X is streamed again in chunks of 32 rows into G's space (G is dead now)
        __nv_bfloat16* Xc = reinterpret_cast<__nv_bfloat16*>(G);
        float* Xf = G;
        auto xcs = [&](int r, int c) -> float {
            return (DT == SEKV_BF16) ? __bfloat162float(Xc[r * ldx + c]) : Xf[r * ldx + c];
        };
        if (rows_form) {
            // A[t][j] = U[t][j];  B[j][k] = sum_t U[t][j] X[t][k]
            for (int i = tid; i < len * rS; i += T) {
                const int t = i / rS, j = i % rS;
                store1<DT>(fac_row, tile8_index(t, j, r8), Z[(size_t)j * ldz + t]);
            }
            // each thread owns outputs (j, k) = i, i + T, ... of the rS x d product, in
            // blocks of kMaxOut (X is streamed once per block)
            constexpr int kMaxOut = 16;
            const int nout = (rS * d + T - 1) / T;
            for (int q0 = 0; q0 < nout; q0 += kMaxOut) {
                float acc[kMaxOut];
#pragma unroll
                for (int q = 0; q < kMaxOut; ++q) acc[q] = 0.f;
                for (int t0 = 0; t0 < len; t0 += kChunkRows) {
                    const int rows = min(kChunkRows, len - t0);
                    __syncthreads();
                    stage_rows<DT>(G, ldx, src + (int64_t)t0 * d * E::bytes, d, rows, rows);
                    __syncthreads();
#pragma unroll
                    for (int q = 0; q < kMaxOut; ++q) {
                        const int i = tid + (q0 + q) * T;
                        if (q0 + q < nout && i < rS * d) {
                            const int j = i / d, k = i % d;
                            const float* zj = Z + (size_t)j * ldz + t0;
                            float s = acc[q];
                            for (int t = 0; t < rows; ++t) s = fmaf(zj[t], xcs(t, k), s);
                            acc[q] = s;
                        }
                    }
                }
#pragma unroll
                for (int q = 0; q < kMaxOut; ++q) {
                    const int i = tid + (q0 + q) * T;
                    if (q0 + q < nout && i < rS * d) {
                        const int j = i / d, k = i % d;
                        store1<DT>(fac_col, tile8_index(j, k, d), gate ? acc[q] * gate[j] : acc[q]);
                    }
                }
            }
        } else {
            // B[j][k] = V[k][j];  A[t][j] = sum_k X[t][k] V[k][j]
            for (int i = tid; i < rS * d; i += T) {
                const int j = i / d, k = i % d;
                const float v = Z[(size_t)j * ldz + k];
                store1<DT>(fac_col, tile8_index(j, k, d), gate ? v * gate[j] : v);
            }
            for (int t0 = 0; t0 < len; t0 += kChunkRows) {
                const int rows = min(kChunkRows, len - t0);
                __syncthreads();
                stage_rows<DT>(G, ldx, src + (int64_t)t0 * d * E::bytes, d, rows, rows);
                __syncthreads();
                for (int i = tid; i < rows * rS; i += T) {
                    const int r = i / rS, j = i % rS;
                    const float* zj = Z + (size_t)j * ldz;
                    float acc = 0.f;
                    for (int k = 0; k < d; ++k) acc = fmaf(xcs(r, k), zj[k], acc);
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
static cudaError_t launch_bucket(const BasisArgs& a, const BasisWork& w, int bucket, size_t cap,
                                 cudaStream_t st) {
    constexpr int T = BasisThreads<NB>::value;
    const BasisSmem L = basis_smem_layout<DT, NB>(a.d, a.rank);
    if (L.total > 227 * 1024) return cudaErrorInvalidConfiguration;
    cudaError_t e = cudaFuncSetAttribute(basis_kernel<DT, NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L.total);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, basis_kernel<DT, NB>, T, L.total);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    basis_kernel<DT, NB><<<sms * per_sm, T, L.total, st>>>(a, w, bucket, cap);
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
                d.L, d.l0, d.l1 - d.l0, d.Hkv, d.n, d.d, d.m_cap, d.rank};
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
