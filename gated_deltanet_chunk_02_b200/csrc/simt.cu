// simt.cu — CUDA-core kernels of libgdn.
//
// * the float32 path of every per-chunk step (A, the Neumann chain with mask
//   and residual, WY, and their fusion), one CTA of 256 threads per chunk, all
//   operands in shared memory, k <= 128;
// * the exact forward substitution (every k), the comparison point of
//   "When Good Enough Is Optimal" (Énoncé du Problème);
// * the INT8 scheme (k = 64) as an integer CUDA-core kernel.
//
// Thread (ty, tx) = (tid / 16, tid % 16) of a 256-thread CTA owns the rows
// ty + 16*ii and the columns tx + 16*jj of every k x k (or k x d) product,
// so each warp reads two rows of the left operand (broadcast) and sixteen
// consecutive columns of the right one (conflict-free with a padded pitch).
#include "common.cuh"
#include "kernels.h"

namespace gdn {

constexpr int kSimtThreads = 256;
constexpr int kD = 128;           // head dim d_k = d_v
constexpr int kLdK = kD + 1;      // padded pitch of a k x d tile in shared memory

// C += X * Y over L, X row pitch ldx, Y row pitch ldy.
template <int RM, int RN>
__device__ __forceinline__ void mm_nn(const float* __restrict__ X, int ldx,
                                      const float* __restrict__ Y, int ldy, int L,
                                      float (&c)[RM][RN], int ty, int tx) {
#pragma unroll 4
    for (int l = 0; l < L; ++l) {
        float a[RM], b[RN];
#pragma unroll
        for (int ii = 0; ii < RM; ++ii) a[ii] = X[(ty + 16 * ii) * ldx + l];
#pragma unroll
        for (int jj = 0; jj < RN; ++jj) b[jj] = Y[l * ldy + tx + 16 * jj];
#pragma unroll
        for (int ii = 0; ii < RM; ++ii)
#pragma unroll
            for (int jj = 0; jj < RN; ++jj) c[ii][jj] = fmaf(a[ii], b[jj], c[ii][jj]);
    }
}

// C += X * Z^T over L (rows of Z indexed by the output column).
template <int RM, int RN>
__device__ __forceinline__ void mm_nt(const float* __restrict__ X, int ldx,
                                      const float* __restrict__ Z, int ldz, int L,
                                      float (&c)[RM][RN], int ty, int tx) {
#pragma unroll 4
    for (int l = 0; l < L; ++l) {
        float a[RM], b[RN];
#pragma unroll
        for (int ii = 0; ii < RM; ++ii) a[ii] = X[(ty + 16 * ii) * ldx + l];
#pragma unroll
        for (int jj = 0; jj < RN; ++jj) b[jj] = Z[(tx + 16 * jj) * ldz + l];
#pragma unroll
        for (int ii = 0; ii < RM; ++ii)
#pragma unroll
            for (int jj = 0; jj < RN; ++jj) c[ii][jj] = fmaf(a[ii], b[jj], c[ii][jj]);
    }
}

template <int RM, int RN>
__device__ __forceinline__ void zero(float (&c)[RM][RN]) {
#pragma unroll
    for (int ii = 0; ii < RM; ++ii)
#pragma unroll
        for (int jj = 0; jj < RN; ++jj) c[ii][jj] = 0.f;
}

// Load one k x d tile (any element type) into shared memory as float32.
template <int K, typename TI>
__device__ __forceinline__ void load_tile_kd(float* __restrict__ dst, const TI* __restrict__ src,
                                             const float* __restrict__ scale) {
    for (int e = threadIdx.x; e < K * kD; e += kSimtThreads) {
        int r = e / kD, c = e % kD;
        float v = ld_elem(src, e);
        dst[r * kLdK + c] = scale ? v * scale[r] : v;
    }
}

// A_ij = -beta_i G_ij exp(g_i - g_j) for i > j (else 0) into X (pitch K+1),
// from K (already in shared memory, pitch kLdK).
template <int K>
__device__ __forceinline__ void build_A_tile(const float* Ks, const float* sb, const float* sg,
                                             float* X, int ty, int tx) {
    constexpr int R = K / 16;
    float G[R][R];
    zero(G);
    mm_nt<R, R>(Ks, kLdK, Ks, kLdK, kD, G, ty, tx);
#pragma unroll
    for (int ii = 0; ii < R; ++ii)
#pragma unroll
        for (int jj = 0; jj < R; ++jj) {
            int i = ty + 16 * ii, j = tx + 16 * jj;
            X[i * (K + 1) + j] = (i > j) ? -sb[i] * G[ii][jj] * expf(sg[i] - sg[j]) : 0.f;
        }
}

// Neumann + mask + residual on one chunk, float32.  On entry X holds A
// (pitch K+1); on exit T0 holds T and X, Y are scratch.  Every step is the
// method's product (Méthodologie §1-§3); the mask multiplies each power as it
// is formed, which equals masking the truncated sum in exact arithmetic.
template <int K>
__device__ void neumann_chain_f32(float* X, float* Y, int N, int mask, int S,
                                  float (&T0)[K / 16][K / 16], int ty, int tx) {
    constexpr int R = K / 16, LD = K + 1;
    float D[R][R];
#pragma unroll
    for (int ii = 0; ii < R; ++ii)
#pragma unroll
        for (int jj = 0; jj < R; ++jj) {
            int i = ty + 16 * ii, j = tx + 16 * jj;
            float a = X[i * LD + j];
            float p = (mask && i - j > N) ? 0.f : a;
            T0[ii][jj] = (i == j ? 1.f : 0.f) + p;
            Y[i * LD + j] = p;
        }
    __syncthreads();
    for (int n = 2; n <= N; ++n) {
        zero(D);
        mm_nn<R, R>(Y, LD, X, LD, K, D, ty, tx);       // P_n = P_{n-1} A
        __syncthreads();
#pragma unroll
        for (int ii = 0; ii < R; ++ii)
#pragma unroll
            for (int jj = 0; jj < R; ++jj) {
                int i = ty + 16 * ii, j = tx + 16 * jj;
                float p = (mask && i - j > N) ? 0.f : D[ii][jj];
                T0[ii][jj] += p;
                Y[i * LD + j] = p;
            }
        __syncthreads();
    }
    if (S <= 0) return;
    // E = I - (I - A) T0 = I - T0 + A T0
#pragma unroll
    for (int ii = 0; ii < R; ++ii)
#pragma unroll
        for (int jj = 0; jj < R; ++jj)
            Y[(ty + 16 * ii) * LD + tx + 16 * jj] = T0[ii][jj];
    __syncthreads();
    zero(D);
    mm_nn<R, R>(X, LD, Y, LD, K, D, ty, tx);             // A T0
    __syncthreads();
    // Q_1 = E; Horner Q_{m+1} = (I + Q_m) E gives Q_S = sum_{s=1}^{S} E^s
#pragma unroll
    for (int ii = 0; ii < R; ++ii)
#pragma unroll
        for (int jj = 0; jj < R; ++jj) {
            int i = ty + 16 * ii, j = tx + 16 * jj;
            float e = (i == j ? 1.f : 0.f) - T0[ii][jj] + D[ii][jj];
            X[i * LD + j] = e;
            Y[i * LD + j] = (S > 1 && i == j ? 1.f : 0.f) + e;
        }
    __syncthreads();
    for (int m = 1; m < S; ++m) {
        zero(D);
        mm_nn<R, R>(Y, LD, X, LD, K, D, ty, tx);
        __syncthreads();
        const bool last = (m == S - 1);
#pragma unroll
        for (int ii = 0; ii < R; ++ii)
#pragma unroll
            for (int jj = 0; jj < R; ++jj) {
                int i = ty + 16 * ii, j = tx + 16 * jj;
                Y[i * LD + j] = (!last && i == j ? 1.f : 0.f) + D[ii][jj];
            }
        __syncthreads();
    }
    // T = T0 (I + Q) = T0 + T0 Q
#pragma unroll
    for (int ii = 0; ii < R; ++ii)
#pragma unroll
        for (int jj = 0; jj < R; ++jj) X[(ty + 16 * ii) * LD + tx + 16 * jj] = T0[ii][jj];
    __syncthreads();
    zero(D);
    mm_nn<R, R>(X, LD, Y, LD, K, D, ty, tx);
#pragma unroll
    for (int ii = 0; ii < R; ++ii)
#pragma unroll
        for (int jj = 0; jj < R; ++jj) T0[ii][jj] += D[ii][jj];
    __syncthreads();
}

// out[i][c] = sum_j X[i][j] * Kd[j][c] (X pitch K+1, Kd pitch kLdK), stored as TO.
template <int K, typename TO>
__device__ __forceinline__ void wy_store(const float* X, const float* Kd, TO* out, int ty, int tx) {
    constexpr int R = K / 16, RD = kD / 16;
    float acc[R][RD];
    zero(acc);
    mm_nn<R, RD>(X, K + 1, Kd, kLdK, K, acc, ty, tx);
#pragma unroll
    for (int ii = 0; ii < R; ++ii)
#pragma unroll
        for (int jj = 0; jj < RD; ++jj)
            st_elem(out, (int64_t)(ty + 16 * ii) * kD + tx + 16 * jj, acc[ii][jj]);
}

// ------------------------------------------------------------------------- //
// kernels
// ------------------------------------------------------------------------- //
template <int K, typename TI>
__global__ void __launch_bounds__(kSimtThreads)
k_build_A_simt(const TI* __restrict__ Kp, const float* __restrict__ beta,
               const float* __restrict__ g, float* __restrict__ A) {
    extern __shared__ float sm[];
    float* Ks = sm;
    float* X = Ks + K * kLdK;
    float* sb = X + K * (K + 1);
    float* sg = sb + K;
    const int64_t c = blockIdx.x;
    const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
    load_tile_kd<K>(Ks, Kp + c * K * kD, (const float*)nullptr);
    for (int i = threadIdx.x; i < K; i += kSimtThreads) {
        sb[i] = beta[c * K + i];
        sg[i] = g[c * K + i];
    }
    __syncthreads();
    build_A_tile<K>(Ks, sb, sg, X, ty, tx);
    __syncthreads();
    float* Ac = A + c * K * K;
    for (int e = threadIdx.x; e < K * K; e += kSimtThreads) Ac[e] = X[(e / K) * (K + 1) + e % K];
}

// k = 256: K K^T by 128 x 128 quadrants (upper quadrant is zero), A written
// straight to global memory.
template <typename TI>
__global__ void __launch_bounds__(kSimtThreads)
k_build_A_simt256(const TI* __restrict__ Kp, const float* __restrict__ beta,
                  const float* __restrict__ g, float* __restrict__ A) {
    constexpr int K = 256, R = 8;
    extern __shared__ float sm[];
    float* Ks = sm;                       // [256][129]
    float* sb = Ks + K * kLdK;
    float* sg = sb + K;
    const int64_t c = blockIdx.x;
    const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
    load_tile_kd<K>(Ks, Kp + c * K * kD, (const float*)nullptr);
    for (int i = threadIdx.x; i < K; i += kSimtThreads) {
        sb[i] = beta[c * K + i];
        sg[i] = g[c * K + i];
    }
    __syncthreads();
    float* Ac = A + c * K * K;
    for (int q = 0; q < 4; ++q) {
        const int qi = q >> 1, qj = q & 1;
        if (qj > qi) {
            for (int ii = 0; ii < R; ++ii)
                for (int jj = 0; jj < R; ++jj)
                    Ac[(128 * qi + ty + 16 * ii) * K + 128 * qj + tx + 16 * jj] = 0.f;
            continue;
        }
        float G[R][R];
        zero(G);
        mm_nt<R, R>(Ks + 128 * qi * kLdK, kLdK, Ks + 128 * qj * kLdK, kLdK, kD, G, ty, tx);
#pragma unroll
        for (int ii = 0; ii < R; ++ii)
#pragma unroll
            for (int jj = 0; jj < R; ++jj) {
                const int i = 128 * qi + ty + 16 * ii, j = 128 * qj + tx + 16 * jj;
                Ac[i * K + j] = (i > j) ? -sb[i] * G[ii][jj] * expf(sg[i] - sg[j]) : 0.f;
            }
    }
}

template <int K>
__global__ void __launch_bounds__(kSimtThreads)
k_neumann_simt(const float* __restrict__ A, float* __restrict__ T, int N, int mask, int S) {
    extern __shared__ float sm[];
    float* X = sm;
    float* Y = X + K * (K + 1);
    const int64_t c = blockIdx.x;
    const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
    const float* Ac = A + c * K * K;
    for (int e = threadIdx.x; e < K * K; e += kSimtThreads) X[(e / K) * (K + 1) + e % K] = Ac[e];
    __syncthreads();
    float T0[K / 16][K / 16];
    neumann_chain_f32<K>(X, Y, N, mask, S, T0, ty, tx);
    float* Tc = T + c * K * K;
#pragma unroll
    for (int ii = 0; ii < K / 16; ++ii)
#pragma unroll
        for (int jj = 0; jj < K / 16; ++jj) Tc[(ty + 16 * ii) * K + tx + 16 * jj] = T0[ii][jj];
}

template <int K, typename TI>
__global__ void __launch_bounds__(kSimtThreads)
k_wy_simt(const float* __restrict__ T, const TI* __restrict__ Kp, const TI* __restrict__ Vp,
          const float* __restrict__ beta, const float* __restrict__ g,
          TI* __restrict__ W, TI* __restrict__ U) {
    extern __shared__ float sm[];
    float* Ks = sm;
    float* X = Ks + K * kLdK;
    float* sb = X + K * (K + 1);
    float* sw = sb + K;
    const int64_t c = blockIdx.x;
    const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
    for (int i = threadIdx.x; i < K; i += kSimtThreads) {
        float b = beta[c * K + i];
        sb[i] = b;
        sw[i] = g ? b * expf(g[c * K + i]) : b;
    }
    const float* Tc = T + c * K * K;
    for (int e = threadIdx.x; e < K * K; e += kSimtThreads) X[(e / K) * (K + 1) + e % K] = Tc[e];
    __syncthreads();
    load_tile_kd<K>(Ks, Kp + c * K * kD, sw);
    __syncthreads();
    wy_store<K>(X, Ks, W + c * K * kD, ty, tx);
    __syncthreads();
    load_tile_kd<K>(Ks, Vp + c * K * kD, sb);
    __syncthreads();
    wy_store<K>(X, Ks, U + c * K * kD, ty, tx);
}

template <int K, typename TI>
__global__ void __launch_bounds__(kSimtThreads)
k_fused_simt(const TI* __restrict__ Kp, const TI* __restrict__ Vp, const float* __restrict__ beta,
             const float* __restrict__ g, int N, int mask, int S, int gated,
             TI* __restrict__ W, TI* __restrict__ U, float* __restrict__ Tout) {
    extern __shared__ float sm[];
    float* Ks = sm;
    float* X = Ks + K * kLdK;
    float* Y = X + K * (K + 1);
    float* sb = Y + K * (K + 1);
    float* sg = sb + K;
    float* sw = sg + K;
    const int64_t c = blockIdx.x;
    const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
    load_tile_kd<K>(Ks, Kp + c * K * kD, (const float*)nullptr);
    for (int i = threadIdx.x; i < K; i += kSimtThreads) {
        sb[i] = beta[c * K + i];
        sg[i] = g[c * K + i];
    }
    __syncthreads();
    build_A_tile<K>(Ks, sb, sg, X, ty, tx);
    __syncthreads();
    float T0[K / 16][K / 16];
    neumann_chain_f32<K>(X, Y, N, mask, S, T0, ty, tx);
#pragma unroll
    for (int ii = 0; ii < K / 16; ++ii)
#pragma unroll
        for (int jj = 0; jj < K / 16; ++jj) {
            int i = ty + 16 * ii, j = tx + 16 * jj;
            X[i * (K + 1) + j] = T0[ii][jj];
            if (Tout) Tout[c * K * K + i * K + j] = T0[ii][jj];
        }
    for (int i = threadIdx.x; i < K; i += kSimtThreads)
        sw[i] = gated ? sb[i] * expf(sg[i]) : sb[i];
    __syncthreads();
    // W = T diag(w) K: fold w into the rows of K
    for (int e = threadIdx.x; e < K * kD; e += kSimtThreads) Ks[(e / kD) * kLdK + e % kD] *= sw[e / kD];
    __syncthreads();
    wy_store<K>(X, Ks, W + c * K * kD, ty, tx);
    __syncthreads();
    load_tile_kd<K>(Ks, Vp + c * K * kD, sb);
    __syncthreads();
    wy_store<K>(X, Ks, U + c * K * kD, ty, tx);
}

// Exact forward substitution: T = (I - A)^{-1}, row i of T = e_i + sum_{l<i} A_il T_l.
// Each thread owns one column j of T (columns are independent solves) and
// sweeps the rows in blocks of 8; the A entries of a row block are staged
// transposed in shared memory so that one 16-byte broadcast read feeds four
// rows.  Grid: (chunk, column block of CB = min(K, 128) columns).
template <int K>
__global__ void __launch_bounds__(128)
k_fwdsub(const float* __restrict__ A, float* __restrict__ T) {
    constexpr int CB = K < 128 ? K : 128;
    extern __shared__ float sm[];
    const int64_t c = blockIdx.x;
    const int c0 = blockIdx.y * CB;
    const int tid = threadIdx.x;
    const int j = c0 + tid;
    const int L = K - c0;                    // rows/cols at or after c0
    float* xs = sm;                          // [L][CB] solved entries of the owned columns
    float* At = xs + L * CB;                 // [L][8] A[i0 + r][c0 + l] staged transposed
    const float* Ac = A + c * K * K;
    float* Tc = T + c * K * K;
    if (tid < CB) {
        for (int i = 0; i < c0; ++i) Tc[i * K + j] = 0.f;
    }
    for (int i0 = c0; i0 < K; i0 += 8) {
        const int nl = i0 + 8 - c0;          // columns c0 .. i0+7 of the 8 rows
        __syncthreads();
        for (int e = tid; e < 8 * nl; e += CB) {
            int r = e / nl, l = e % nl;
            At[l * 8 + r] = Ac[(i0 + r) * K + c0 + l];
        }
        __syncthreads();
        if (tid < CB) {
            float acc[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) acc[r] = 0.f;
            for (int l = 0; l < i0 - c0; ++l) {
                const float x = xs[l * CB + tid];
                const float4 a0 = *reinterpret_cast<const float4*>(At + l * 8);
                const float4 a1 = *reinterpret_cast<const float4*>(At + l * 8 + 4);
                acc[0] = fmaf(a0.x, x, acc[0]);
                acc[1] = fmaf(a0.y, x, acc[1]);
                acc[2] = fmaf(a0.z, x, acc[2]);
                acc[3] = fmaf(a0.w, x, acc[3]);
                acc[4] = fmaf(a1.x, x, acc[4]);
                acc[5] = fmaf(a1.y, x, acc[5]);
                acc[6] = fmaf(a1.z, x, acc[6]);
                acc[7] = fmaf(a1.w, x, acc[7]);
            }
            float xr[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int i = i0 + r;
                float x = acc[r];
#pragma unroll
                for (int rp = 0; rp < r; ++rp) x = fmaf(At[(i0 - c0 + rp) * 8 + r], xr[rp], x);
                x += (i == j) ? 1.f : 0.f;
                xr[r] = x;
                xs[(i - c0) * CB + tid] = x;
                Tc[i * K + j] = x;
            }
        }
    }
}

// Forward substitution for k <= 64: one warp per chunk.  The chunk's A is
// copied to shared memory in one coalesced pass (cp.async); lane l owns the
// columns j = l + 32c of T and keeps them in registers; the row sweep
// T[i][j] = [i == j] + sum_{l < i} A[i][l] T[l][j] reads each row of A as
// float4 broadcasts (every lane needs the same A[i][l]).  Column group c is
// zero above row 32c, so its sweep starts there.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}

constexpr int kFwdWarps = 4;                     // chunks per CTA (one per warp)

template <int K>
__global__ void __launch_bounds__(32 * kFwdWarps)
k_fwdsub_warp(const float* __restrict__ A, float* __restrict__ T, int64_t nc) {
    constexpr int NC = K / 32;                   // column groups per lane
    extern __shared__ __align__(16) float smf[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* sA = smf + warp * K * K;
    const int64_t stride = (int64_t)gridDim.x * kFwdWarps;
    for (int64_t c = (int64_t)blockIdx.x * kFwdWarps + warp; c < nc; c += stride) {
        const float* Ac = A + c * K * K;
        __syncwarp();                            // the previous chunk's reads of sA are done
#pragma unroll
        for (int q = 0; q < K * K / 128; ++q) {
            const int e = (q * 32 + lane) * 4;
            cp_async16(sA + e, Ac + e);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncwarp();
        float x[NC][K];
#pragma unroll
        for (int cc = 0; cc < NC; ++cc) {
            const int cb = 32 * cc;
            const int j = cb + lane;
#pragma unroll
            for (int i = cb; i < K; ++i) {
                const float* ar = sA + i * K;
                float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
                for (int l = cb; l + 4 <= i; l += 4) {
                    const float4 a = *reinterpret_cast<const float4*>(ar + l);
                    s0 = fmaf(a.x, x[cc][l], s0);
                    s1 = fmaf(a.y, x[cc][l + 1], s1);
                    s2 = fmaf(a.z, x[cc][l + 2], s2);
                    s3 = fmaf(a.w, x[cc][l + 3], s3);
                }
                const int l0 = cb + ((i - cb) & ~3);
                if (l0 < i) {
                    const float4 a = *reinterpret_cast<const float4*>(ar + l0);
                    s0 = fmaf(a.x, x[cc][l0], s0);
                    if (l0 + 1 < i) s1 = fmaf(a.y, x[cc][l0 + 1], s1);
                    if (l0 + 2 < i) s2 = fmaf(a.z, x[cc][l0 + 2], s2);
                }
                x[cc][i] = (i == j ? 1.f : 0.f) + ((s0 + s1) + (s2 + s3));
            }
        }
        float* Tc = T + c * K * K;
#pragma unroll
        for (int cc = 0; cc < NC; ++cc)
#pragma unroll
            for (int i = 0; i < K; ++i) Tc[i * K + 32 * cc + lane] = i < 32 * cc ? 0.f : x[cc][i];
    }
}

// Forward substitution for k = 128 by 64 x 64 blocks, exact in exact arithmetic:
// T00 = (I - A00)^-1 and T11 = (I - A11)^-1 by the row sweep above (one warp
// per 32-column group), then T10 = T11 (A10 T00) with both products on the
// CUDA cores in fp32.  One chunk per 128-thread CTA at a time.
template <int CB>
__device__ __forceinline__ void fwd_sweep64(const float* sA, int pitch, int lane, float* sT,
                                            float* Tg, int tpitch) {
    // rows of the 64 x 64 block at sA (row pitch `pitch`), columns CB + lane
    const int j = CB + lane;
    float x[64];
#pragma unroll
    for (int i = CB; i < 64; ++i) {
        const float* ar = sA + i * pitch;
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
        for (int l = CB; l + 4 <= i; l += 4) {
            const float4 a = *reinterpret_cast<const float4*>(ar + l);
            s0 = fmaf(a.x, x[l], s0);
            s1 = fmaf(a.y, x[l + 1], s1);
            s2 = fmaf(a.z, x[l + 2], s2);
            s3 = fmaf(a.w, x[l + 3], s3);
        }
        const int l0 = CB + ((i - CB) & ~3);
        if (l0 < i) {
            const float4 a = *reinterpret_cast<const float4*>(ar + l0);
            s0 = fmaf(a.x, x[l0], s0);
            if (l0 + 1 < i) s1 = fmaf(a.y, x[l0 + 1], s1);
            if (l0 + 2 < i) s2 = fmaf(a.z, x[l0 + 2], s2);
        }
        x[i] = (i == j ? 1.f : 0.f) + ((s0 + s1) + (s2 + s3));
    }
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        const float v = i < CB ? 0.f : x[i];
        sT[i * 64 + j] = v;
        Tg[(int64_t)i * tpitch + j] = v;
    }
}

// acc[8][4] += P[r0 + rr][l] Q[l][c0 + cc] over l in [l_lo, l_hi), a multiple of
// 4 wide: per 4 values of l, 8 float4 reads of P rows and 4 of Q rows.
template <int PP, int QP>
__device__ __forceinline__ void mm_tile84(const float* P, const float* Q, int r0, int c0, int l_lo,
                                          int l_hi, float (&acc)[8][4]) {
#pragma unroll 1
    for (int l = l_lo; l < l_hi; l += 4) {
        float4 q[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) q[u] = *reinterpret_cast<const float4*>(Q + (l + u) * QP + c0);
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            const float4 pv = *reinterpret_cast<const float4*>(P + (r0 + rr) * PP + l);
            const float pu[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                acc[rr][0] = fmaf(pu[u], q[u].x, acc[rr][0]);
                acc[rr][1] = fmaf(pu[u], q[u].y, acc[rr][1]);
                acc[rr][2] = fmaf(pu[u], q[u].z, acc[rr][2]);
                acc[rr][3] = fmaf(pu[u], q[u].w, acc[rr][3]);
            }
        }
    }
}

// `nc` 128 x 128 diagonal blocks: block c is diagonal block (c % nb) of chunk
// c / nb, rows `pitch` floats apart (k = 128: nb = 1, pitch 128; k = 256: nb = 2,
// pitch 256, the off-diagonal block then comes from k_fwdsub256_off).
template <int PITCH>
__global__ void __launch_bounds__(128)
k_fwdsub128(const float* __restrict__ A, float* __restrict__ T, int64_t nc) {
    constexpr int K = 128, pitch = PITCH, nb = PITCH / 128;
    extern __shared__ __align__(16) float smf[];
    float* sA = smf;                        // [128][128]
    float* sT00 = sA + K * K;               // [64][64]
    float* sT11 = sT00 + 64 * 64;
    float* sX = sT11 + 64 * 64;             // A10 T00
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int64_t c = blockIdx.x; c < nc; c += gridDim.x) {
        const int64_t boff = (c / nb) * (int64_t)pitch * pitch + (c % nb) * ((int64_t)K * pitch + K);
        const float* Ac = A + boff;
        float* Tc = T + boff;
        __syncthreads();                    // the previous chunk is done with shared memory
#pragma unroll
        for (int q = 0; q < K * K / 4 / 128; ++q) {
            const int e = q * 128 + tid;    // float4 index: row e / 32, column 4 (e % 32)
            cp_async16(sA + e * 4, Ac + (int64_t)(e >> 5) * pitch + (e & 31) * 4);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        // the upper-right block of T is zero
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int e = q * 128 + tid;        // 1024 float4 of rows 0..63, columns 64..127
            reinterpret_cast<float4*>(Tc + (int64_t)(e >> 4) * pitch + 64)[e & 15] =
                make_float4(0.f, 0.f, 0.f, 0.f);
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
        switch (warp) {                     // diagonal blocks, 32 columns per warp
            case 0: fwd_sweep64<0>(sA, K, lane, sT00, Tc, pitch); break;
            case 1: fwd_sweep64<32>(sA, K, lane, sT00, Tc, pitch); break;
            case 2: fwd_sweep64<0>(sA + 64 * K + 64, K, lane, sT11, Tc + 64 * pitch + 64, pitch); break;
            default: fwd_sweep64<32>(sA + 64 * K + 64, K, lane, sT11, Tc + 64 * pitch + 64, pitch); break;
        }
        __syncthreads();
        // 8 x 4 register tiles: rows 8 (tid / 16) .., columns 4 (tid % 16) ..
        const int r0 = 8 * (tid >> 4), c0 = 4 * (tid & 15);
        float acc[8][4];
#pragma unroll
        for (int rr = 0; rr < 8; ++rr)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) acc[rr][cc] = 0.f;
        mm_tile84<K, 64>(sA + 64 * K, sT00, r0, c0, c0, 64, acc);   // X = A10 T00 (T00[l][c] = 0, l < c)
#pragma unroll
        for (int rr = 0; rr < 8; ++rr)
            *reinterpret_cast<float4*>(sX + (r0 + rr) * 64 + c0) =
                make_float4(acc[rr][0], acc[rr][1], acc[rr][2], acc[rr][3]);
        __syncthreads();
#pragma unroll
        for (int rr = 0; rr < 8; ++rr)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) acc[rr][cc] = 0.f;
        mm_tile84<64, 64>(sT11, sX, r0, c0, 0, r0 + 8, acc);        // T10 = T11 X (T11[r][l] = 0, l > r)
#pragma unroll
        for (int rr = 0; rr < 8; ++rr)
            *reinterpret_cast<float4*>(Tc + (int64_t)(64 + r0 + rr) * pitch + c0) =
                make_float4(acc[rr][0], acc[rr][1], acc[rr][2], acc[rr][3]);
    }
}

// k = 256 off-diagonal block: with T00, T11 (128 x 128) already in T,
// T10 = T11 (A10 T00) and T01 = 0.  One chunk per 256-thread CTA; thread
// (tr, tc) owns rows 8 tr .., columns 8 tc .. of each 128 x 128 product.
__device__ __forceinline__ void mm128_tile(const float* P, const float* Q, int r0, int c0, int l_lo,
                                           int l_hi, float (&acc)[8][8]) {
#pragma unroll 1
    for (int l = l_lo; l < l_hi; l += 4) {
        float4 qa[4], qb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            qa[u] = *reinterpret_cast<const float4*>(Q + (l + u) * 128 + c0);
            qb[u] = *reinterpret_cast<const float4*>(Q + (l + u) * 128 + c0 + 4);
        }
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            const float4 pv = *reinterpret_cast<const float4*>(P + (r0 + rr) * 128 + l);
            const float pu[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                acc[rr][0] = fmaf(pu[u], qa[u].x, acc[rr][0]);
                acc[rr][1] = fmaf(pu[u], qa[u].y, acc[rr][1]);
                acc[rr][2] = fmaf(pu[u], qa[u].z, acc[rr][2]);
                acc[rr][3] = fmaf(pu[u], qa[u].w, acc[rr][3]);
                acc[rr][4] = fmaf(pu[u], qb[u].x, acc[rr][4]);
                acc[rr][5] = fmaf(pu[u], qb[u].y, acc[rr][5]);
                acc[rr][6] = fmaf(pu[u], qb[u].z, acc[rr][6]);
                acc[rr][7] = fmaf(pu[u], qb[u].w, acc[rr][7]);
            }
        }
    }
}

__global__ void __launch_bounds__(256)
k_fwdsub256_off(const float* __restrict__ A, float* __restrict__ T, int64_t nc) {
    constexpr int K = 256, H = 128;
    extern __shared__ __align__(16) float smf[];
    float* sP = smf;                        // A10, then T11   [128][128]
    float* sQ = sP + H * H;                 // T00             [128][128]
    float* sX = sQ + H * H;                 // A10 T00         [128][128]
    const int tid = threadIdx.x;
    const int r0 = 8 * (tid >> 4), c0 = 8 * (tid & 15);
    auto load_block = [&](float* dst, const float* src) {   // 128 x 128 block, row pitch K
#pragma unroll 4
        for (int q = 0; q < H * H / 4 / 256; ++q) {
            const int e = q * 256 + tid;
            cp_async16(dst + e * 4, src + (int64_t)(e >> 5) * K + (e & 31) * 4);
        }
    };
    for (int64_t c = blockIdx.x; c < nc; c += gridDim.x) {
        const float* Ac = A + c * K * K;
        float* Tc = T + c * K * K;
        __syncthreads();
        load_block(sP, Ac + H * K);                          // A10
        load_block(sQ, Tc);                                  // T00
        asm volatile("cp.async.commit_group;" ::: "memory");
        // T01 = 0
#pragma unroll 4
        for (int q = 0; q < H * H / 4 / 256; ++q) {
            const int e = q * 256 + tid;
            reinterpret_cast<float4*>(Tc + (int64_t)(e >> 5) * K + H)[e & 31] =
                make_float4(0.f, 0.f, 0.f, 0.f);
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
        float acc[8][8];
#pragma unroll
        for (int rr = 0; rr < 8; ++rr)
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) acc[rr][cc] = 0.f;
        mm128_tile(sP, sQ, r0, c0, c0, H, acc);              // X = A10 T00 (T00[l][c] = 0, l < c)
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            float4* xr = reinterpret_cast<float4*>(sX + (r0 + rr) * H + c0);
            xr[0] = make_float4(acc[rr][0], acc[rr][1], acc[rr][2], acc[rr][3]);
            xr[1] = make_float4(acc[rr][4], acc[rr][5], acc[rr][6], acc[rr][7]);
        }
        __syncthreads();                                     // A10 is read: T11 takes its place
        load_block(sP, Tc + H * K + H);                      // T11
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
#pragma unroll
        for (int rr = 0; rr < 8; ++rr)
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) acc[rr][cc] = 0.f;
        mm128_tile(sP, sX, r0, c0, 0, r0 + 8, acc);          // T10 = T11 X (T11[r][l] = 0, l > r)
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            float4* dst = reinterpret_cast<float4*>(Tc + (int64_t)(H + r0 + rr) * K + c0);
            dst[0] = make_float4(acc[rr][0], acc[rr][1], acc[rr][2], acc[rr][3]);
            dst[1] = make_float4(acc[rr][4], acc[rr][5], acc[rr][6], acc[rr][7]);
        }
    }
}

// INT8 truncated Neumann, k = 64 (see gdn_invert_neumann_i8 for the scheme).
__device__ __forceinline__ float block_max_f(float v, float* red) {
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float m = red[0];
    for (int w = 1; w < kSimtThreads / 32; ++w) m = fmaxf(m, red[w]);
    return m;
}
__device__ __forceinline__ int block_max_i(int v, int* red) {
    for (int o = 16; o; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    int m = red[0];
    for (int w = 1; w < kSimtThreads / 32; ++w) m = max(m, red[w]);
    return m;
}
__device__ __forceinline__ int quant_code(float x, float r) {
    float y = rintf(__fmul_rn(x, r));
    y = fminf(fmaxf(y, -127.f), 127.f);
    return (int)y;
}

__global__ void __launch_bounds__(kSimtThreads)
k_neumann_i8_simt(const float* __restrict__ A, float* __restrict__ T, int N, int mask,
                  int8_t* __restrict__ qd, int32_t* __restrict__ accd, float* __restrict__ sd) {
    constexpr int K = 64, R = 4, LD = K + 1;
    __shared__ int q1s[K * LD];
    __shared__ int qps[K * LD];
    __shared__ float redf[8];
    __shared__ int redi[8];
    const int64_t c = blockIdx.x;
    const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
    const float* Ac = A + c * K * K;
    float a[R][R], t[R][R];
    float amax = 0.f;
#pragma unroll
    for (int ii = 0; ii < R; ++ii)
#pragma unroll
        for (int jj = 0; jj < R; ++jj) {
            int i = ty + 16 * ii, j = tx + 16 * jj;
            float v = Ac[i * K + j];
            if (mask && i - j > N) v = 0.f;
            a[ii][jj] = v;
            amax = fmaxf(amax, fabsf(v));
        }
    amax = block_max_f(amax, redf);
    const float r1 = amax > 0.f ? __fdiv_rn(127.f, amax) : 0.f;
    const float s1 = amax > 0.f ? __fdiv_rn(amax, 127.f) : 0.f;
#pragma unroll
    for (int ii = 0; ii < R; ++ii)
#pragma unroll
        for (int jj = 0; jj < R; ++jj) {
            int i = ty + 16 * ii, j = tx + 16 * jj;
            int q = amax > 0.f ? quant_code(a[ii][jj], r1) : 0;
            q1s[i * LD + j] = q;
            qps[i * LD + j] = q;
            t[ii][jj] = __fadd_rn(i == j ? 1.f : 0.f, __fmul_rn(s1, (float)q));
            if (qd) qd[((c * N) * K + i) * K + j] = (int8_t)q;
            if (accd) accd[((c * N) * K + i) * K + j] = 0;
        }
    if (sd && threadIdx.x == 0) sd[c * N] = s1;
    float sprev = s1;
    for (int n = 1; n < N; ++n) {
        __syncthreads();
        int acc[R][R];
#pragma unroll
        for (int ii = 0; ii < R; ++ii)
#pragma unroll
            for (int jj = 0; jj < R; ++jj) acc[ii][jj] = 0;
        for (int l = 0; l < K; ++l) {
            int x[R], y[R];
#pragma unroll
            for (int ii = 0; ii < R; ++ii) x[ii] = qps[(ty + 16 * ii) * LD + l];
#pragma unroll
            for (int jj = 0; jj < R; ++jj) y[jj] = q1s[l * LD + tx + 16 * jj];
#pragma unroll
            for (int ii = 0; ii < R; ++ii)
#pragma unroll
                for (int jj = 0; jj < R; ++jj) acc[ii][jj] += x[ii] * y[jj];
        }
        int m = 0;
#pragma unroll
        for (int ii = 0; ii < R; ++ii)
#pragma unroll
            for (int jj = 0; jj < R; ++jj) {
                int i = ty + 16 * ii, j = tx + 16 * jj;
                if (mask && i - j > N) acc[ii][jj] = 0;
                m = max(m, abs(acc[ii][jj]));
            }
        m = block_max_i(m, redi);
        const float mf = (float)m;
        const float rn = m > 0 ? __fdiv_rn(127.f, mf) : 0.f;
        const float sn = m > 0 ? __fmul_rn(__fmul_rn(sprev, s1), __fdiv_rn(mf, 127.f)) : 0.f;
        __syncthreads();
#pragma unroll
        for (int ii = 0; ii < R; ++ii)
#pragma unroll
            for (int jj = 0; jj < R; ++jj) {
                int i = ty + 16 * ii, j = tx + 16 * jj;
                int q = m > 0 ? quant_code((float)acc[ii][jj], rn) : 0;
                qps[i * LD + j] = q;
                t[ii][jj] = __fadd_rn(t[ii][jj], __fmul_rn(sn, (float)q));
                if (qd) qd[((c * N + n) * K + i) * K + j] = (int8_t)q;
                if (accd) accd[((c * N + n) * K + i) * K + j] = acc[ii][jj];
            }
        if (sd && threadIdx.x == 0) sd[c * N + n] = sn;
        sprev = sn;
    }
    float* Tc = T + c * K * K;
#pragma unroll
    for (int ii = 0; ii < R; ++ii)
#pragma unroll
        for (int jj = 0; jj < R; ++jj) Tc[(ty + 16 * ii) * K + tx + 16 * jj] = t[ii][jj];
}

// ------------------------------------------------------------------------- //
// launchers
// ------------------------------------------------------------------------- //
template <typename F>
static cudaError_t prep(F* f, size_t smem) {
    if (smem > 48 * 1024)
        return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return cudaSuccess;
}

#define GDN_DISPATCH_K(k, ...)                     \
    switch (k) {                                   \
        case 32: { constexpr int KK = 32; __VA_ARGS__; } break;   \
        case 64: { constexpr int KK = 64; __VA_ARGS__; } break;   \
        case 128: { constexpr int KK = 128; __VA_ARGS__; } break; \
        default: return cudaErrorInvalidValue;     \
    }

template <typename TI>
static cudaError_t build_A_t(const TI* K, const float* beta, const float* g, float* A,
                             int64_t nc, int k, cudaStream_t st) {
    GDN_DISPATCH_K(k, {
        size_t smem = (KK * kLdK + KK * (KK + 1) + 2 * KK) * sizeof(float);
        cudaError_t e = prep(k_build_A_simt<KK, TI>, smem);
        if (e != cudaSuccess) return e;
        k_build_A_simt<KK, TI><<<(unsigned)nc, kSimtThreads, smem, st>>>(K, beta, g, A);
    });
    return cudaGetLastError();
}

cudaError_t launch_build_A_simt(const void* K, const float* beta, const float* g, float* A,
                                int64_t nc, int k, bool bf16, cudaStream_t st) {
    if (k == 256) {
        const size_t smem = (256 * kLdK + 2 * 256) * sizeof(float);
        cudaError_t e;
        if (bf16) {
            e = prep(k_build_A_simt256<__nv_bfloat16>, smem);
            if (e != cudaSuccess) return e;
            k_build_A_simt256<__nv_bfloat16><<<(unsigned)nc, kSimtThreads, smem, st>>>(
                (const __nv_bfloat16*)K, beta, g, A);
        } else {
            e = prep(k_build_A_simt256<float>, smem);
            if (e != cudaSuccess) return e;
            k_build_A_simt256<float><<<(unsigned)nc, kSimtThreads, smem, st>>>((const float*)K,
                                                                              beta, g, A);
        }
        return cudaGetLastError();
    }
    return bf16 ? build_A_t((const __nv_bfloat16*)K, beta, g, A, nc, k, st)
                : build_A_t((const float*)K, beta, g, A, nc, k, st);
}

cudaError_t launch_neumann_simt(const float* A, float* T, int64_t nc, int k, int N, int mask,
                                int S, cudaStream_t st) {
    GDN_DISPATCH_K(k, {
        size_t smem = 2 * KK * (KK + 1) * sizeof(float);
        cudaError_t e = prep(k_neumann_simt<KK>, smem);
        if (e != cudaSuccess) return e;
        k_neumann_simt<KK><<<(unsigned)nc, kSimtThreads, smem, st>>>(A, T, N, mask, S);
    });
    return cudaGetLastError();
}

template <typename TI>
static cudaError_t wy_t(const float* T, const TI* K, const TI* V, const float* beta,
                        const float* g, TI* W, TI* U, int64_t nc, int k, cudaStream_t st) {
    GDN_DISPATCH_K(k, {
        size_t smem = (KK * kLdK + KK * (KK + 1) + 2 * KK) * sizeof(float);
        cudaError_t e = prep(k_wy_simt<KK, TI>, smem);
        if (e != cudaSuccess) return e;
        k_wy_simt<KK, TI><<<(unsigned)nc, kSimtThreads, smem, st>>>(T, K, V, beta, g, W, U);
    });
    return cudaGetLastError();
}

cudaError_t launch_wy_simt(const float* T, const void* K, const void* V, const float* beta,
                           const float* g, void* W, void* U, int64_t nc, int k, bool bf16,
                           cudaStream_t st) {
    return bf16 ? wy_t(T, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, beta, g,
                       (__nv_bfloat16*)W, (__nv_bfloat16*)U, nc, k, st)
                : wy_t(T, (const float*)K, (const float*)V, beta, g, (float*)W, (float*)U,
                       nc, k, st);
}

template <typename TI>
static cudaError_t fused_t(const TI* K, const TI* V, const float* beta, const float* g, int N,
                           int mask, int S, int gated, TI* W, TI* U, float* Tout, int64_t nc,
                           int k, cudaStream_t st) {
    GDN_DISPATCH_K(k, {
        size_t smem = (KK * kLdK + 2 * KK * (KK + 1) + 3 * KK) * sizeof(float);
        cudaError_t e = prep(k_fused_simt<KK, TI>, smem);
        if (e != cudaSuccess) return e;
        k_fused_simt<KK, TI><<<(unsigned)nc, kSimtThreads, smem, st>>>(K, V, beta, g, N, mask, S,
                                                                      gated, W, U, Tout);
    });
    return cudaGetLastError();
}

cudaError_t launch_fused_simt(const void* K, const void* V, const float* beta, const float* g,
                              int N, int mask, int S, int gated, void* W, void* U, float* Tout,
                              int64_t nc, int k, bool bf16, cudaStream_t st) {
    return bf16 ? fused_t((const __nv_bfloat16*)K, (const __nv_bfloat16*)V, beta, g, N, mask, S,
                          gated, (__nv_bfloat16*)W, (__nv_bfloat16*)U, Tout, nc, k, st)
                : fused_t((const float*)K, (const float*)V, beta, g, N, mask, S, gated, (float*)W,
                          (float*)U, Tout, nc, k, st);
}

cudaError_t launch_fwdsub(const float* A, float* T, int64_t nc, int k, cudaStream_t st) {
    if (k <= 64) {
        const size_t smem = (size_t)kFwdWarps * k * k * sizeof(float);
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int64_t need = (nc + kFwdWarps - 1) / kFwdWarps;
        const int64_t cap = (int64_t)sms * 8;
        const unsigned grid = (unsigned)(need < cap ? need : cap);
        cudaError_t e;
        if (k == 32) {
            e = prep(k_fwdsub_warp<32>, smem);
            if (!e) k_fwdsub_warp<32><<<grid, 32 * kFwdWarps, smem, st>>>(A, T, nc);
        } else {
            e = prep(k_fwdsub_warp<64>, smem);
            if (!e) k_fwdsub_warp<64><<<grid, 32 * kFwdWarps, smem, st>>>(A, T, nc);
        }
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    if (k == 128) {
        const size_t smem = (size_t)(128 * 128 + 3 * 64 * 64) * sizeof(float);
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int64_t cap = (int64_t)sms * 2;
        const unsigned grid = (unsigned)(nc < cap ? nc : cap);
        cudaError_t e = prep(k_fwdsub128<128>, smem);
        if (e != cudaSuccess) return e;
        k_fwdsub128<128><<<grid, 128, smem, st>>>(A, T, nc);
        return cudaGetLastError();
    }
    if (k == 256) {                            // diagonal 128-blocks, then the off-diagonal one
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const size_t smem1 = (size_t)(128 * 128 + 3 * 64 * 64) * sizeof(float);
        cudaError_t e = prep(k_fwdsub128<256>, smem1);
        if (e != cudaSuccess) return e;
        const int64_t nd = 2 * nc, cap1 = (int64_t)sms * 2;
        k_fwdsub128<256><<<(unsigned)(nd < cap1 ? nd : cap1), 128, smem1, st>>>(A, T, nd);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        const size_t smem2 = (size_t)3 * 128 * 128 * sizeof(float);
        e = prep(k_fwdsub256_off, smem2);
        if (e != cudaSuccess) return e;
        const int64_t cap2 = sms;
        k_fwdsub256_off<<<(unsigned)(nc < cap2 ? nc : cap2), 256, smem2, st>>>(A, T, nc);
        return cudaGetLastError();
    }
    const int CB = k < 128 ? k : 128;
    const int nb = k / CB;
    dim3 grid((unsigned)nc, (unsigned)nb);
    // shared memory is sized for the first column block (largest L = k)
    size_t smem = (size_t)(k * CB + k * 8) * sizeof(float);
    cudaError_t e = cudaSuccess;
    switch (k) {
        case 32: e = prep(k_fwdsub<32>, smem); if (!e) k_fwdsub<32><<<grid, CB, smem, st>>>(A, T); break;
        case 64: e = prep(k_fwdsub<64>, smem); if (!e) k_fwdsub<64><<<grid, CB, smem, st>>>(A, T); break;
        case 128: e = prep(k_fwdsub<128>, smem); if (!e) k_fwdsub<128><<<grid, CB, smem, st>>>(A, T); break;
        case 256: e = prep(k_fwdsub<256>, smem); if (!e) k_fwdsub<256><<<grid, CB, smem, st>>>(A, T); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_neumann_i8_simt(const float* A, float* T, int N, int mask, int8_t* q,
                                   int32_t* acc, float* sc, int64_t nc, cudaStream_t st) {
    k_neumann_i8_simt<<<(unsigned)nc, kSimtThreads, 0, st>>>(A, T, N, mask, q, acc, sc);
    return cudaGetLastError();
}

}  // namespace gdn
