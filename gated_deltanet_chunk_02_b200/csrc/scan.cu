// scan.cu — the inter-chunk state recurrence of the chunk-wise Gated DeltaNet
// forward (CUDA cores, fp32 state).
//
// With W_g = T diag(beta e^g) K and U = T diag(beta) V per chunk (computed in
// parallel beforehand), the chunk-wise form of the gated delta rule is, for a
// chunk with chunk-local cumulative log-gates g, gamma = e^g and start state S
// (d_v x d_k):
//     V~ = U - W_g S^T
//     O  = diag(gamma) Q S^T + (Q K^T . Gamma . L) V~,   Gamma_ij = e^{g_i - g_j}
//     S' = gamma_last S + V~^T diag(e^{g_last - g}) K
// (L: lower triangle with the diagonal).  Row v of S only ever meets column v
// of V~, U and O, so the d_v rows split across CTAs with no exchange: grid =
// (B*H, d_v / DV), each CTA walks its head's chunks in order holding a DV x d_k
// slice of S in shared memory.  The chunk's Q, K, W_g tiles are staged in
// shared memory as fp32; the intra-chunk scores Q K^T are recomputed per slice.
#include "common.cuh"
#include "kernels.h"

namespace gdn {

constexpr int kScanThreads = 256;
constexpr int kSD = 128;          // d_k = d_v
constexpr int kSLd = kSD + 1;     // padded pitch
constexpr int kDV = 16;           // state rows per CTA
constexpr int kSK = 64;           // chunk size served by the scan

template <typename TI>
__device__ __forceinline__ void stage_tile(float* dst, const TI* src) {
    for (int e = threadIdx.x; e < kSK * kSD; e += kScanThreads)
        dst[(e / kSD) * kSLd + e % kSD] = ld_elem(src, e);
}

template <typename TI>
__global__ void __launch_bounds__(kScanThreads)
k_scan(const TI* __restrict__ Q, const TI* __restrict__ K, const TI* __restrict__ Wg,
       const TI* __restrict__ U, const float* __restrict__ g, const float* __restrict__ S0,
       TI* __restrict__ O, float* __restrict__ Sfin, int64_t nchunk) {
    extern __shared__ float sm[];
    float* sQ = sm;                         // [64][129]
    float* sK = sQ + kSK * kSLd;            // [64][129]
    float* sW = sK + kSK * kSLd;            // [64][129]
    float* sS = sW + kSK * kSLd;            // [DV][129]   state slice
    float* sVt = sS + kDV * kSLd;           // [64][DV]    V~ slice
    float* sP = sVt + kSK * kDV;            // [64][DV]    Q S^T slice
    float* sA = sP + kSK * kDV;             // [64][65]    scores . Gamma . L
    float* sg = sA + kSK * (kSK + 1);       // [64] g
    float* sgam = sg + kSK;                 // [64] e^{g_t}
    float* sdec = sgam + kSK;               // [64] e^{g_last - g_t}
    const int64_t bh = blockIdx.x;
    const int v0 = blockIdx.y * kDV;
    const int tid = threadIdx.x;

    // state slice
    for (int e = tid; e < kDV * kSD; e += kScanThreads) {
        const int v = e / kSD, c = e % kSD;
        sS[v * kSLd + c] = S0 ? S0[(bh * kSD + v0 + v) * kSD + c] : 0.f;
    }
    for (int64_t ci = 0; ci < nchunk; ++ci) {
        const int64_t row0 = (bh * nchunk + ci) * kSK;
        __syncthreads();
        stage_tile(sQ, Q + row0 * kSD);
        stage_tile(sK, K + row0 * kSD);
        stage_tile(sW, Wg + row0 * kSD);
        if (tid < kSK) sg[tid] = g[row0 + tid];
        __syncthreads();
        if (tid < kSK) {
            sgam[tid] = expf(sg[tid]);
            sdec[tid] = expf(sg[kSK - 1] - sg[tid]);
        }
        // scores: A[t][j] = (q_t . k_j) e^{g_t - g_j} for j <= t; thread -> 16 entries
        for (int e = tid; e < kSK * kSK; e += kScanThreads) {
            const int t = e / kSK, j = e % kSK;
            float a = 0.f;
            if (j <= t) {
                const float* qr = sQ + t * kSLd;
                const float* kr = sK + j * kSLd;
#pragma unroll 8
                for (int c = 0; c < kSD; ++c) a = fmaf(qr[c], kr[c], a);
                a *= expf(sg[t] - sg[j]);
            }
            sA[t * (kSK + 1) + j] = a;
        }
        // V~ = U - W_g S^T and P = Q S^T on the slice: 64 x DV each, 4 per thread
        for (int e = tid; e < kSK * kDV; e += kScanThreads) {
            const int t = e / kDV, v = e % kDV;
            const float* wr = sW + t * kSLd;
            const float* qr = sQ + t * kSLd;
            const float* sr = sS + v * kSLd;
            float ws = 0.f, qs = 0.f;
#pragma unroll 8
            for (int c = 0; c < kSD; ++c) {
                ws = fmaf(wr[c], sr[c], ws);
                qs = fmaf(qr[c], sr[c], qs);
            }
            sVt[t * kDV + v] = ld_elem(U, (row0 + t) * kSD + v0 + v) - ws;
            sP[t * kDV + v] = qs;
        }
        __syncthreads();
        // O = diag(gamma) P + A V~
        for (int e = tid; e < kSK * kDV; e += kScanThreads) {
            const int t = e / kDV, v = e % kDV;
            float o = sgam[t] * sP[t * kDV + v];
            const float* ar = sA + t * (kSK + 1);
            for (int j = 0; j <= t; ++j) o = fmaf(ar[j], sVt[j * kDV + v], o);
            st_elem(O, (row0 + t) * kSD + v0 + v, o);
        }
        // S' = gamma_last S + V~^T diag(e^{g_last - g}) K: DV x 128, 8 per thread
        const float gam = sgam[kSK - 1];
        for (int e = tid; e < kDV * kSD; e += kScanThreads) {
            const int v = e / kSD, c = e % kSD;
            float acc = gam * sS[v * kSLd + c];
            for (int t = 0; t < kSK; ++t)
                acc = fmaf(sVt[t * kDV + v] * sdec[t], sK[t * kSLd + c], acc);
            sS[v * kSLd + c] = acc;
        }
    }
    __syncthreads();
    for (int e = tid; e < kDV * kSD; e += kScanThreads) {
        const int v = e / kSD, c = e % kSD;
        Sfin[(bh * kSD + v0 + v) * kSD + c] = sS[v * kSLd + c];
    }
}

cudaError_t launch_scan(const void* Q, const void* K, const void* Wg, const void* U, const float* g,
                        const float* S0, void* O, float* Sfin, int64_t BH, int64_t nchunk,
                        bool bf16, cudaStream_t st) {
    const size_t smem = (size_t)(3 * kSK * kSLd + kDV * kSLd + 2 * kSK * kDV +
                                 kSK * (kSK + 1) + 3 * kSK) * sizeof(float);
    dim3 grid((unsigned)BH, kSD / kDV);
    cudaError_t e;
    if (bf16) {
        e = cudaFuncSetAttribute(k_scan<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        k_scan<__nv_bfloat16><<<grid, kScanThreads, smem, st>>>(
            (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)Wg,
            (const __nv_bfloat16*)U, g, S0, (__nv_bfloat16*)O, Sfin, nchunk);
    } else {
        e = cudaFuncSetAttribute(k_scan<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        k_scan<float><<<grid, kScanThreads, smem, st>>>((const float*)Q, (const float*)K,
                                                         (const float*)Wg, (const float*)U, g, S0,
                                                         (float*)O, Sfin, nchunk);
    }
    return cudaGetLastError();
}

}  // namespace gdn
