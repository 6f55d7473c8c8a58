// scan.cu — the inter-chunk state recurrence of the chunk-wise Gated DeltaNet
// forward (fp32 state).
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
// slice of S.
//
// bf16 data: only V~ and S' are on the serial path.  k_state_tc runs them
// alone (tiles fetched two chunks ahead by TMA, which one thread issues while
// the others compute, the state slice held as fp32 mma.sync accumulator
// fragments), writing V~ over U and each
// chunk's start state S_c to the workspace; the output pass (k_output_tc in
// tc.cu, on the tensor cores) then forms O for every chunk in parallel.  fp32
// data: k_scan does the whole recurrence and O in one pass with fp32 FMA loops.
#include <cuda.h>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "tc.h"

namespace gdn {

constexpr int kScanThreads = 256;
constexpr int kSD = 128;          // d_k = d_v
constexpr int kDV = 16;           // state rows per CTA
constexpr int kSK = 64;           // chunk size served by the scan

template <typename TI>
struct ScanTile {
    static constexpr int kPitch = (sizeof(TI) == 2) ? kSD + 8 : kSD + 4;   // elements, 16-B rows
    static constexpr int kTileBytes = kSK * kPitch * (int)sizeof(TI);
    static constexpr int kUBytes = kSK * kDV * (int)sizeof(TI);
    // one stage: Q, K, W tiles, the U slice and g
    static constexpr int kStage = 3 * kTileBytes + kUBytes + kSK * 4;
    static constexpr int kStages = (sizeof(TI) == 2) ? 2 : 1;   // fp32 tiles: single buffer
};

// e^x = 2^(x log2 e), with the PTX base-2 exponential ex2.approx.ftz
// (relative error about 2^-22 by the PTX ISA); arguments here are <= 0.
__device__ __forceinline__ float exp_e(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x * 1.4426950408889634f));
    return y;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// Fetch chunk `row0`'s tiles into stage buffer `st` (all threads; async).
template <typename TI>
__device__ __forceinline__ void fetch_chunk(uint8_t* st, const TI* Q, const TI* K, const TI* Wg,
                                            const TI* U, const float* g, int64_t row0, int v0) {
    using L = ScanTile<TI>;
    constexpr int kVec = 16 / sizeof(TI);                 // elements per 16-byte copy
    constexpr int kPerRow = kSD / kVec;
    const TI* src[3] = {Q + row0 * kSD, K + row0 * kSD, Wg + row0 * kSD};
#pragma unroll
    for (int m = 0; m < 3; ++m) {
        TI* dst = reinterpret_cast<TI*>(st + m * L::kTileBytes);
        for (int e = threadIdx.x; e < kSK * kPerRow; e += kScanThreads) {
            const int r = e / kPerRow, c = (e % kPerRow) * kVec;
            cp_async16(dst + r * L::kPitch + c, src[m] + r * kSD + c);
        }
    }
    {
        constexpr int kUVec = kDV / kVec;                 // 16-byte copies per U row slice
        TI* dst = reinterpret_cast<TI*>(st + 3 * L::kTileBytes);
        for (int e = threadIdx.x; e < kSK * kUVec; e += kScanThreads) {
            const int r = e / kUVec, c = (e % kUVec) * kVec;
            cp_async16(dst + r * kDV + c, U + (row0 + r) * kSD + v0 + c);
        }
        float* gd = reinterpret_cast<float*>(st + 3 * L::kTileBytes + L::kUBytes);
        if (threadIdx.x < kSK / 4) cp_async16(gd + threadIdx.x * 4, g + row0 + threadIdx.x * 4);
    }
}

// sA[t][j] = (q_t . k_j) e^{g_t - g_j} for j <= t, else 0 (pitch 65).
__device__ __forceinline__ void chunk_scores(const float* Qs, const float* Ks, const float* gs,
                                             float* sA) {
    constexpr int P = ScanTile<float>::kPitch;
    for (int e = threadIdx.x; e < kSK * kSK; e += kScanThreads) {
        const int t = e / kSK, j = e % kSK;
        float a = 0.f;
        if (j <= t) {
            const float* qr = Qs + t * P;
            const float* kr = Ks + j * P;
#pragma unroll 8
            for (int c = 0; c < kSD; ++c) a = fmaf(qr[c], kr[c], a);
            a *= exp_e(gs[t] - gs[j]);
        }
        sA[t * (kSK + 1) + j] = a;
    }
}

template <typename TI>
__global__ void __launch_bounds__(kScanThreads)
k_scan(const TI* __restrict__ Q, const TI* __restrict__ K, const TI* __restrict__ Wg,
       const TI* __restrict__ U, const float* __restrict__ g, const float* __restrict__ S0,
       TI* __restrict__ O, float* __restrict__ Sfin, int64_t nchunk) {
    using L = ScanTile<TI>;
    constexpr int P = L::kPitch;
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* stage[2] = {smem, smem + (L::kStages - 1) * L::kStage};
    float* sS = reinterpret_cast<float*>(smem + L::kStages * L::kStage);   // [DV][129] state
    constexpr int kSP = kSD + 1;
    float* sVt = sS + kDV * kSP;            // [64][DV]  V~ slice (times e^{g_last - g_t} later)
    float* sP = sVt + kSK * kDV;            // [64][DV]  Q S^T slice
    float* sA = sP + kSK * kDV;             // [64][65]  scores . Gamma . L
    float* sgam = sA + kSK * (kSK + 1);     // [64] e^{g_t}
    float* sdec = sgam + kSK;               // [64] e^{g_last - g_t}
    const int64_t bh = blockIdx.x;
    const int v0 = blockIdx.y * kDV;
    const int tid = threadIdx.x;

    for (int e = tid; e < kDV * kSD; e += kScanThreads) {
        const int v = e / kSD, c = e % kSD;
        sS[v * kSP + c] = S0 ? S0[(bh * kSD + v0 + v) * kSD + c] : 0.f;
    }
    if (L::kStages == 2) {
        fetch_chunk(stage[0], Q, K, Wg, U, g, bh * nchunk * kSK, v0);
        cp_async_commit();
    }

    // thread -> (token t, 4 state rows) for the 64 x DV products
    const int pt = tid >> 2, pv = (tid & 3) * 4;
    // thread -> (state row v, 8 columns) for the DV x 128 state update
    const int uv = tid >> 4, uc = (tid & 15) * 8;

    for (int64_t ci = 0; ci < nchunk; ++ci) {
        const int64_t row0 = (bh * nchunk + ci) * kSK;
        uint8_t* cur = stage[ci & 1];
        if (L::kStages == 1) {
            fetch_chunk(cur, Q, K, Wg, U, g, row0, v0);
            cp_async_commit();
            cp_async_wait0();
        } else if (ci + 1 < nchunk) {
            fetch_chunk(stage[(ci + 1) & 1], Q, K, Wg, U, g, row0 + kSK, v0);
            cp_async_commit();
            cp_async_wait1();
        } else {
            cp_async_wait0();
        }
        __syncthreads();
        const TI* Qs = reinterpret_cast<const TI*>(cur);
        const TI* Ks = reinterpret_cast<const TI*>(cur + L::kTileBytes);
        const TI* Ws = reinterpret_cast<const TI*>(cur + 2 * L::kTileBytes);
        const TI* Us = reinterpret_cast<const TI*>(cur + 3 * L::kTileBytes);
        const float* gs = reinterpret_cast<const float*>(cur + 3 * L::kTileBytes + L::kUBytes);
        if (tid < kSK) {
            sgam[tid] = exp_e(gs[tid]);
            sdec[tid] = exp_e(gs[kSK - 1] - gs[tid]);
        }
        chunk_scores(Qs, Ks, gs, sA);
        // V~ = U - W_g S^T and P = Q S^T on the slice
        {
            float w[4] = {0.f, 0.f, 0.f, 0.f}, q[4] = {0.f, 0.f, 0.f, 0.f};
            const TI* wr = Ws + pt * P;
            const TI* qr = Qs + pt * P;
#pragma unroll 4
            for (int c = 0; c < kSD; ++c) {
                const float wc = to_f(wr[c]), qc = to_f(qr[c]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float sv = sS[(pv + i) * kSP + c];
                    w[i] = fmaf(wc, sv, w[i]);
                    q[i] = fmaf(qc, sv, q[i]);
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                sVt[pt * kDV + pv + i] = to_f(Us[pt * kDV + pv + i]) - w[i];
                sP[pt * kDV + pv + i] = q[i];
            }
        }
        __syncthreads();
        // O = diag(gamma) P + (scores . Gamma . L) V~
        {
            const float* ar = sA + pt * (kSK + 1);
            float o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) o[i] = sgam[pt] * sP[pt * kDV + pv + i];
            for (int j = 0; j <= pt; ++j) {
                const float a = ar[j];
                const float4 vv = *reinterpret_cast<const float4*>(sVt + j * kDV + pv);
                o[0] = fmaf(a, vv.x, o[0]);
                o[1] = fmaf(a, vv.y, o[1]);
                o[2] = fmaf(a, vv.z, o[2]);
                o[3] = fmaf(a, vv.w, o[3]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) st_elem(O, (row0 + pt) * kSD + v0 + pv + i, o[i]);
        }
        // S' = gamma_last S + V~^T diag(e^{g_last - g}) K
        {
            float acc[8];
            const float gam = sgam[kSK - 1];
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[c] = gam * sS[uv * kSP + uc + c];
            for (int t = 0; t < kSK; ++t) {
                const float a = sVt[t * kDV + uv] * sdec[t];
                const TI* kr = Ks + t * P + uc;
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[c] = fmaf(a, to_f(kr[c]), acc[c]);
            }
#pragma unroll
            for (int c = 0; c < 8; ++c) sS[uv * kSP + uc + c] = acc[c];
        }
        __syncthreads();                // stage buffer and state free for the next chunk
    }
    for (int e = tid; e < kDV * kSD; e += kScanThreads) {
        const int v = e / kSD, c = e % kSD;
        Sfin[(bh * kSD + v0 + v) * kSD + c] = sS[v * kSP + c];
    }
}

// ------------------------------------------------------------------------- //
// bf16 data: mma.sync m16n8k16 with fp32 accumulation.  Operands pass through
// shared memory as fp16 (W_g, Q converted exactly from bf16; S, V~, scores
// rounded to fp16) or bf16 (K, V~ diag(decay)).
// ------------------------------------------------------------------------- //
struct ScanMma {
    static constexpr int kP16 = kSK + 8;          // pitch of 64-wide fp16/bf16 rows
    static constexpr int kPS = kSD + 8;           // pitch of the fp16 copy of S
};

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_h2f(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_b2f(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// ---------------------------------------------------------------------------
// bf16 forward in two kernels.  The recurrence is the only serial part, so it
// runs alone (k_state_tc: per chunk V~ = U - W_g S^T, written over U as fp16,
// the chunk's start state S_c stored as fp16, S <- gamma_last S + (V~ dec)^T K),
// and the output of every chunk follows in parallel (k_output_tc in tc.cu:
// O = diag(gamma) Q S_c^T + (Q K^T . Gamma . L) V~ on the tensor cores).
// ---------------------------------------------------------------------------
constexpr int kStThreads = 128;
constexpr int kStStages = 3;

// One stage: the chunk's K and W_g tiles as two 64-column panels each with the
// 128-byte swizzle (the TMA layout), the U slice [64][16] and g [64], dense.
struct StTile {
    static constexpr int kTile = kSK * kSD * 2;                // 16 KB, 1024-byte aligned
    static constexpr int kU = kSK * kDV * 2;
    static constexpr int kTx = 2 * kTile + kU + kSK * 4;       // bytes the TMA brings
    static constexpr int kStage = (kTx + 1023) / 1024 * 1024;  // K, W_g, U slice, g
};
// byte offset of element (row, col) of a staged [64][128] bf16 tile
__device__ __forceinline__ uint32_t sw128(int row, int col) {
    return (uint32_t)(((col >> 6) << 13) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) +
                      ((col & 7) << 1));
}
__device__ __forceinline__ uint32_t sh32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
// four 8 x 8 b16 matrices: lanes 8j .. 8j + 7 give the row addresses of matrix j
__device__ __forceinline__ void ldsm_x4(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(a));
}
__device__ __forceinline__ void ldsm_x4t(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                         uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(a));
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ void sbar_init(uint64_t* b) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sh32(b)) : "memory");
}
__device__ __forceinline__ void sbar_expect(uint64_t* b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(sh32(b)),
                 "r"(bytes) : "memory");
}
__device__ __forceinline__ bool sbar_try(uint64_t* b, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(sh32(b)), "r"(parity) : "memory");
    return ok != 0;
}
// bounded (2 s of %globaltimer): false when the tiles never landed
__device__ __forceinline__ bool sbar_wait(uint64_t* b, uint32_t parity) {
    if (sbar_try(b, parity)) return true;
    unsigned long long t0, t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    while (true) {
        for (int i = 0; i < 64; ++i)
            if (sbar_try(b, parity)) return true;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        if (t - t0 > 2000000000ull) return false;
    }
}
__device__ __forceinline__ void tma2d(void* dst, const CUtensorMap* m, int x, int y, uint64_t* b) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(sh32(dst)), "l"(m), "r"(x), "r"(y), "r"(sh32(b))
        : "memory");
}
__device__ __forceinline__ void tma1d(void* dst, const CUtensorMap* m, int x, uint64_t* b) {
    asm volatile(
        "cp.async.bulk.tensor.1d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2}], [%3];" ::"r"(sh32(dst)), "l"(m), "r"(x), "r"(sh32(b))
        : "memory");
}

// the producer warp's lane 0: the TMA copies of one stage (chunk rows row0 ..
// row0 + 63)
__device__ __forceinline__ void fetch_state(uint8_t* st, uint64_t* bar, const CUtensorMap* mK,
                                            const CUtensorMap* mW, const CUtensorMap* mU,
                                            const CUtensorMap* mG, int row0, int v0) {
    // the stage's previous reads were generic; its new writes come from the async proxy
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    sbar_expect(bar, StTile::kTx);
    tma2d(st, mK, 0, row0, bar);
    tma2d(st + StTile::kTile / 2, mK, 64, row0, bar);
    tma2d(st + StTile::kTile, mW, 0, row0, bar);
    tma2d(st + StTile::kTile + StTile::kTile / 2, mW, 64, row0, bar);
    tma2d(st + 2 * StTile::kTile, mU, v0, row0, bar);
    tma1d(st + 2 * StTile::kTile + StTile::kU, mG, row0, bar);
}

// kStThreads compute threads (4 warps) plus one producer warp that only issues
// the stages' TMA copies between the two barriers of each chunk step
__global__ void __launch_bounds__(kStThreads + 32, 1)
k_state_tc(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mW,
           const __grid_constant__ CUtensorMap mU, const __grid_constant__ CUtensorMap mG,
           __nv_bfloat16* __restrict__ U, const float* __restrict__ S0,
           __half* __restrict__ Sst, float* __restrict__ Sfin, int64_t nchunk, int* status) {
    constexpr int P16 = ScanMma::kP16;
    constexpr int PS = ScanMma::kPS;
    extern __shared__ __align__(1024) uint8_t smem[];
    if ((sh32(smem) & 1023u) != 0) {                // the swizzled tiles need 1024-byte alignment
        if (threadIdx.x == 0) raise_status(status, 2);
        return;
    }
    // kStStages stages: the tiles of chunks ci + 1 .. ci + kStStages - 1 stream
    // in while chunk ci is used
    // S as bf16 (the right operand of W_g S^T, bf16 like W_g; the state itself
    // stays fp32 in the accumulator fragments)
    __nv_bfloat16* sSh = reinterpret_cast<__nv_bfloat16*>(smem + kStStages * StTile::kStage);
    __nv_bfloat16* sVd = reinterpret_cast<__nv_bfloat16*>(sSh + kDV * PS);      // [16][72]
    uint64_t* sbar = reinterpret_cast<uint64_t*>(sVd + kDV * P16);                // [kStStages]
    // raised by a thread whose wait ran out, only before the first barrier of a
    // chunk step, and read only after it: the step's second barrier keeps the
    // next step's writes away from this step's reads, so all threads agree
    int* sstop = reinterpret_cast<int*>(sbar + kStStages);   // barriers order its accesses
    const int64_t bh = blockIdx.x;
    const int v0 = blockIdx.y * kDV;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gr = lane >> 2, gc = (lane & 3) * 2;
    const int mt = 16 * warp;                      // token rows of this warp (V~)

    if (tid == kStThreads) {
        *sstop = 0;
        for (int q = 0; q < kStStages; ++q) sbar_init(&sbar[q]);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int q = 0; q < kStStages - 1; ++q)
            if (q < nchunk)
                fetch_state(smem + q * StTile::kStage, &sbar[q], &mK, &mW, &mU, &mG,
                            (int)((bh * nchunk + q) * kSK), v0);
    }
    if (warp == kStThreads / 32) {                 // the producer warp
        __syncthreads();                           // the barriers exist
        int64_t ci = 0;
        for (; ci < nchunk; ++ci) {
            if (!sbar_wait(&sbar[ci % kStStages], (uint32_t)((ci / kStStages) & 1))) *sstop = 1;
            __syncthreads();                       // stage of chunk ci - 1 is free
            if (*sstop) break;
            if (lane == 0 && ci + kStStages - 1 < nchunk) {
                const int nx = (int)((ci + kStStages - 1) % kStStages);
                fetch_state(smem + nx * StTile::kStage, &sbar[nx], &mK, &mW, &mU, &mG,
                            (int)((bh * nchunk + ci + kStStages - 1) * kSK), v0);
            }
            __syncthreads();
        }
        // after a stop, the copies already started (chunks ci .. ci + kStStages - 2)
        // land before the CTA's shared memory goes away; each wait is bounded
        if (ci < nchunk && lane == 0) {
            const int64_t last = ci + kStStages - 1 < nchunk ? ci + kStStages - 1 : nchunk;
            for (int64_t cj = ci; cj < last; ++cj)
                sbar_wait(&sbar[cj % kStStages], (uint32_t)((cj / kStStages) & 1));
        }
        return;
    }
    __syncthreads();                               // the barriers exist

    float Sacc[4][4];                              // columns 32w + 8nt + gc, rows gr, gr + 8
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        const int c = 32 * warp + 8 * nt + gc;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int v = gr + 8 * hh;
            const float s0 = S0 ? S0[(bh * kSD + v0 + v) * kSD + c] : 0.f;
            const float s1 = S0 ? S0[(bh * kSD + v0 + v) * kSD + c + 1] : 0.f;
            Sacc[nt][2 * hh] = s0;
            Sacc[nt][2 * hh + 1] = s1;
            *reinterpret_cast<uint32_t*>(sSh + v * PS + c) = pack_b2f(s0, s1);
        }
    }

    // Two barriers per chunk: the first makes this chunk's tiles and the
    // previous S' (sSh) visible and frees the stage of chunk ci - 1 for the
    // prefetch;
    // the second makes V~ (sVd) visible to the state update.
    for (int64_t ci = 0; ci < nchunk; ++ci) {
        const int64_t row0 = (bh * nchunk + ci) * kSK;
        uint8_t* cur = smem + (ci % kStStages) * StTile::kStage;
        // this chunk's stage has landed (the later ones may be in flight); the
        // CTA stops together when any thread's wait ran out
        if (!sbar_wait(&sbar[ci % kStStages], (uint32_t)((ci / kStStages) & 1))) *sstop = 1;
        __syncthreads();
        if (*sstop) {
            if (tid == 0) raise_status(status, kStatusTimeout);
            return;                                // the state is not written
        }
        const uint32_t Ksa = sh32(cur), Wsa = sh32(cur + StTile::kTile);
        const __nv_bfloat16* Us = reinterpret_cast<const __nv_bfloat16*>(cur + 2 * StTile::kTile);
        const float* gs = reinterpret_cast<const float*>(cur + 2 * StTile::kTile + StTile::kU);
        // the chunk's start state, for the output pass
        {
            __half* dst = Sst + ((bh * nchunk + ci) * kSD + v0) * kSD;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int c = 32 * warp + 8 * nt + gc;
                *reinterpret_cast<uint32_t*>(dst + gr * kSD + c) = pack_h2f(Sacc[nt][0], Sacc[nt][1]);
                *reinterpret_cast<uint32_t*>(dst + (gr + 8) * kSD + c) =
                    pack_h2f(Sacc[nt][2], Sacc[nt][3]);
            }
        }
        // V~ = U - W_g S^T on rows mt .. mt + 15 (two accumulation chains)
        {
            float acc[2][4], acc2[2][4];
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[n][i] = acc2[n][i] = 0.f;
            // fragments by ldmatrix: A rows lane % 16, columns + 8 (lane / 16);
            // B (rows of S) rows (lane % 8) + 8 (lane / 16), columns + 8 ((lane / 8) % 2)
            const int lr = lane & 15, lc = (lane >> 4) * 8;
            const uint32_t sbase = sh32(sSh) + (uint32_t)((((lane & 7) + ((lane >> 4) << 3)) * PS +
                                                           ((lane >> 3) & 1) * 8) * 2);
#pragma unroll
            for (int k0 = 0; k0 < kSD; k0 += 16) {
                uint32_t a0, a1, a2, a3, b00, b01, b10, b11;
                ldsm_x4(Wsa + sw128(mt + lr, k0 + lc), a0, a1, a2, a3);
                ldsm_x4(sbase + k0 * 2, b00, b01, b10, b11);
                mma_bf16(k0 < kSD / 2 ? acc[0] : acc2[0], a0, a1, a2, a3, b00, b01);
                mma_bf16(k0 < kSD / 2 ? acc[1] : acc2[1], a0, a1, a2, a3, b10, b11);
            }
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[n][i] += acc2[n][i];
            const float gl1 = gs[kSK - 1];
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                const int v = 8 * n + gc;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int t = mt + gr + 8 * hh;
                    const float dec = exp_e(gl1 - gs[t]);
                    const float x0 = __bfloat162float(Us[t * kDV + v]) - acc[n][2 * hh];
                    const float x1 = __bfloat162float(Us[t * kDV + v + 1]) - acc[n][2 * hh + 1];
                    sVd[v * P16 + t] = __float2bfloat16_rn(x0 * dec);
                    sVd[(v + 1) * P16 + t] = __float2bfloat16_rn(x1 * dec);
                    // V~ replaces U (fp16 bits)
                    *reinterpret_cast<uint32_t*>(U + (row0 + t) * kSD + v0 + v) = pack_h2f(x0, x1);
                }
            }
        }
        __syncthreads();
        // S' = gamma_last S + (V~ dec)^T K, columns 32w .. 32w + 31
        {
            const float gl = exp_e(gs[kSK - 1]);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) Sacc[nt][i] *= gl;
            const uint32_t vbase = sh32(sVd) + (uint32_t)(((lane & 15) * P16 + (lane >> 4) * 8) * 2);
#pragma unroll
            for (int k0 = 0; k0 < kSK; k0 += 16) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4(vbase + k0 * 2, a0, a1, a2, a3);
                const int krow = k0 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
                for (int nt = 0; nt < 4; nt += 2) {
                    uint32_t b0, b1, b2, b3;             // columns n0 and n0 + 8
                    ldsm_x4t(Ksa + sw128(krow, 32 * warp + 8 * nt + (lane >> 4) * 8), b0, b1, b2, b3);
                    mma_bf16(Sacc[nt], a0, a1, a2, a3, b0, b1);
                    mma_bf16(Sacc[nt + 1], a0, a1, a2, a3, b2, b3);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int c = 32 * warp + 8 * nt + gc;
                *reinterpret_cast<uint32_t*>(sSh + gr * PS + c) = pack_b2f(Sacc[nt][0], Sacc[nt][1]);
                *reinterpret_cast<uint32_t*>(sSh + (gr + 8) * PS + c) =
                    pack_b2f(Sacc[nt][2], Sacc[nt][3]);
            }
        }
    }
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        const int c = 32 * warp + 8 * nt + gc;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int v = gr + 8 * hh;
            Sfin[(bh * kSD + v0 + v) * kSD + c] = Sacc[nt][2 * hh];
            Sfin[(bh * kSD + v0 + v) * kSD + c + 1] = Sacc[nt][2 * hh + 1];
        }
    }
}

// tensor maps of the recurrence's stages
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
static EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)ptr;
    }
    return fn;
}
// [rows, 128] bf16, box box_cols x box_rows
static bool map_bf16_2d(CUtensorMap* m, const void* base, int64_t rows, int box_cols,
                        int box_rows, CUtensorMapSwizzle sw) {
    EncodeTiledFn f = encode_tiled();
    if (!f) return false;
    memset(m, 0, sizeof *m);
    cuuint64_t dims[2] = {(cuuint64_t)kSD, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)kSD * 2};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// [rows] fp32, box box_rows
static bool map_f32_1d(CUtensorMap* m, const void* base, int64_t rows, int box_rows) {
    EncodeTiledFn f = encode_tiled();
    if (!f) return false;
    memset(m, 0, sizeof *m);
    cuuint64_t dims[1] = {(cuuint64_t)rows};
    cuuint64_t strides[1] = {4};
    cuuint32_t box[1] = {(cuuint32_t)box_rows};
    cuuint32_t es[1] = {1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_scan(const void* Q, const void* K, const void* Wg, void* U, const float* g,
                        const float* S0, void* O, float* Sfin, void* Sstates, int64_t BH,
                        int64_t nchunk, bool bf16, cudaStream_t st, bool normalize_q) {
    dim3 grid((unsigned)BH, kSD / kDV);
    if (bf16) {
        const size_t s1 = kStStages * StTile::kStage + (size_t)kDV * ScanMma::kPS * 2 +
                          (size_t)kDV * ScanMma::kP16 * 2 + (kStStages + 1) * sizeof(uint64_t);
        const int64_t rows = BH * nchunk * kSK;
        CUtensorMap mK, mW, mU, mG;
        if (!map_bf16_2d(&mK, K, rows, 64, kSK, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !map_bf16_2d(&mW, Wg, rows, 64, kSK, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !map_bf16_2d(&mU, U, rows, kDV, kSK, CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !map_f32_1d(&mG, g, rows, kSK))
            return cudaErrorInvalidValue;
        cudaError_t e = cudaFuncSetAttribute(k_state_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)s1);
        if (e != cudaSuccess) return e;
        k_state_tc<<<grid, kStThreads + 32, s1, st>>>(mK, mW, mU, mG, (__nv_bfloat16*)U, S0,
                                                 (__half*)Sstates, Sfin, nchunk, status_ptr());
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        return launch_output_tc(Q, K, U, g, Sstates, O, BH * nchunk, normalize_q, st);
    }
    auto smem_for = [](int stage, int nstages) {
        return (size_t)(nstages * stage) + (size_t)(kDV * (kSD + 1) + 2 * kSK * kDV +
                                                    kSK * (kSK + 1) + 2 * kSK) * sizeof(float);
    };
    const size_t smem = smem_for(ScanTile<float>::kStage, 1);
    cudaError_t e = cudaFuncSetAttribute(k_scan<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    k_scan<float><<<grid, kScanThreads, smem, st>>>((const float*)Q, (const float*)K,
                                                     (const float*)Wg, (const float*)U, g, S0,
                                                     (float*)O, Sfin, nchunk);
    return cudaGetLastError();
}

}  // namespace gdn
