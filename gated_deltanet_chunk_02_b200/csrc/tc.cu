// tc.cu — tcgen05 tensor-core kernels of libgdn (sm_100a).
//
// One persistent kernel template serves the bf16 chunk pipeline in four
// modes: the fused inverse + WY step, A alone, the Neumann inverse alone and
// WY alone.  Design:
//
// * A "tile" is 128 consecutive rows of the flattened [B*H*T, d] arrays, i.e.
//   128/KB chunks of KB tokens (KB = 64 or 128; k = 32 is run as 64-token
//   blocks holding two 32-token chunks block-diagonally).  Every k x k product
//   of the method is one M=128 tcgen05.mma over the tile: the left operand
//   stacks the tile's chunks along M, the right operand places them side by
//   side along N, and each chunk reads only its own diagonal block of the
//   128 x 128 fp32 accumulator in tensor memory (TMEM).
// * Warp 0 is the TMA producer (K, V tiles with 128-byte swizzle, beta and g).
//   Each further 4-warp group ("slot") owns one tile at a time: one elected
//   thread issues its MMAs, all 128 threads run the epilogues (TMEM -> registers
//   -> mask / accumulate / convert -> swizzled shared-memory operand).  Two slots
//   per CTA keep the tensor pipe busy while the other slot's epilogue runs.
// * Thread r of a slot owns row r of the tile: the TMEM lane it may read
//   (lane quarter = warp % 4) is the row it computes.
// * The WY step is computed transposed, W^T = K^T (T diag(beta))^T, so that it
//   is a full-rate M=128 (= d) product; its epilogue writes W, U row-wise.
// * Every wait is bounded (2 s); on expiry the kernel sets the status word,
//   stops issuing work, waits for its own copies/MMAs (bounded) and frees TMEM.
#include <cuda.h>

#include "common.cuh"
#include "tc.h"

namespace gdn {
namespace tcg {

constexpr int kD = 128;
constexpr int kRows = 128;                       // rows per tile
constexpr unsigned long long kTimeoutNs = 2000000000ull;

enum Mode { kFused = 0, kBuildA = 1, kNeumann = 2, kWY = 3 };

__host__ __device__ constexpr bool uses_K(int m) { return m == kFused || m == kBuildA || m == kWY; }
__host__ __device__ constexpr bool uses_V(int m) { return m == kFused || m == kWY; }
__host__ __device__ constexpr bool uses_ops(int m) { return m != kBuildA; }

// Per-slot shared-memory layout (bytes); every region is 1024-byte aligned.
template <int KB, int MODE>
struct SlotLayout {
    static constexpr int kK = uses_K(MODE) ? kRows * kD * 2 : 0;        // bf16 [2][128][64]
    static constexpr int kV = uses_V(MODE) ? kRows * kD * 2 : 0;
    static constexpr int kOp = uses_ops(MODE) ? kRows * KB * 2 : 0;     // 16-bit [KB/64][128][64]
    static constexpr int offK = 0;
    static constexpr int offV = offK + kK;
    static constexpr int offAop = offV + kV;
    static constexpr int offX = offAop + (MODE == kWY ? 0 : kOp);
    static constexpr int offY = offX + kOp;
    static constexpr int bytes = offY + kOp;
};

// ------------------------------------------------------------------------- //
// PTX wrappers
// ------------------------------------------------------------------------- //
__device__ __forceinline__ uint32_t su32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long gtime() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t n) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(n) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)),
                 "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(su32(b)), "r"(parity) : "memory");
    return ok != 0;
}
// Bounded wait on the phase with the given parity; false if it ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity) {
    if (mbar_try(b, parity)) return true;
    const unsigned long long t0 = gtime();
    while (true) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try(b, parity)) return true;
        if (gtime() - t0 > kTimeoutNs) return false;
    }
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* m, int x, int y,
                                            uint64_t* b) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(su32(dst)), "l"(m), "r"(x), "r"(y), "r"(su32(b))
        : "memory");
}
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(dst)),
                 "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* b) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     su32(b))
                 : "memory");
}
// 32 consecutive TMEM columns of this thread's lane -> 32 floats.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 floats -> 32 consecutive TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm100 layout: version 1).
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor of kind::f16 with fp32 accumulation.
// fmt: 0 = fp16, 1 = bf16; major: 0 = K-major, 1 = MN-major.
__host__ __device__ constexpr uint32_t idesc_f16(int fmt, int amaj, int bmaj, int N, int M) {
    return (1u << 4) | ((uint32_t)fmt << 7) | ((uint32_t)fmt << 10) | ((uint32_t)amaj << 15) |
           ((uint32_t)bmaj << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Byte offset of the 16-byte group q (elements 8q .. 8q+7) of row r in a
// 16-bit [KB/64][128][64] operand buffer with the 128-byte swizzle.
__device__ __forceinline__ uint32_t op_off(int r, int q) {
    return (uint32_t)(r * 128 + (q >> 3) * (kRows * 128) + ((((q & 7) ^ (r & 7))) << 4));
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_b2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
// Store 32 values (columns 32p .. 32p+31 of row r) into an operand buffer.
template <bool BF16>
__device__ __forceinline__ void st_op32(uint8_t* buf, int r, int p, const float (&v)[32]) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        uint4 u;
        if (BF16) {
            u.x = pack_b2(v[8 * g + 0], v[8 * g + 1]);
            u.y = pack_b2(v[8 * g + 2], v[8 * g + 3]);
            u.z = pack_b2(v[8 * g + 4], v[8 * g + 5]);
            u.w = pack_b2(v[8 * g + 6], v[8 * g + 7]);
        } else {
            u.x = pack_h2(v[8 * g + 0], v[8 * g + 1]);
            u.y = pack_h2(v[8 * g + 2], v[8 * g + 3]);
            u.z = pack_h2(v[8 * g + 4], v[8 * g + 5]);
            u.w = pack_h2(v[8 * g + 6], v[8 * g + 7]);
        }
        *reinterpret_cast<uint4*>(buf + op_off(r, 4 * p + g)) = u;
    }
}

struct Params {
    int64_t rows;        // B*H*T
    int ntiles;
    int k;               // user chunk size (32, 64, 128)
    int N, mask, S, gated;
    const float* beta;   // [rows]
    const float* g;      // [rows]
    const float* Ain;    // kNeumann
    const float* Tin;    // kWY
    float* Aout;         // kBuildA
    float* Tout;         // kFused (optional), kNeumann
    __nv_bfloat16* W;
    __nv_bfloat16* U;
    int* status;
};

struct __align__(8) Ctrl {
    uint64_t full[2];
    uint64_t kvfree[2];
    uint64_t mma[2];
    uint32_t tmem;
    int abort;
};

// ------------------------------------------------------------------------- //
// the kernel
// ------------------------------------------------------------------------- //
template <int KB, int MODE, int NS>
__global__ void __launch_bounds__(32 + 128 * NS, 1)
k_chunk_tc(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
           const Params p) {
    using L = SlotLayout<KB, MODE>;
    constexpr int NP = KB / 32;                    // 32-column pieces per row of a block
    constexpr int NCH = kRows / KB;                // blocks per tile
    constexpr uint32_t kTmemCols = NS == 2 ? 512 : 256;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem);
    uint8_t* slots = smem + 1024;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&ctrl->full[s], 1);
            mbar_init(&ctrl->kvfree[s], 1);
            mbar_init(&ctrl->mma[s], 1);
        }
        ctrl->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) tmem_alloc(&ctrl->tmem, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctrl->tmem;

    if (warp == 0) {
        // ------------------------------ producer ----------------------------
        if (uses_K(MODE) && lane == 0) {
            constexpr uint32_t kBytes = (uses_K(MODE) ? kRows * kD * 2 : 0) +
                                        (uses_V(MODE) ? kRows * kD * 2 : 0);
            int issued[2] = {0, 0};
            for (int n = 0;; ++n) {
                const int tile = blockIdx.x + n * gridDim.x;
                if (tile >= p.ntiles) break;
                const int s = n % NS, use = n / NS;
                if (use > 0 && !mbar_wait(&ctrl->kvfree[s], (use - 1) & 1)) {
                    atomicExch(&ctrl->abort, 1);
                    break;
                }
                if (*(volatile int*)&ctrl->abort) break;
                uint8_t* base = slots + s * L::bytes;
                const int y = tile * kRows;
                mbar_expect_tx(&ctrl->full[s], kBytes);
                tma_load_2d(base + L::offK, &mK, 0, y, &ctrl->full[s]);
                tma_load_2d(base + L::offK + kRows * 128, &mK, 64, y, &ctrl->full[s]);
                if (uses_V(MODE)) {
                    tma_load_2d(base + L::offV, &mV, 0, y, &ctrl->full[s]);
                    tma_load_2d(base + L::offV + kRows * 128, &mV, 64, y, &ctrl->full[s]);
                }
                issued[s] = use + 1;
            }
            // every copy this warp issued lands before the CTA exits
            for (int s = 0; s < NS; ++s)
                if (issued[s] > 0) mbar_wait(&ctrl->full[s], (issued[s] - 1) & 1);
        }
    } else {
        // ------------------------------ slot s ------------------------------
        // T0 (then T) lives in TMEM columns [128, 128 + KB) of the slot, row r
        // in lane r, so the epilogues carry only 32-column pieces in registers.
        const int s = (warp - 1) / 4;
        const int r = ((warp & 3) << 5) | lane;       // tile row == TMEM lane
        const int blk = r / KB;                        // block of this row in the tile
        const int i = r % KB;                          // row inside the block
        const int sub = (p.k < KB) ? (i / p.k) : 0;    // 32-token chunk inside a 64 block
        const int cl = (p.k < KB) ? sub * p.k : 0;     // first column of that chunk
        const int ch = cl + (p.k < KB ? p.k : KB);     // one past its last column
        uint8_t* base = slots + s * L::bytes;
        uint8_t* sK = base + L::offK;
        uint8_t* sV = base + L::offV;
        uint8_t* sAop = base + L::offAop;
        uint8_t* sX = base + L::offX;
        uint8_t* sY = base + L::offY;
        const uint32_t tm = tmem_base + (uint32_t)(s * 256);
        const uint32_t tl = tm + ((uint32_t)((warp & 3) * 32) << 16);   // this warp's lanes
        const uint32_t tD = tl + blk * KB;            // this row's diagonal block of D
        const uint32_t tT = tl + 128;                 // this row's T0 / T
        const bool leader = ((warp - 1) & 3) == 0 && lane == 0;
        const int bar_id = 1 + s;
        uint32_t mma_phase = 0;
        bool ok = true;

        auto wait_mma = [&]() -> bool {
            bool good = mbar_wait(&ctrl->mma[s], mma_phase);
            mma_phase ^= 1;
            if (!good) { atomicExch(&ctrl->abort, 1); raise_status(p.status, kStatusTimeout); }
            tc_fence_after();
            return good;
        };
        // hand the operands written by this slot to the tensor pipe
        auto publish = [&]() {
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            fence_async_smem();
            tc_fence_before();
            bar_sync(bar_id, 128);
            tc_fence_after();
        };
        // k x k chain product D = a_buf[128 x KB] * b_buf[KB x 128] (b: MN-major)
        auto mma_chain = [&](const uint8_t* a_buf, const uint8_t* b_buf) {
            if (leader) {
                constexpr uint32_t id = idesc_f16(0, 0, 1, 128, 128);
#pragma unroll
                for (int kk = 0; kk < KB / 16; ++kk) {
                    uint64_t a = sdesc(su32(a_buf) + (kk >> 2) * (kRows * 128) + (kk & 3) * 32, 16,
                                       1024);
                    uint64_t b = sdesc(su32(b_buf) + kk * 2048, KB * 128, 1024);
                    mma_ss(tm, a, b, id, kk > 0);
                }
                mma_commit(&ctrl->mma[s]);
            }
        };
        auto in_chunk = [&](int j) { return j >= cl && j < ch; };
        auto eye = [&](int j) { return i == j ? 1.f : 0.f; };

        for (int n = s;; n += NS) {
            const int tile = blockIdx.x + n * gridDim.x;
            if (tile >= p.ntiles) break;
            const int use = n / NS;
            const int64_t row0 = (int64_t)tile * kRows;
            const int64_t grow = row0 + r;
            const bool valid = grow < p.rows;
            const int64_t cidx = grow / p.k;                 // chunk of this row
            const int64_t rin = grow % p.k;                  // row inside the chunk
            const int64_t jrow0 = row0 + blk * KB;           // global row of block column 0
            if (uses_K(MODE)) {
                bool good = mbar_wait(&ctrl->full[s], use & 1);
                if (!good) { atomicExch(&ctrl->abort, 1); raise_status(p.status, kStatusTimeout); }
            }
            bar_sync(bar_id, 128);
            if (*(volatile int*)&ctrl->abort) { ok = false; break; }

            if (MODE == kFused || MODE == kBuildA) {
                // ---- G = K K^T over the tile, then A = -beta_i G_ij exp(g_i - g_j) ----
                if (leader) {
                    tc_fence_after();
                    constexpr uint32_t id = idesc_f16(1, 0, 0, 128, 128);
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk) {
                        uint64_t a = sdesc(su32(sK) + (kk >> 2) * (kRows * 128) + (kk & 3) * 32,
                                           16, 1024);
                        mma_ss(tm, a, a, id, kk > 0);
                    }
                    mma_commit(&ctrl->mma[s]);
                    if (MODE == kBuildA) mma_commit(&ctrl->kvfree[s]);
                }
                if (!wait_mma()) { ok = false; break; }
                const float bi = valid ? __ldg(p.beta + grow) : 0.f;
                const float gi = valid ? __ldg(p.g + grow) : 0.f;
#pragma unroll 1
                for (int pc = 0; pc < NP; ++pc) {
                    float v[32];
                    tmem_ld32(tD + pc * 32, v);
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int j = pc * 32 + jj;
                        const bool in = in_chunk(j) && j < i;
                        const float gj = (in && jrow0 + j < p.rows) ? __ldg(p.g + jrow0 + j) : 0.f;
                        v[jj] = in ? -bi * v[jj] * expf(gi - gj) : 0.f;
                    }
                    if (MODE == kBuildA) {
                        if (valid && pc * 32 >= cl && pc * 32 < ch) {
                            float* dst = p.Aout + cidx * p.k * p.k + rin * p.k + (pc * 32 - cl);
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                reinterpret_cast<float4*>(dst)[q] =
                                    make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                        }
                    } else {
                        float t[32];
                        st_op32<false>(sX, r, pc, v);             // A (chain's right operand)
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const int j = pc * 32 + jj;
                            v[jj] = (p.mask && i - j > p.N) ? 0.f : v[jj];
                            t[jj] = eye(j) + v[jj];
                        }
                        st_op32<false>(sAop, r, pc, v);           // P_1 = M . A
                        tmem_st32(tT + pc * 32, t);                // T0 = I + P_1
                    }
                }
                if (MODE == kBuildA) {
                    tc_fence_before();
                    bar_sync(bar_id, 128);
                    continue;
                }
            } else if (MODE == kNeumann) {
                // ---- A row from global memory ----
#pragma unroll 1
                for (int pc = 0; pc < NP; ++pc) {
                    float v[32], t[32];
                    const bool have = valid && pc * 32 >= cl && pc * 32 < ch;
                    if (have) {
                        const float4* src = reinterpret_cast<const float4*>(
                            p.Ain + cidx * p.k * p.k + rin * p.k + (pc * 32 - cl));
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            float4 a = __ldg(src + q);
                            v[4 * q] = a.x; v[4 * q + 1] = a.y; v[4 * q + 2] = a.z; v[4 * q + 3] = a.w;
                        }
                    } else {
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) v[jj] = 0.f;
                    }
                    st_op32<false>(sX, r, pc, v);
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int j = pc * 32 + jj;
                        v[jj] = (p.mask && i - j > p.N) ? 0.f : v[jj];
                        t[jj] = eye(j) + v[jj];
                    }
                    st_op32<false>(sAop, r, pc, v);
                    tmem_st32(tT + pc * 32, t);
                }
            } else {
                // ---- kWY: T row from global memory ----
#pragma unroll 1
                for (int pc = 0; pc < NP; ++pc) {
                    float t[32];
                    const bool have = valid && pc * 32 >= cl && pc * 32 < ch;
                    if (have) {
                        const float4* src = reinterpret_cast<const float4*>(
                            p.Tin + cidx * p.k * p.k + rin * p.k + (pc * 32 - cl));
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            float4 a = __ldg(src + q);
                            t[4 * q] = a.x; t[4 * q + 1] = a.y; t[4 * q + 2] = a.z; t[4 * q + 3] = a.w;
                        }
                    } else {
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) t[jj] = 0.f;
                    }
                    tmem_st32(tT + pc * 32, t);
                }
            }

            if (MODE == kFused || MODE == kNeumann) {
                // ---- truncated Neumann series, band mask on every power ----
                for (int pw = 2; pw <= p.N; ++pw) {
                    publish();
                    mma_chain(sAop, sX);                                   // P_{n-1} A
                    if (!wait_mma()) { ok = false; break; }
#pragma unroll 1
                    for (int pc = 0; pc < NP; ++pc) {
                        float v[32], t[32];
                        tmem_ld32(tD + pc * 32, v);
                        tmem_ld32(tT + pc * 32, t);
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const int j = pc * 32 + jj;
                            v[jj] = (!in_chunk(j) || (p.mask && i - j > p.N)) ? 0.f : v[jj];
                            t[jj] += v[jj];
                        }
                        tmem_st32(tT + pc * 32, t);
                        if (pw < p.N) st_op32<false>(sAop, r, pc, v);
                    }
                }
                if (!ok) break;
                // ---- parallel residual correction ----
                if (p.S > 0) {
#pragma unroll 1
                    for (int pc = 0; pc < NP; ++pc) {
                        float t[32];
                        tmem_ld32(tT + pc * 32, t);
                        st_op32<false>(sY, r, pc, t);                      // T0
                    }
                    publish();
                    mma_chain(sX, sY);                                      // A T0
                    if (!wait_mma()) { ok = false; break; }
#pragma unroll 1
                    for (int pc = 0; pc < NP; ++pc) {
                        float v[32], t[32];
                        tmem_ld32(tD + pc * 32, v);
                        tmem_ld32(tT + pc * 32, t);
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const int j = pc * 32 + jj;
                            v[jj] = in_chunk(j) ? eye(j) - t[jj] + v[jj] : 0.f;   // E
                        }
                        if (p.S == 1) {
                            st_op32<false>(sY, r, pc, v);                   // Q = E
                            st_op32<false>(sAop, r, pc, t);                 // T0
                        } else {
                            st_op32<false>(sX, r, pc, v);                   // E
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj) v[jj] += eye(pc * 32 + jj);
                            st_op32<false>(sAop, r, pc, v);                 // I + Q_1
                        }
                    }
                    for (int m = 1; m < p.S; ++m) {
                        publish();
                        mma_chain(sAop, sX);                                // (I + Q_m) E
                        if (!wait_mma()) { ok = false; break; }
                        const bool last = (m == p.S - 1);
#pragma unroll 1
                        for (int pc = 0; pc < NP; ++pc) {
                            float v[32];
                            tmem_ld32(tD + pc * 32, v);
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj)
                                if (!in_chunk(pc * 32 + jj)) v[jj] = 0.f;
                            if (last) {
                                float t[32];
                                st_op32<false>(sY, r, pc, v);               // Q_S
                                tmem_ld32(tT + pc * 32, t);
                                st_op32<false>(sAop, r, pc, t);             // T0
                            } else {
#pragma unroll
                                for (int jj = 0; jj < 32; ++jj) v[jj] += eye(pc * 32 + jj);
                                st_op32<false>(sAop, r, pc, v);             // I + Q_{m+1}
                            }
                        }
                    }
                    if (!ok) break;
                    publish();
                    mma_chain(sAop, sY);                                    // T0 Q_S
                    if (!wait_mma()) { ok = false; break; }
#pragma unroll 1
                    for (int pc = 0; pc < NP; ++pc) {
                        float v[32], t[32];
                        tmem_ld32(tD + pc * 32, v);
                        tmem_ld32(tT + pc * 32, t);
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj)
                            if (in_chunk(pc * 32 + jj)) t[jj] += v[jj];         // T = T0 + T0 Q
                        tmem_st32(tT + pc * 32, t);
                    }
                }
                // ---- T out ----
                if (p.Tout) {
#pragma unroll 1
                    for (int pc = 0; pc < NP; ++pc) {
                        float t[32];
                        tmem_ld32(tT + pc * 32, t);
                        if (valid && pc * 32 >= cl && pc * 32 < ch) {
                            float* dst = p.Tout + cidx * p.k * p.k + rin * p.k + (pc * 32 - cl);
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                reinterpret_cast<float4*>(dst)[q] =
                                    make_float4(t[4 * q], t[4 * q + 1], t[4 * q + 2], t[4 * q + 3]);
                        }
                    }
                }
            }

            if (MODE == kFused || MODE == kWY) {
                // ---- WY: T diag(beta [exp g]) -> X (bf16), T diag(beta) -> Y ----
#pragma unroll 1
                for (int pc = 0; pc < NP; ++pc) {
                    float t[32], v[32];
                    tmem_ld32(tT + pc * 32, t);
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int j = pc * 32 + jj;
                        const bool jv = jrow0 + j < p.rows;
                        const float b = jv ? __ldg(p.beta + jrow0 + j) : 0.f;
                        const float bw = p.gated ? b * expf(jv ? __ldg(p.g + jrow0 + j) : 0.f) : b;
                        v[jj] = t[jj] * bw;
                        t[jj] = t[jj] * b;
                    }
                    st_op32<true>(sX, r, pc, v);
                    if (p.gated) st_op32<true>(sY, r, pc, t);
                }
                publish();
                if (leader) {
                    constexpr uint32_t id = idesc_f16(1, 1, 0, KB, 128);
                    const uint8_t* bu = p.gated ? sY : sX;
#pragma unroll
                    for (int c = 0; c < NCH; ++c) {
#pragma unroll
                        for (int kk = 0; kk < KB / 16; ++kk) {
                            const uint32_t ka = su32(sK) + (c * KB + kk * 16) * 128;
                            const uint32_t va = su32(sV) + (c * KB + kk * 16) * 128;
                            const uint32_t bo = (c * KB) * 128 + (kk >> 2) * (kRows * 128) +
                                                (kk & 3) * 32;
                            mma_ss(tm + c * KB, sdesc(ka, kRows * 128, 1024),
                                   sdesc(su32(sX) + bo, 16, 1024), id, kk > 0);
                            mma_ss(tm + 128 + c * KB, sdesc(va, kRows * 128, 1024),
                                   sdesc(su32(bu) + bo, 16, 1024), id, kk > 0);
                        }
                    }
                    mma_commit(&ctrl->mma[s]);
                    mma_commit(&ctrl->kvfree[s]);
                }
                if (!wait_mma()) { ok = false; break; }
                // lane r of the W^T / U^T accumulators is head-dim column d = r
                const int d = r;
#pragma unroll 1
                for (int c = 0; c < NCH; ++c) {
#pragma unroll 1
                    for (int pc = 0; pc < NP; ++pc) {
                        float w[32], u[32];
                        tmem_ld32(tl + c * KB + pc * 32, w);
                        tmem_ld32(tl + 128 + c * KB + pc * 32, u);
                        const int64_t t0 = row0 + c * KB + pc * 32;
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            if (t0 + jj < p.rows) {
                                p.W[(t0 + jj) * kD + d] = __float2bfloat16_rn(w[jj]);
                                p.U[(t0 + jj) * kD + d] = __float2bfloat16_rn(u[jj]);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            bar_sync(bar_id, 128);                 // accumulators free for the next tile
        }
        if (!ok) {
            atomicExch(&ctrl->abort, 1);
            // outstanding MMAs of this slot finish before TMEM is released
            mbar_wait(&ctrl->mma[s], mma_phase);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ------------------------------------------------------------------------- //
// host side
// ------------------------------------------------------------------------- //
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    }
    return fn;
}

// [rows, 128] bf16, box 64 x 128 rows, 128-byte swizzle
static bool map_kd(CUtensorMap* m, const void* base, int64_t rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kRows};
    cuuint32_t es[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int num_sms() {
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

template <int KB, int MODE, int NS>
static cudaError_t launch(const void* K, const void* V, const float* beta, const float* g,
                          const Params& p0, cudaStream_t st) {
    using L = SlotLayout<KB, MODE>;
    CUtensorMap mK, mV;
    memset(&mK, 0, sizeof mK);
    memset(&mV, 0, sizeof mV);
    if (uses_K(MODE) && !map_kd(&mK, K, p0.rows)) return cudaErrorInvalidValue;
    if (uses_V(MODE) && !map_kd(&mV, V, p0.rows)) return cudaErrorInvalidValue;
    Params p = p0;
    p.beta = beta;
    p.g = g;
    p.status = status_ptr();
    size_t smem = 1024 + 1024 + (size_t)NS * L::bytes;
    if (smem < 120 * 1024) smem = 120 * 1024;     // one CTA per SM: it owns the SM's TMEM
    cudaError_t e = cudaFuncSetAttribute(k_chunk_tc<KB, MODE, NS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = p.ntiles < num_sms() ? p.ntiles : num_sms();
    k_chunk_tc<KB, MODE, NS><<<grid, 32 + 128 * NS, smem, st>>>(mK, mV, p);
    return cudaGetLastError();
}

static Params base_params(int64_t nc, int k) {
    Params p;
    memset(&p, 0, sizeof p);
    p.rows = nc * k;
    p.ntiles = (int)((p.rows + kRows - 1) / kRows);
    p.k = k;
    return p;
}

}  // namespace tcg

bool tc_available() { return true; }
bool tc_i8_available() { return false; }

#define GDN_TC_DISPATCH(k, MODE, NS128, ...)                                       \
    (k == 128 ? tcg::launch<128, MODE, NS128>(__VA_ARGS__)                           \
              : tcg::launch<64, MODE, 2>(__VA_ARGS__))

cudaError_t launch_build_A_tc(const void* K, const float* beta, const float* g, float* A,
                              int64_t nc, int k, cudaStream_t st) {
    if (k > 128) return cudaErrorNotSupported;
    tcg::Params p = tcg::base_params(nc, k);
    p.Aout = A;
    return GDN_TC_DISPATCH(k, tcg::kBuildA, 2, K, nullptr, beta, g, p, st);
}

cudaError_t launch_neumann_tc(const float* A, float* T, int64_t nc, int k, int N, int mask, int S,
                              cudaStream_t st) {
    if (k > 128) return cudaErrorNotSupported;
    tcg::Params p = tcg::base_params(nc, k);
    p.Ain = A;
    p.Tout = T;
    p.N = N;
    p.mask = mask;
    p.S = S;
    return GDN_TC_DISPATCH(k, tcg::kNeumann, 2, nullptr, nullptr, nullptr, nullptr, p, st);
}

cudaError_t launch_wy_tc(const float* T, const void* K, const void* V, const float* beta,
                         const float* g, void* W, void* U, int64_t nc, int k, cudaStream_t st) {
    if (k > 128) return cudaErrorNotSupported;
    tcg::Params p = tcg::base_params(nc, k);
    p.Tin = T;
    p.gated = g != nullptr;
    p.W = (__nv_bfloat16*)W;
    p.U = (__nv_bfloat16*)U;
    return GDN_TC_DISPATCH(k, tcg::kWY, 1, K, V, beta, g, p, st);
}

cudaError_t launch_neumann_i8_tc(const float*, float*, int, int, int8_t*, int32_t*, float*,
                                 int64_t, cudaStream_t) {
    return cudaErrorNotSupported;
}

cudaError_t launch_fused_tc(const void* K, const void* V, const float* beta, const float* g,
                            int N, int mask, int S, int gated, void* W, void* U, float* Tout,
                            int64_t nc, int k, cudaStream_t st) {
    if (k > 128) return cudaErrorNotSupported;
    tcg::Params p = tcg::base_params(nc, k);
    p.N = N;
    p.mask = mask;
    p.S = S;
    p.gated = gated;
    p.W = (__nv_bfloat16*)W;
    p.U = (__nv_bfloat16*)U;
    p.Tout = Tout;
    return GDN_TC_DISPATCH(k, tcg::kFused, 1, K, V, beta, g, p, st);
}

}  // namespace gdn
