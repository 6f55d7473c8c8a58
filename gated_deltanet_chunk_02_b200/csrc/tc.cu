// tc.cu — tcgen05 tensor-core kernels of libgdn (sm_100a).
//
// One persistent kernel template serves the bf16 chunk pipeline in four
// modes: the fused inverse + WY step, A alone, the Neumann inverse alone and
// WY alone.  Design:
//
// * A "tile" is 128 consecutive rows of the flattened [B*H*T, d] arrays, i.e.
//   128/KB blocks of KB tokens (KB = 64 or 128; chunks of k = 32 run as 64-token
//   blocks holding two chunks block-diagonally).  Every k x k product of the
//   method is ONE M=128 tcgen05.mma over the tile: the left operand stacks the
//   tile's blocks along M, the right operand places them side by side along N,
//   and each row reads only its own diagonal block of the 128 x 128 fp32
//   accumulator in tensor memory (TMEM).
// * Warp 0 is the TMA producer: K and V tiles (128-byte swizzle), beta and g.
//   Each "slot" of 8 warps owns one tile at a time; its elected thread issues
//   the tile's MMAs and TMA stores, and its 256 threads run the epilogues
//   (TMEM -> registers -> mask / accumulate / convert -> swizzled shared-memory
//   operand).  Thread (r, h) owns row r of the tile (its TMEM lane; the lane
//   quarter is warp % 4) and the column half h.  Two slots per CTA keep the
//   tensor pipe busy while the other slot runs an epilogue.
// * T0 (then T) stays in TMEM columns [128, 128 + KB) of the slot, next to the
//   product accumulator in columns [0, 128).
// * WY is computed transposed, W^T = K^T (T diag(beta))^T, a full-rate M=128
//   (= d) product; its epilogue transposes through the (now free) K/V tiles in
//   shared memory and leaves with TMA bulk stores.
// * Every wait is bounded (2 s).  On expiry the kernel sets the status word,
//   stops issuing work, waits (bounded) for its own copies and MMAs and frees
//   TMEM before returning.
#include <cuda.h>

#include "common.cuh"
#include "tc.h"

namespace gdn {
namespace tcg {

constexpr int kD = 128;
constexpr int kRows = 128;                       // rows per tile
constexpr unsigned long long kTimeoutNs = 2000000000ull;
constexpr int kStatusSmemAlign = 2;              // dynamic shared memory not 1024-aligned

enum Mode { kFused = 0, kBuildA = 1, kNeumann = 2, kWY = 3 };

__host__ __device__ constexpr bool uses_K(int m) { return m == kFused || m == kBuildA || m == kWY; }
__host__ __device__ constexpr bool uses_V(int m) { return m == kFused || m == kWY; }
__host__ __device__ constexpr int block_of(int kc) { return kc < 64 ? 64 : kc; }

// Per-slot shared-memory layout (bytes).  The 1024-byte aligned operand
// regions of all slots come first, then each slot's beta/g, then control.
template <int KB, int MODE>
struct SlotLayout {
    static constexpr int kK = uses_K(MODE) ? kRows * kD * 2 : 0;        // bf16 [2][128][64]
    static constexpr int kV = uses_V(MODE) ? kRows * kD * 2 : 0;
    static constexpr int kAop = (MODE == kFused || MODE == kNeumann) ? kRows * KB * 2 : 0;
    static constexpr int kXY = (MODE == kBuildA) ? 0 : kRows * KB * 2;  // 16-bit [KB/64][128][64]
    static constexpr int offK = 0;
    static constexpr int offV = offK + kK;
    static constexpr int offAop = offV + kV;
    static constexpr int offX = offAop + kAop;
    static constexpr int offY = offX + kXY;
    static constexpr int bytes = offY + kXY;
    static constexpr int bg_bytes = uses_K(MODE) ? 2 * kRows * 4 : 0;  // beta[128], g[128]
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

__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(b)) : "memory");
}
__device__ __forceinline__ void tma_load_1d(void* dst, const CUtensorMap* m, int x, uint64_t* b) {
    asm volatile(
        "cp.async.bulk.tensor.1d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2}], [%3];" ::"r"(su32(dst)), "l"(m), "r"(x), "r"(su32(b))
        : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, int x, int y, const void* src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(m),
                 "r"(x), "r"(y), "r"(su32(src))
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// 32 consecutive TMEM columns of this thread's lane -> 32 raw words, no wait.
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t (&r)[32]) {
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
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// two 32-column pieces (e.g. an accumulator piece and a T0 piece) with one wait
__device__ __forceinline__ void tmem_ld2(uint32_t a0, float (&v0)[32], uint32_t a1, float (&v1)[32]) {
    uint32_t r0[32], r1[32];
    tmem_ld32_async(a0, r0);
    tmem_ld32_async(a1, r1);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        v0[i] = __uint_as_float(r0[i]);
        v1[i] = __uint_as_float(r1[i]);
    }
}

struct Params {
    int64_t rows;        // B*H*T
    int ntiles;
    int N, mask, S, gated;
    const float* Ain;    // kNeumann
    const float* Tin;    // kWY
    float* Aout;         // kBuildA
    float* Tout;         // kFused (optional), kNeumann
    int* status;
};

struct __align__(8) Ctrl {
    uint64_t full[2];
    uint64_t kvfree[2];
    uint64_t mma[2];
    uint32_t tmem;
    int abort;
};

template <int KC, int MODE, int NS>
struct KernelShape {
    static constexpr int KB = block_of(KC);
    using L = SlotLayout<KB, MODE>;
    static constexpr int threads = 32 + 256 * NS;
    static constexpr int smem = NS * L::bytes + NS * L::bg_bytes + (int)sizeof(Ctrl);
};

// ------------------------------------------------------------------------- //
// the kernel
// ------------------------------------------------------------------------- //
template <int KC, int MODE, int NS>
__global__ void __launch_bounds__(32 + 256 * NS, 1)
k_chunk_tc(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
           const __grid_constant__ CUtensorMap mW, const __grid_constant__ CUtensorMap mU,
           const __grid_constant__ CUtensorMap mB, const __grid_constant__ CUtensorMap mG,
           const Params p) {
    constexpr int KB = block_of(KC);
    constexpr bool SUB = KC < KB;                  // two 32-token chunks per 64 block
    using L = SlotLayout<KB, MODE>;
    constexpr int NP = KB / 32;                    // 32-column pieces per block row
    constexpr int PPT = NP / 2;                    // pieces per thread (two threads per row)
    constexpr int NCH = kRows / KB;                // blocks per tile
    constexpr uint32_t kTmemCols = NS == 2 ? 512 : 256;

    extern __shared__ __align__(1024) uint8_t smem[];
    if ((su32(smem) & 1023u) != 0) {              // swizzled operands need 1024-byte alignment
        if (threadIdx.x == 0) raise_status(p.status, kStatusSmemAlign);
        return;
    }
    uint8_t* bg_base = smem + NS * L::bytes;
    Ctrl* ctrl = reinterpret_cast<Ctrl*>(bg_base + NS * L::bg_bytes);

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
                                        (uses_V(MODE) ? kRows * kD * 2 : 0) + 2 * kRows * 4;
            int issued[2] = {0, 0};
            for (int n = 0;; ++n) {
                const int tile = blockIdx.x + n * gridDim.x;
                if (tile >= p.ntiles) break;
                const int s = n % NS, use = n / NS;
                if (use > 0 && !mbar_wait(&ctrl->kvfree[s], (use - 1) & 1)) {
                    atomicExch(&ctrl->abort, 1);
                    raise_status(p.status, kStatusTimeout);
                    break;
                }
                if (*(volatile int*)&ctrl->abort) break;
                uint8_t* base = smem + s * L::bytes;
                float* bg = reinterpret_cast<float*>(bg_base + s * L::bg_bytes);
                const int y = tile * kRows;
                mbar_expect_tx(&ctrl->full[s], kBytes);
                tma_load_2d(base + L::offK, &mK, 0, y, &ctrl->full[s]);
                tma_load_2d(base + L::offK + kRows * 128, &mK, 64, y, &ctrl->full[s]);
                if (uses_V(MODE)) {
                    tma_load_2d(base + L::offV, &mV, 0, y, &ctrl->full[s]);
                    tma_load_2d(base + L::offV + kRows * 128, &mV, 64, y, &ctrl->full[s]);
                }
                tma_load_1d(bg, &mB, y, &ctrl->full[s]);
                tma_load_1d(bg + kRows, &mG, y, &ctrl->full[s]);
                issued[s] = use + 1;
            }
            // every copy this warp issued lands before the CTA exits
            for (int s = 0; s < NS; ++s)
                if (issued[s] > 0) mbar_wait(&ctrl->full[s], (issued[s] - 1) & 1);
        }
    } else {
        // ------------------------------ slot s ------------------------------
        const int s = (warp - 1) / 8;
        const int h = ((warp - 1) % 8) / 4;            // column half of the row
        const int r = ((warp & 3) << 5) | lane;       // tile row == TMEM lane
        const int blk = r / KB;                        // block of this row in the tile
        const int i = r % KB;                          // row inside the block
        const int cl = SUB ? (i / KC) * KC : 0;        // first column of this row's chunk
        const int ch = cl + KC;                        // one past its last column
        const int jmin = p.mask ? i - p.N : -KB;       // band mask keeps columns j >= jmin
        uint8_t* base = smem + s * L::bytes;
        uint8_t* sK = base + L::offK;
        uint8_t* sV = base + L::offV;
        uint8_t* sAop = base + L::offAop;
        uint8_t* sX = base + L::offX;
        uint8_t* sY = base + L::offY;
        const float* sb = reinterpret_cast<const float*>(bg_base + s * L::bg_bytes);
        const float* sg = sb + kRows;
        const uint32_t tm = tmem_base + (uint32_t)(s * 256);
        const uint32_t tl = tm + ((uint32_t)((warp & 3) * 32) << 16);   // this warp's lanes
        const uint32_t tD = tl + blk * KB;            // this row's diagonal block of D
        const uint32_t tT = tl + 128;                 // this row's T0 / T
        const bool leader = ((warp - 1) % 8) == 0 && lane == 0;
        const int bar_id = 1 + s;
        const int pc0 = h * PPT;
        uint32_t mma_phase = 0;
        bool ok = true;

        auto fail_wait = [&]() {
            atomicExch(&ctrl->abort, 1);
            raise_status(p.status, kStatusTimeout);
        };
        auto wait_mma = [&]() -> bool {
            bool good = mbar_wait(&ctrl->mma[s], mma_phase);
            mma_phase ^= 1;
            if (!good) fail_wait();
            tc_fence_after();
            return good;
        };
        // hand the operands written by this slot to the tensor pipe
        auto publish = [&]() {
            tmem_wait_st();
            fence_async_smem();
            tc_fence_before();
            bar_sync(bar_id, 256);
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
        auto in_chunk = [&](int j) { return SUB ? (j >= cl && j < ch) : true; };
        auto eye = [&](int j) { return i == j ? 1.f : 0.f; };

        for (int n = s;; n += NS) {
            const int tile = blockIdx.x + n * gridDim.x;
            if (tile >= p.ntiles) break;
            const int use = n / NS;
            const int64_t row0 = (int64_t)tile * kRows;
            const int64_t grow = row0 + r;
            const bool valid = grow < p.rows;
            const int64_t cidx = grow / KC;                  // chunk of this row
            const int64_t rin = grow % KC;                   // row inside the chunk
            if (uses_K(MODE) && !mbar_wait(&ctrl->full[s], use & 1)) fail_wait();
            bar_sync(bar_id, 256);
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
                }
                if (!wait_mma()) { ok = false; break; }
                const float bi = sb[r], gi = sg[r];
                const float* gcol = sg + blk * KB;
#pragma unroll
                for (int pp = 0; pp < PPT; ++pp) {
                    const int pc = pc0 + pp;
                    float v[32];
                    tmem_ld32(tD + pc * 32, v);
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int j = pc * 32 + jj;
                        const bool in = in_chunk(j) && j < i;
                        v[jj] = in ? -bi * v[jj] * expf(gi - gcol[j]) : 0.f;
                    }
                    if (MODE == kBuildA) {
                        if (valid && (!SUB || (pc * 32 >= cl && pc * 32 < ch))) {
                            float* dst = p.Aout + cidx * KC * KC + rin * KC + (pc * 32 - cl);
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
                            v[jj] = j >= jmin ? v[jj] : 0.f;
                            t[jj] = eye(j) + v[jj];
                        }
                        st_op32<false>(sAop, r, pc, v);           // P_1 = M . A
                        tmem_st32(tT + pc * 32, t);                // T0 = I + P_1
                    }
                }
                if (MODE == kBuildA) {
                    tc_fence_before();
                    bar_sync(bar_id, 256);                 // beta/g read, accumulator read
                    if (leader) mbar_arrive(&ctrl->kvfree[s]);
                    continue;
                }
            } else if (MODE == kNeumann) {
                // ---- A row from global memory ----
#pragma unroll
                for (int pp = 0; pp < PPT; ++pp) {
                    const int pc = pc0 + pp;
                    float v[32], t[32];
                    const bool have = valid && (!SUB || (pc * 32 >= cl && pc * 32 < ch));
                    if (have) {
                        const float4* src = reinterpret_cast<const float4*>(
                            p.Ain + cidx * KC * KC + rin * KC + (pc * 32 - cl));
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
                        v[jj] = j >= jmin ? v[jj] : 0.f;
                        t[jj] = eye(j) + v[jj];
                    }
                    st_op32<false>(sAop, r, pc, v);
                    tmem_st32(tT + pc * 32, t);
                }
            } else {
                // ---- kWY: T row from global memory ----
#pragma unroll
                for (int pp = 0; pp < PPT; ++pp) {
                    const int pc = pc0 + pp;
                    float t[32];
                    const bool have = valid && (!SUB || (pc * 32 >= cl && pc * 32 < ch));
                    if (have) {
                        const float4* src = reinterpret_cast<const float4*>(
                            p.Tin + cidx * KC * KC + rin * KC + (pc * 32 - cl));
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
#pragma unroll
                    for (int pp = 0; pp < PPT; ++pp) {
                        const int pc = pc0 + pp;
                        float v[32], t[32];
                        tmem_ld2(tD + pc * 32, v, tT + pc * 32, t);
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const int j = pc * 32 + jj;
                            v[jj] = (in_chunk(j) && j >= jmin) ? v[jj] : 0.f;
                            t[jj] += v[jj];
                        }
                        tmem_st32(tT + pc * 32, t);
                        if (pw < p.N) st_op32<false>(sAop, r, pc, v);
                    }
                }
                if (!ok) break;
                // ---- parallel residual correction ----
                if (p.S > 0) {
#pragma unroll
                    for (int pp = 0; pp < PPT; ++pp) {
                        const int pc = pc0 + pp;
                        float t[32];
                        tmem_ld32(tT + pc * 32, t);
                        st_op32<false>(sY, r, pc, t);                      // T0
                    }
                    publish();
                    mma_chain(sX, sY);                                      // A T0
                    if (!wait_mma()) { ok = false; break; }
#pragma unroll
                    for (int pp = 0; pp < PPT; ++pp) {
                        const int pc = pc0 + pp;
                        float v[32], t[32];
                        tmem_ld2(tD + pc * 32, v, tT + pc * 32, t);
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
#pragma unroll
                        for (int pp = 0; pp < PPT; ++pp) {
                            const int pc = pc0 + pp;
                            float v[32];
                            if (last) {
                                float t[32];
                                tmem_ld2(tD + pc * 32, v, tT + pc * 32, t);
#pragma unroll
                                for (int jj = 0; jj < 32; ++jj)
                                    if (!in_chunk(pc * 32 + jj)) v[jj] = 0.f;
                                st_op32<false>(sY, r, pc, v);               // Q_S
                                st_op32<false>(sAop, r, pc, t);             // T0
                            } else {
                                tmem_ld32(tD + pc * 32, v);
#pragma unroll
                                for (int jj = 0; jj < 32; ++jj) {
                                    const int j = pc * 32 + jj;
                                    v[jj] = in_chunk(j) ? v[jj] + eye(j) : 0.f;
                                }
                                st_op32<false>(sAop, r, pc, v);             // I + Q_{m+1}
                            }
                        }
                    }
                    if (!ok) break;
                    publish();
                    mma_chain(sAop, sY);                                    // T0 Q_S
                    if (!wait_mma()) { ok = false; break; }
#pragma unroll
                    for (int pp = 0; pp < PPT; ++pp) {
                        const int pc = pc0 + pp;
                        float v[32], t[32];
                        tmem_ld2(tD + pc * 32, v, tT + pc * 32, t);
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj)
                            if (in_chunk(pc * 32 + jj)) t[jj] += v[jj];     // T = T0 + T0 Q
                        tmem_st32(tT + pc * 32, t);
                    }
                }
                // ---- T out ----
                if (p.Tout) {
#pragma unroll
                    for (int pp = 0; pp < PPT; ++pp) {
                        const int pc = pc0 + pp;
                        float t[32];
                        tmem_ld32(tT + pc * 32, t);
                        if (valid && (!SUB || (pc * 32 >= cl && pc * 32 < ch))) {
                            float* dst = p.Tout + cidx * KC * KC + rin * KC + (pc * 32 - cl);
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
                const float* bcol = sb + blk * KB;
                const float* gcol = sg + blk * KB;
#pragma unroll
                for (int pp = 0; pp < PPT; ++pp) {
                    const int pc = pc0 + pp;
                    float t[32], v[32];
                    tmem_ld32(tT + pc * 32, t);
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int j = pc * 32 + jj;
                        const float b = bcol[j];
                        v[jj] = p.gated ? t[jj] * (b * expf(gcol[j])) : t[jj] * b;
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
                }
                if (!wait_mma()) { ok = false; break; }
                // Lane r of the W^T / U^T accumulators is head-dim column d = r and
                // accumulator column x is tile row x.  Thread half h transposes
                // rows [64h, 64h + 64) through the K (W) and V (U) tiles, which
                // the finished MMAs no longer read, in the TMA load layout.
                {
                    const int d = r;
                    const uint32_t dbase = (uint32_t)((d >> 6) * (kRows * 128) + (d & 7) * 2);
                    const int c16 = (d & 63) >> 3;
#pragma unroll
                    for (int pp = 0; pp < 2; ++pp) {
                        const int x0 = h * 64 + pp * 32;
                        float w[32], u[32];
                        tmem_ld2(tl + x0, w, tl + 128 + x0, u);
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const int x = x0 + jj;
                            const uint32_t off = dbase + x * 128 + ((c16 ^ (x & 7)) << 4);
                            *reinterpret_cast<__nv_bfloat16*>(sK + off) = __float2bfloat16_rn(w[jj]);
                            *reinterpret_cast<__nv_bfloat16*>(sV + off) = __float2bfloat16_rn(u[jj]);
                        }
                    }
                }
                fence_async_smem();
                tc_fence_before();
                bar_sync(bar_id, 256);
                if (leader) {
                    const int y = (int)row0;
                    tma_store_2d(&mW, 0, y, sK);
                    tma_store_2d(&mW, 64, y, sK + kRows * 128);
                    tma_store_2d(&mU, 0, y, sV);
                    tma_store_2d(&mU, 64, y, sV + kRows * 128);
                    bulk_commit();
                    bulk_wait_read();                       // tiles may be reloaded now
                    mbar_arrive(&ctrl->kvfree[s]);
                }
                continue;
            }
            tc_fence_before();
            bar_sync(bar_id, 256);                 // accumulators free for the next tile
        }
        if (!ok) {
            atomicExch(&ctrl->abort, 1);
            // outstanding MMAs of this slot finish before TMEM is released
            mbar_wait(&ctrl->mma[s], mma_phase);
        }
        if (leader) bulk_wait_all();               // W, U stores complete
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
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)ptr;
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

// [rows] fp32, box 128 (rows past the end read as zero)
static bool map_vec(CUtensorMap* m, const void* base, int64_t rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[1] = {(cuuint64_t)rows};
    cuuint64_t strides[1] = {4};
    cuuint32_t box[1] = {(cuuint32_t)kRows};
    cuuint32_t es[1] = {1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int num_sms() {
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

struct IO {
    const void* K = nullptr;
    const void* V = nullptr;
    const float* beta = nullptr;
    const float* g = nullptr;
    void* W = nullptr;
    void* U = nullptr;
};

template <int KC, int MODE, int NS>
static cudaError_t launch(const IO& io, const Params& p0, cudaStream_t st) {
    using KS = KernelShape<KC, MODE, NS>;
    static_assert(KS::smem <= 232448, "shared memory budget");
    CUtensorMap mK, mV, mW, mU, mB, mG;
    memset(&mK, 0, sizeof mK);
    memset(&mV, 0, sizeof mV);
    memset(&mW, 0, sizeof mW);
    memset(&mU, 0, sizeof mU);
    memset(&mB, 0, sizeof mB);
    memset(&mG, 0, sizeof mG);
    if (uses_K(MODE)) {
        if (!map_kd(&mK, io.K, p0.rows) || !map_vec(&mB, io.beta, p0.rows) ||
            !map_vec(&mG, io.g ? io.g : io.beta, p0.rows))
            return cudaErrorInvalidValue;
    }
    if (uses_V(MODE)) {
        if (!map_kd(&mV, io.V, p0.rows) || !map_kd(&mW, io.W, p0.rows) ||
            !map_kd(&mU, io.U, p0.rows))
            return cudaErrorInvalidValue;
    }
    Params p = p0;
    p.status = status_ptr();
    size_t smem = KS::smem;
    if (smem < 120 * 1024) smem = 120 * 1024;     // one CTA per SM: it owns the SM's TMEM
    cudaError_t e = cudaFuncSetAttribute(k_chunk_tc<KC, MODE, NS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = p.ntiles < num_sms() ? p.ntiles : num_sms();
    k_chunk_tc<KC, MODE, NS><<<grid, KS::threads, smem, st>>>(mK, mV, mW, mU, mB, mG, p);
    return cudaGetLastError();
}

static Params base_params(int64_t nc, int k) {
    Params p;
    memset(&p, 0, sizeof p);
    p.rows = nc * k;
    p.ntiles = (int)((p.rows + kRows - 1) / kRows);
    return p;
}

// chunk size -> kernel instance; NS128 = slots per CTA at k = 128
template <int MODE, int NS128>
static cudaError_t dispatch(int k, const IO& io, const Params& p, cudaStream_t st) {
    switch (k) {
        case 32: return launch<32, MODE, 2>(io, p, st);
        case 64: return launch<64, MODE, 2>(io, p, st);
        case 128: return launch<128, MODE, NS128>(io, p, st);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace tcg

bool tc_available() { return true; }
bool tc_i8_available() { return false; }

cudaError_t launch_build_A_tc(const void* K, const float* beta, const float* g, float* A,
                              int64_t nc, int k, cudaStream_t st) {
    tcg::Params p = tcg::base_params(nc, k);
    p.Aout = A;
    tcg::IO io;
    io.K = K;
    io.beta = beta;
    io.g = g;
    return tcg::dispatch<tcg::kBuildA, 2>(k, io, p, st);
}

cudaError_t launch_neumann_tc(const float* A, float* T, int64_t nc, int k, int N, int mask, int S,
                              cudaStream_t st) {
    tcg::Params p = tcg::base_params(nc, k);
    p.Ain = A;
    p.Tout = T;
    p.N = N;
    p.mask = mask;
    p.S = S;
    return tcg::dispatch<tcg::kNeumann, 2>(k, tcg::IO(), p, st);
}

cudaError_t launch_wy_tc(const float* T, const void* K, const void* V, const float* beta,
                         const float* g, void* W, void* U, int64_t nc, int k, cudaStream_t st) {
    tcg::Params p = tcg::base_params(nc, k);
    p.Tin = T;
    p.gated = g != nullptr;
    tcg::IO io;
    io.K = K;
    io.V = V;
    io.beta = beta;
    io.g = g;
    io.W = W;
    io.U = U;
    return tcg::dispatch<tcg::kWY, 1>(k, io, p, st);
}

cudaError_t launch_neumann_i8_tc(const float*, float*, int, int, int8_t*, int32_t*, float*,
                                 int64_t, cudaStream_t) {
    return cudaErrorNotSupported;
}

cudaError_t launch_fused_tc(const void* K, const void* V, const float* beta, const float* g,
                            int N, int mask, int S, int gated, void* W, void* U, float* Tout,
                            int64_t nc, int k, cudaStream_t st) {
    tcg::Params p = tcg::base_params(nc, k);
    p.N = N;
    p.mask = mask;
    p.S = S;
    p.gated = gated;
    p.Tout = Tout;
    tcg::IO io;
    io.K = K;
    io.V = V;
    io.beta = beta;
    io.g = g;
    io.W = W;
    io.U = U;
    return tcg::dispatch<tcg::kFused, 1>(k, io, p, st);
}

}  // namespace gdn
