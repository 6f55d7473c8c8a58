// decode.cu — decode steps of the gated delta rule (gdn_decode).
//
// "A Persistent-State Dataflow Accelerator for Memory-Bound Linear Attention
// Decode on FPGA" (technical summary, §1-§2): generating one token touches the
// whole d_v x d_k state of every value head, so the step is bound by moving
// that state; the summary's rewrite needs one read and one write of the state
// per token, and the value heads of a group share one query and one key.
// The rewrite used here: with u = S k and p = S q (the read pass),
//   v~ = b (v - a u),   S' = a S + v~ k^T (the write pass),   o = a p + v~ (k . q),
// which equals S' = a S (I - b k k^T) + b v k^T and o = S' q.
//
// GPU mapping.  Rows of the state never mix: row i of S' needs row i of S, the
// key and v_i only.  Eight lanes share a row, lane j holding its columns
// 32c + 4j .. 32c + 4j + 3 (c < 4; each load instruction of the 8 lanes covers
// 128 contiguous bytes) in registers for all n tokens of a call, so the state crosses HBM once per
// call (the summary's state kept on chip) rather than once per token, and the
// row sums u_i, p_i and k . q take three shuffle levels.  A warp holds 4 x R
// rows, a CTA of 4 warps 16 R rows; R = 2 (4 CTAs per value head) when the
// grid fills the GPU, R = 1 otherwise.  Grid = (Hv * 128 / (16 R), B).
// Token t + 1's vectors load while token t computes.
#include "common.cuh"
#include "kernels.h"

namespace gdn {
namespace {

constexpr int kDh = 128;                               // head dim (d_k = d_v)
constexpr int kDecWarps = 4;
constexpr int kSeg = 16;                               // columns per lane

// this lane's 16 columns (4 groups of 4, 32 apart) as floats; p points at
// column 4j of the row
__device__ __forceinline__ void ld16(const float* p, float (&x)[kSeg]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float4 f = __ldg(reinterpret_cast<const float4*>(p + 32 * c));
        x[4 * c] = f.x; x[4 * c + 1] = f.y; x[4 * c + 2] = f.z; x[4 * c + 3] = f.w;
    }
}
__device__ __forceinline__ void ld16(const __nv_bfloat16* p, float (&x)[kSeg]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(p + 32 * c));
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        x[4 * c] = a.x; x[4 * c + 1] = a.y; x[4 * c + 2] = b.x; x[4 * c + 3] = b.y;
    }
}
// sum over the 8 lanes of a row group
__device__ __forceinline__ float row_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x;
}

template <typename T, int R>
__global__ void __launch_bounds__(kDecWarps * 32)
k_decode(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
         const float* __restrict__ beta, const float* __restrict__ loggate, float* S, T* O,
         int Hk, int Hv, int n) {
    constexpr int kCtaRows = kDecWarps * 4 * R;
    constexpr int kGroups = kDh / kCtaRows;            // CTAs per value head
    const int b = blockIdx.y;
    const int hv = blockIdx.x / kGroups;
    const int hk = hv / (Hv / Hk);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane & 7;                          // columns 32c + 4 sub + (0..3)
    // this thread's rows: row0 + r, r < R
    const int row0 = (blockIdx.x % kGroups) * kCtaRows + warp * 4 * R + (lane >> 3) * R;
    const int64_t bh = (int64_t)b * Hv + hv;
    const int64_t bk = (int64_t)b * Hk + hk;

    float* Sh = S + bh * kDh * kDh + (int64_t)row0 * kDh + 4 * sub;
    float s[R][kSeg];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float4 f = *reinterpret_cast<const float4*>(Sh + r * kDh + 32 * c);
            s[r][4 * c] = f.x; s[r][4 * c + 1] = f.y; s[r][4 * c + 2] = f.z; s[r][4 * c + 3] = f.w;
        }

    const T* qp = Q + bk * n * kDh + 4 * sub;
    const T* kp = K + bk * n * kDh + 4 * sub;
    const T* vp = V + bh * n * kDh + row0;
    T* op = O + bh * n * kDh + row0;
    const float* bp = beta + bh * n;
    const float* gp = loggate + bh * n;

    float kn[kSeg], qn[kSeg], vn[R];
    ld16(kp, kn);
    ld16(qp, qn);
#pragma unroll
    for (int r = 0; r < R; ++r) vn[r] = ld_elem(vp, r);
    float bn = __ldg(bp), gn = __ldg(gp);
    for (int t = 0; t < n; ++t) {
        float k[kSeg], q[kSeg], v[R];
#pragma unroll
        for (int c = 0; c < kSeg; ++c) { k[c] = kn[c]; q[c] = qn[c]; }
#pragma unroll
        for (int r = 0; r < R; ++r) v[r] = vn[r];
        const float bt = bn, a = expf(gn);
        if (t + 1 < n) {                                   // next token's inputs
            const int64_t o1 = (int64_t)(t + 1) * kDh;
            ld16(kp + o1, kn);
            ld16(qp + o1, qn);
#pragma unroll
            for (int r = 0; r < R; ++r) vn[r] = ld_elem(vp, o1 + r);
            bn = __ldg(bp + t + 1);
            gn = __ldg(gp + t + 1);
        }
        float kq = 0.f, u[R], p[R];
#pragma unroll
        for (int r = 0; r < R; ++r) { u[r] = 0.f; p[r] = 0.f; }
#pragma unroll
        for (int c = 0; c < kSeg; ++c) {
            kq += k[c] * q[c];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                u[r] += s[r][c] * k[c];
                p[r] += s[r][c] * q[c];
            }
        }
        kq = row_sum(kq);
#pragma unroll
        for (int r = 0; r < R; ++r) {
            u[r] = row_sum(u[r]);
            p[r] = row_sum(p[r]);
            const float dv = bt * (v[r] - a * u[r]);                   // v~
#pragma unroll
            for (int c = 0; c < kSeg; ++c) s[r][c] = a * s[r][c] + dv * k[c];
            if (sub == r) st_elem(op, (int64_t)t * kDh + r, a * p[r] + dv * kq);
        }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c)
            *reinterpret_cast<float4*>(Sh + r * kDh + 32 * c) =
                make_float4(s[r][4 * c], s[r][4 * c + 1], s[r][4 * c + 2], s[r][4 * c + 3]);
}

template <typename T, int R>
void run_decode(const void* Q, const void* K, const void* V, const float* beta,
                const float* loggate, float* S, void* O, int64_t B, int64_t Hk, int64_t Hv,
                int64_t n, cudaStream_t st) {
    constexpr int kGroups = kDh / (kDecWarps * 4 * R);
    const dim3 grid((unsigned)(Hv * kGroups), (unsigned)B);
    k_decode<T, R><<<grid, kDecWarps * 32, 0, st>>>(
        static_cast<const T*>(Q), static_cast<const T*>(K), static_cast<const T*>(V), beta,
        loggate, S, static_cast<T*>(O), (int)Hk, (int)Hv, (int)n);
}

}  // namespace

cudaError_t launch_decode(const void* Q, const void* K, const void* V, const float* beta,
                          const float* loggate, float* S, void* O, int64_t B, int64_t Hk,
                          int64_t Hv, int64_t n, bool bf16, cudaStream_t st) {
    static int sms_of[64] = {0};                       // SM count per device, looked up once
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
        if (!sms_of[dev]) cudaDeviceGetAttribute(&sms_of[dev], cudaDevAttrMultiProcessorCount, dev);
        if (sms_of[dev] > 0) sms = sms_of[dev];
    }
    const bool wide = B * Hv * 4 >= 2LL * sms;        // 4 CTAs per head fill the GPU
    if (bf16) {
        if (wide) run_decode<__nv_bfloat16, 2>(Q, K, V, beta, loggate, S, O, B, Hk, Hv, n, st);
        else run_decode<__nv_bfloat16, 1>(Q, K, V, beta, loggate, S, O, B, Hk, Hv, n, st);
    } else {
        if (wide) run_decode<float, 2>(Q, K, V, beta, loggate, S, O, B, Hk, Hv, n, st);
        else run_decode<float, 1>(Q, K, V, beta, loggate, S, O, B, Hk, Hv, n, st);
    }
    return cudaGetLastError();
}

}  // namespace gdn
