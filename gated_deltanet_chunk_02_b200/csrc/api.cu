// api.cu — the C ABI of libgdn: argument checks, dispatch, status word.
//
// Every entry point validates its arguments on the host before launching
// anything; on failure it returns a negative code, launches nothing and keeps
// a message for gdn_last_error().  Kernels report device-side failures by
// OR-ing bits into a per-device status word (never by trapping).
#include <cstdio>
#include <cstdarg>
#include <string>

#include "../../include/gdn.h"
#include "common.cuh"
#include "kernels.h"
#include "tc.h"

namespace gdn {
__device__ int g_status = 0;
}  // namespace gdn

namespace {

thread_local std::string t_last_error;
thread_local int64_t t_launches = 0;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(GDN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by all entry points; *nc receives the chunk count.
int check_shape(const gdn_shape& s, int64_t* nc) {
    if (s.B < 0 || s.H < 0 || s.T < 0) return fail(GDN_ERR_ARG, "negative B, H or T");
    if (s.k != 32 && s.k != 64 && s.k != 128 && s.k != 256)
        return fail(GDN_ERR_ARG, "chunk size k=%d not in {32, 64, 128, 256}", s.k);
    if (s.T % s.k) return fail(GDN_ERR_ARG, "T=%lld is not a multiple of k=%d", (long long)s.T, s.k);
    if (s.d != 128) return fail(GDN_ERR_UNSUPPORTED, "head dim d=%d (only 128 is built)", s.d);
    // each factor is below 2^31, so the products below cannot overflow int64
    if (s.B > 0x7fffffffLL || s.H > 0x7fffffffLL || s.T / s.k > 0x7fffffffLL)
        return fail(GDN_ERR_ARG, "too many chunks (B=%lld, H=%lld, T/k=%lld)", (long long)s.B,
                    (long long)s.H, (long long)(s.T / s.k));
    const int64_t bh = s.B * s.H;
    if (bh > 0x7fffffffLL) return fail(GDN_ERR_ARG, "too many chunks (B*H=%lld)", (long long)bh);
    const int64_t n = bh * (s.T / s.k);
    if (n > 0x7fffffffLL) return fail(GDN_ERR_ARG, "too many chunks (%lld)", (long long)n);
    *nc = n;
    return GDN_OK;
}

int check_ptrs(std::initializer_list<std::pair<const void*, const char*>> ps) {
    for (auto& p : ps) {
        if (!p.first) return fail(GDN_ERR_ARG, "%s is NULL", p.second);
        if (!aligned16(p.first)) return fail(GDN_ERR_ALIGN, "%s is not 16-byte aligned", p.second);
    }
    return GDN_OK;
}

int check_opt_ptr(const void* p, const char* name) {
    if (p && !aligned16(p)) return fail(GDN_ERR_ALIGN, "%s is not 16-byte aligned", name);
    return GDN_OK;
}

int check_dtype(gdn_dtype dt) {
    if (dt != GDN_F32 && dt != GDN_BF16) return fail(GDN_ERR_ARG, "unknown dtype %d", (int)dt);
    return GDN_OK;
}

int check_NS(int N, int mask, int S, int k) {
    if (N < 1 || N > k - 1) return fail(GDN_ERR_ARG, "Neumann order N=%d outside [1, k-1]", N);
    if (mask != 0 && mask != 1) return fail(GDN_ERR_ARG, "mask must be 0 or 1");
    if (S < 0 || S > 64) return fail(GDN_ERR_ARG, "residual steps S=%d outside [0, 64]", S);
    return GDN_OK;
}

int launched(cudaError_t e, const char* what) {
    if (e != cudaSuccess) return cuda_fail(e, what);
    ++t_launches;
    return GDN_OK;
}

}  // namespace

#define GDN_TRY(x)                  \
    do {                            \
        int _rc = (x);              \
        if (_rc != GDN_OK) return _rc; \
    } while (0)

extern "C" {

int gdn_build_A(const void* K, const float* beta, const float* g, float* A, gdn_shape s,
                gdn_dtype dtype, void* stream) {
    int64_t nc;
    GDN_TRY(check_shape(s, &nc));
    GDN_TRY(check_dtype(dtype));
    if (nc == 0) return GDN_OK;
    GDN_TRY(check_ptrs({{K, "K"}, {beta, "beta"}, {g, "g"}, {A, "A"}}));
    cudaStream_t st = (cudaStream_t)stream;
    if (dtype == GDN_BF16 && gdn::tc_available() && s.k <= 128)
        return launched(gdn::launch_build_A_tc(K, beta, g, A, nc, s.k, st), "build_A (tcgen05)");
    if (dtype == GDN_BF16 && gdn::tc_available() && s.k == 256)
        return launched(gdn::launch_build_A256_tc(K, beta, g, A, nc, st), "build_A k=256 (tcgen05)");
    return launched(gdn::launch_build_A_simt(K, beta, g, A, nc, s.k, dtype == GDN_BF16, st),
                    "build_A");
}

int gdn_invert_neumann(const float* A, float* T, gdn_shape s, int N, int mask, int S,
                       gdn_prec prec, void* stream) {
    int64_t nc;
    GDN_TRY(check_shape(s, &nc));
    GDN_TRY(check_NS(N, mask, S, s.k));
    if (prec != GDN_PREC_F32 && prec != GDN_PREC_F16) return fail(GDN_ERR_ARG, "unknown precision");
    if (nc == 0) return GDN_OK;
    GDN_TRY(check_ptrs({{A, "A"}, {T, "T"}}));
    cudaStream_t st = (cudaStream_t)stream;
    if (prec == GDN_PREC_F16) {
        if (!gdn::tc_available()) return fail(GDN_ERR_UNSUPPORTED, "tensor-core path not built");
        if (s.k == 256)
            return launched(gdn::launch_neumann256_tc(A, T, nc, N, mask, S, st),
                            "neumann k=256 (tcgen05)");
        return launched(gdn::launch_neumann_tc(A, T, nc, s.k, N, mask, S, st), "neumann (tcgen05)");
    }
    if (s.k > 128) return fail(GDN_ERR_UNSUPPORTED, "float32 Neumann chain supports k <= 128");
    return launched(gdn::launch_neumann_simt(A, T, nc, s.k, N, mask, S, st), "neumann");
}

int gdn_invert_newton(const float* A, float* T, gdn_shape s, int N, int mask, int M,
                      void* stream) {
    int64_t nc;
    GDN_TRY(check_shape(s, &nc));
    GDN_TRY(check_NS(N, mask, 0, s.k));
    if (M < 0 || M > 6) return fail(GDN_ERR_ARG, "correction steps M=%d outside [0, 6]", M);
    if (s.k == 256) return fail(GDN_ERR_UNSUPPORTED, "sequential correction supports k <= 128");
    if (nc == 0) return GDN_OK;
    GDN_TRY(check_ptrs({{A, "A"}, {T, "T"}}));
    if (!gdn::tc_available()) return fail(GDN_ERR_UNSUPPORTED, "tensor-core path not built");
    return launched(gdn::launch_newton_tc(A, T, nc, s.k, N, mask, M, (cudaStream_t)stream),
                    "newton (tcgen05)");
}

int gdn_invert_blocked(const float* A, float* T, gdn_shape s, void* stream) {
    int64_t nc;
    GDN_TRY(check_shape(s, &nc));
    if (s.k > 64) return fail(GDN_ERR_UNSUPPORTED, "the block-decomposition inverse supports k <= 64");
    if (nc == 0) return GDN_OK;
    GDN_TRY(check_ptrs({{A, "A"}, {T, "T"}}));
    if (!gdn::tc_available()) return fail(GDN_ERR_UNSUPPORTED, "tensor-core path not built");
    return launched(gdn::launch_blockinv_tc(A, T, nc, s.k, (cudaStream_t)stream),
                    "blocked inverse (tcgen05)");
}

int gdn_invert_fwdsub(const float* A, float* T, gdn_shape s, void* stream) {
    int64_t nc;
    GDN_TRY(check_shape(s, &nc));
    if (nc == 0) return GDN_OK;
    GDN_TRY(check_ptrs({{A, "A"}, {T, "T"}}));
    return launched(gdn::launch_fwdsub(A, T, nc, s.k, (cudaStream_t)stream), "fwdsub");
}

int gdn_wy(const float* T, const void* K, const void* V, const float* beta, const float* g,
           void* W, void* U, gdn_shape s, gdn_dtype dtype, void* stream) {
    int64_t nc;
    GDN_TRY(check_shape(s, &nc));
    GDN_TRY(check_dtype(dtype));
    if (nc == 0) return GDN_OK;
    GDN_TRY(check_ptrs({{T, "T"}, {K, "K"}, {V, "V"}, {beta, "beta"}, {W, "W"}, {U, "U"}}));
    GDN_TRY(check_opt_ptr(g, "g"));
    cudaStream_t st = (cudaStream_t)stream;
    if (s.k > 128) return fail(GDN_ERR_UNSUPPORTED, "wy serves k <= 128");
    if (dtype == GDN_BF16 && gdn::tc_available())
        return launched(gdn::launch_wy_tc(T, K, V, beta, g, W, U, nc, s.k, st), "wy (tcgen05)");
    return launched(gdn::launch_wy_simt(T, K, V, beta, g, W, U, nc, s.k, dtype == GDN_BF16, st),
                    "wy");
}

int gdn_invert_neumann_i8(const float* A, float* T, int N, int mask, int8_t* q_dbg,
                          int32_t* acc_dbg, float* scale_dbg, gdn_shape s, void* stream) {
    int64_t nc;
    GDN_TRY(check_shape(s, &nc));
    if (s.k != 64) return fail(GDN_ERR_UNSUPPORTED, "INT8 path is built for k=64");
    if (N < 1 || N > 8) return fail(GDN_ERR_ARG, "INT8 path: N=%d outside [1, 8]", N);
    if (mask != 0 && mask != 1) return fail(GDN_ERR_ARG, "mask must be 0 or 1");
    if (nc == 0) return GDN_OK;
    GDN_TRY(check_ptrs({{A, "A"}, {T, "T"}}));
    GDN_TRY(check_opt_ptr(q_dbg, "q_dbg"));
    GDN_TRY(check_opt_ptr(acc_dbg, "acc_dbg"));
    GDN_TRY(check_opt_ptr(scale_dbg, "scale_dbg"));
    cudaStream_t st = (cudaStream_t)stream;
    if (gdn::tc_i8_available())
        return launched(gdn::launch_neumann_i8_tc(A, T, N, mask, q_dbg, acc_dbg, scale_dbg, nc, st),
                        "neumann_i8 (tcgen05)");
    return launched(gdn::launch_neumann_i8_simt(A, T, N, mask, q_dbg, acc_dbg, scale_dbg, nc, st),
                    "neumann_i8");
}

int gdn_invert_neumann_i8_residual(const float* A, float* T, int N, int mask, int S,
                                   gdn_shape s, void* stream) {
    int64_t nc;
    GDN_TRY(check_shape(s, &nc));
    if (s.k != 64) return fail(GDN_ERR_UNSUPPORTED, "INT8 path is built for k=64");
    if (N < 1 || N > 8) return fail(GDN_ERR_ARG, "INT8 path: N=%d outside [1, 8]", N);
    if (mask != 0 && mask != 1) return fail(GDN_ERR_ARG, "mask must be 0 or 1");
    if (S < 1 || S > 64) return fail(GDN_ERR_ARG, "residual steps S=%d outside [1, 64]", S);
    if (nc == 0) return GDN_OK;
    GDN_TRY(check_ptrs({{A, "A"}, {T, "T"}}));
    if (!gdn::tc_i8_available()) return fail(GDN_ERR_UNSUPPORTED, "integer tensor-core path not built");
    return launched(gdn::launch_neumann_i8_tc(A, T, N, mask, nullptr, nullptr, nullptr, nc,
                                              (cudaStream_t)stream, S),
                    "neumann_i8 with residual (tcgen05)");
}

int gdn_invert_neumann_i16(const float* A, float* T, int N, int mask, int16_t* q_dbg,
                           int64_t* acc_dbg, double* scale_dbg, gdn_shape s, void* stream) {
    int64_t nc;
    GDN_TRY(check_shape(s, &nc));
    if (s.k != 64) return fail(GDN_ERR_UNSUPPORTED, "the INT16 path is built for k = 64");
    if (N < 1 || N > 8) return fail(GDN_ERR_ARG, "INT16 Neumann order N=%d outside [1, 8]", N);
    if (mask != 0 && mask != 1) return fail(GDN_ERR_ARG, "mask must be 0 or 1");
    if (nc == 0) return GDN_OK;
    GDN_TRY(check_ptrs({{A, "A"}, {T, "T"}}));
    GDN_TRY(check_opt_ptr(q_dbg, "q"));
    GDN_TRY(check_opt_ptr(acc_dbg, "acc"));
    GDN_TRY(check_opt_ptr(scale_dbg, "scale"));
    if (!gdn::tc_i8_available()) return fail(GDN_ERR_UNSUPPORTED, "integer tensor-core path not built");
    return launched(gdn::launch_neumann_i16_tc(A, T, N, mask, q_dbg, acc_dbg, scale_dbg, nc,
                                               (cudaStream_t)stream),
                    "neumann int16 (tcgen05)");
}

int gdn_invert_neumann_i16_residual(const float* A, float* T, int N, int mask, int S,
                                    gdn_shape s, void* stream) {
    int64_t nc;
    GDN_TRY(check_shape(s, &nc));
    if (s.k != 64) return fail(GDN_ERR_UNSUPPORTED, "the INT16 path is built for k = 64");
    if (N < 1 || N > 8) return fail(GDN_ERR_ARG, "INT16 Neumann order N=%d outside [1, 8]", N);
    if (mask != 0 && mask != 1) return fail(GDN_ERR_ARG, "mask must be 0 or 1");
    if (S < 1 || S > 64) return fail(GDN_ERR_ARG, "residual steps S=%d outside [1, 64]", S);
    if (nc == 0) return GDN_OK;
    GDN_TRY(check_ptrs({{A, "A"}, {T, "T"}}));
    if (!gdn::tc_i8_available()) return fail(GDN_ERR_UNSUPPORTED, "integer tensor-core path not built");
    return launched(gdn::launch_neumann_i16_tc(A, T, N, mask, nullptr, nullptr, nullptr, nc,
                                               (cudaStream_t)stream, S),
                    "neumann int16 with residual (tcgen05)");
}

int gdn_chunk_wy_fused(const void* K, const void* V, const float* beta, const float* g, int N,
                       int mask, int S, int gated, void* W, void* U, float* T_out, gdn_shape s,
                       gdn_dtype dtype, void* stream) {
    int64_t nc;
    GDN_TRY(check_shape(s, &nc));
    GDN_TRY(check_dtype(dtype));
    GDN_TRY(check_NS(N, mask, S, s.k));
    if (gated != 0 && gated != 1) return fail(GDN_ERR_ARG, "gated must be 0 or 1");
    if (nc == 0) return GDN_OK;
    GDN_TRY(check_ptrs({{K, "K"}, {V, "V"}, {beta, "beta"}, {g, "g"}, {W, "W"}, {U, "U"}}));
    GDN_TRY(check_opt_ptr(T_out, "T_out"));
    cudaStream_t st = (cudaStream_t)stream;
    if (dtype == GDN_BF16 && gdn::tc_available()) {
        if (s.k > 128) return fail(GDN_ERR_UNSUPPORTED, "fused tensor-core path serves k <= 128");
        return launched(gdn::launch_fused_tc(K, V, beta, g, N, mask, S, gated, W, U, T_out, nc,
                                             s.k, st),
                        "chunk_wy_fused (tcgen05)");
    }
    if (s.k > 128) return fail(GDN_ERR_UNSUPPORTED, "fused CUDA-core path supports k <= 128");
    return launched(gdn::launch_fused_simt(K, V, beta, g, N, mask, S, gated, W, U, T_out, nc,
                                           s.k, dtype == GDN_BF16, st),
                    "chunk_wy_fused");
}

int gdn_chunk_wy_fused_raw(const void* K_raw, const void* V, const float* beta,
                           const float* loggate, int N, int mask, int S, int gated, void* W,
                           void* U, float* T_out, void* K_out, float* g_out, gdn_shape s,
                           gdn_dtype dtype, void* stream) {
    int64_t nc;
    GDN_TRY(check_shape(s, &nc));
    GDN_TRY(check_dtype(dtype));
    GDN_TRY(check_NS(N, mask, S, s.k));
    if (dtype != GDN_BF16) return fail(GDN_ERR_UNSUPPORTED, "the prologue is built for bf16 data");
    if (s.k == 256) return fail(GDN_ERR_UNSUPPORTED, "the fused step supports k <= 128");
    if (nc == 0) return GDN_OK;
    GDN_TRY(check_ptrs({{K_raw, "K_raw"}, {V, "V"}, {beta, "beta"}, {loggate, "loggate"},
                        {W, "W"}, {U, "U"}}));
    GDN_TRY(check_opt_ptr(T_out, "T_out"));
    GDN_TRY(check_opt_ptr(K_out, "K_out"));
    GDN_TRY(check_opt_ptr(g_out, "g_out"));
    if (!gdn::tc_available()) return fail(GDN_ERR_UNSUPPORTED, "tensor-core path not built");
    return launched(gdn::launch_fused_raw_tc(K_raw, V, beta, loggate, N, mask, S, gated, W, U,
                                             T_out, K_out, g_out, nc, s.k, (cudaStream_t)stream),
                    "fused with prologue (tcgen05)");
}

int64_t gdn_forward_workspace_bytes(gdn_shape s, gdn_dtype dtype) {
    int64_t nc;
    if (check_shape(s, &nc) != GDN_OK) return -1;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return -1;
    const int64_t elem = dtype == GDN_BF16 ? 2 : 4;
    const int64_t rows = nc * s.k;
    // W_g and U for every chunk, then A and T (exact path)
    return 2 * rows * s.d * elem + 2 * nc * (int64_t)s.k * s.k * 4;
}

int gdn_forward(const void* Q, const void* K, const void* V, const float* beta, const float* g,
                const float* S0, int N, int mask, int S, int exact, void* O, float* S_final,
                void* workspace, int64_t workspace_bytes, gdn_shape s, gdn_dtype dtype,
                void* stream) {
    int64_t nc;
    GDN_TRY(check_shape(s, &nc));
    GDN_TRY(check_dtype(dtype));
    if (s.k != 64) return fail(GDN_ERR_UNSUPPORTED, "gdn_forward is built for k=64");
    if (exact != 0 && exact != 1) return fail(GDN_ERR_ARG, "exact must be 0 or 1");
    if (!exact) GDN_TRY(check_NS(N, mask, S, s.k));
    if (nc == 0) return GDN_OK;
    GDN_TRY(check_ptrs({{Q, "Q"}, {K, "K"}, {V, "V"}, {beta, "beta"}, {g, "g"}, {O, "O"},
                        {S_final, "S_final"}, {workspace, "workspace"}}));
    GDN_TRY(check_opt_ptr(S0, "S0"));
    const int64_t need = gdn_forward_workspace_bytes(s, dtype);
    if (workspace_bytes < need)
        return fail(GDN_ERR_ARG, "workspace of %lld bytes is below the %lld needed",
                    (long long)workspace_bytes, (long long)need);
    cudaStream_t st = (cudaStream_t)stream;
    const bool bf16 = dtype == GDN_BF16;
    const int64_t elem = bf16 ? 2 : 4;
    const int64_t rows = nc * s.k;
    uint8_t* ws = (uint8_t*)workspace;
    void* Wg = ws;
    void* U = ws + rows * s.d * elem;
    float* Abuf = (float*)(ws + 2 * rows * s.d * elem);
    float* Tbuf = Abuf + nc * (int64_t)s.k * s.k;
    if (exact) {
        GDN_TRY(gdn_build_A(K, beta, g, Abuf, s, dtype, stream));
        GDN_TRY(gdn_invert_fwdsub(Abuf, Tbuf, s, stream));
        GDN_TRY(gdn_wy(Tbuf, K, V, beta, g, Wg, U, s, dtype, stream));
    } else {
        GDN_TRY(gdn_chunk_wy_fused(K, V, beta, g, N, mask, S, 1, Wg, U, nullptr, s, dtype,
                                   stream));
    }
    // the A / T region (2 k^2 f32 per chunk = d^2 fp16 at k = 64) takes the
    // chunks' start states of the bf16 scan
    return launched(gdn::launch_scan(Q, K, Wg, U, g, S0, O, S_final, Abuf, s.B * s.H, s.T / s.k,
                                     bf16, st),
                    "forward scan");
}

int64_t gdn_forward_raw_workspace_bytes(gdn_shape s, gdn_dtype dtype) {
    int64_t nc;
    if (check_shape(s, &nc) != GDN_OK || dtype != GDN_BF16) return -1;
    const int64_t rows = nc * s.k;
    // gdn_forward's scratch, then the normalised keys (bf16) and the summed gates
    return gdn_forward_workspace_bytes(s, dtype) + rows * s.d * 2 + rows * 4;
}

int gdn_forward_raw(const void* Q_raw, const void* K_raw, const void* V, const float* beta,
                    const float* loggate, const float* S0, int N, int mask, int S, void* O,
                    float* S_final, void* workspace, int64_t workspace_bytes, gdn_shape s,
                    gdn_dtype dtype, void* stream) {
    int64_t nc;
    GDN_TRY(check_shape(s, &nc));
    GDN_TRY(check_dtype(dtype));
    if (dtype != GDN_BF16) return fail(GDN_ERR_UNSUPPORTED, "gdn_forward_raw is built for bf16 data");
    if (s.k != 64) return fail(GDN_ERR_UNSUPPORTED, "gdn_forward_raw is built for k=64");
    GDN_TRY(check_NS(N, mask, S, s.k));
    if (nc == 0) return GDN_OK;
    GDN_TRY(check_ptrs({{Q_raw, "Q_raw"}, {K_raw, "K_raw"}, {V, "V"}, {beta, "beta"},
                        {loggate, "loggate"}, {O, "O"}, {S_final, "S_final"},
                        {workspace, "workspace"}}));
    GDN_TRY(check_opt_ptr(S0, "S0"));
    if (!gdn::tc_available()) return fail(GDN_ERR_UNSUPPORTED, "tensor-core path not built");
    const int64_t need = gdn_forward_raw_workspace_bytes(s, dtype);
    if (workspace_bytes < need)
        return fail(GDN_ERR_ARG, "workspace of %lld bytes is below the %lld needed",
                    (long long)workspace_bytes, (long long)need);
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t rows = nc * s.k;
    uint8_t* ws = (uint8_t*)workspace;
    void* Wg = ws;
    void* U = ws + rows * s.d * 2;
    float* Sstates = (float*)(ws + 2 * rows * s.d * 2);
    uint8_t* tail = ws + gdn_forward_workspace_bytes(s, dtype);
    void* Kn = tail;                                    // the normalised keys
    float* gsum = (float*)(tail + rows * s.d * 2);      // the chunk-local cumulative gates
    GDN_TRY(gdn_chunk_wy_fused_raw(K_raw, V, beta, loggate, N, mask, S, 1, Wg, U, nullptr, Kn,
                                   gsum, s, dtype, stream));
    return launched(gdn::launch_scan(Q_raw, Kn, Wg, U, gsum, S0, O, S_final, Sstates, s.B * s.H,
                                     s.T / s.k, true, st, true),
                    "forward scan (raw queries)");
}

int gdn_decode(const void* Q, const void* K, const void* V, const float* beta,
               const float* loggate, float* S, void* O, int64_t B, int64_t Hk, int64_t Hv,
               int64_t n, int32_t d, gdn_dtype dtype, void* stream) {
    GDN_TRY(check_dtype(dtype));
    if (B < 0 || Hk < 0 || Hv < 0 || n < 0) return fail(GDN_ERR_ARG, "negative B, Hk, Hv or n");
    if (d != 128) return fail(GDN_ERR_UNSUPPORTED, "head dim d=%d (only 128 is built)", d);
    if (B == 0 || Hv == 0 || n == 0) return GDN_OK;
    if (Hk == 0 || Hv % Hk)
        return fail(GDN_ERR_ARG, "Hv=%lld is not a multiple of Hk=%lld", (long long)Hv,
                    (long long)Hk);
    if (B > 65535 || Hv > (1LL << 28) || n > 0x7fffffffLL)
        return fail(GDN_ERR_ARG, "B, Hv or n too large");
    GDN_TRY(check_ptrs({{Q, "Q"}, {K, "K"}, {V, "V"}, {beta, "beta"}, {loggate, "loggate"},
                        {S, "S"}, {O, "O"}}));
    return launched(gdn::launch_decode(Q, K, V, beta, loggate, S, O, B, Hk, Hv, n,
                                       dtype == GDN_BF16, (cudaStream_t)stream),
                    "decode");
}

int gdn_get_status(void* stream) {
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronise");
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, gdn::g_status, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "read status");
    const int z = 0;
    e = cudaMemcpyToSymbol(gdn::g_status, &z, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clear status");
    if (v & gdn::kStatusTimeout) return fail(GDN_ERR_TIMEOUT, "a bounded device wait ran out");
    if (v) return fail(GDN_ERR_CUDA, "device status bits 0x%x", v);
    return GDN_OK;
}

int gdn_debug_arm_wait_expiry(int tile, int load, double timeout_ms) {
    if (tile < 0) return fail(GDN_ERR_ARG, "tile=%d is negative", tile);
    if (load != 0 && load != 1) return fail(GDN_ERR_ARG, "load=%d is neither 0 (K) nor 1 (V)", load);
    if (!(timeout_ms > 0.0 && timeout_ms <= 2000.0))
        return fail(GDN_ERR_ARG, "timeout_ms=%g outside (0, 2000]", timeout_ms);
    if (!gdn::tc_available()) return fail(GDN_ERR_UNSUPPORTED, "tensor-core path not built");
    gdn::arm_wait_expiry(tile, load, (unsigned long long)(timeout_ms * 1e6));
    return GDN_OK;
}

const char* gdn_last_error(void) { return t_last_error.c_str(); }

int64_t gdn_launch_count(void) { return t_launches; }

}  // extern "C"

// Device address of the status word for kernels in other translation units.
namespace gdn {
void record_error(int code, const char* msg) {
    (void)code;
    t_last_error = msg;
}

int* status_ptr() {
    static thread_local int dev = -1;
    static thread_local int* ptr = nullptr;
    int cur = 0;
    cudaGetDevice(&cur);
    if (cur != dev || !ptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
        ptr = (int*)p;
        dev = cur;
    }
    return ptr;
}
}  // namespace gdn
