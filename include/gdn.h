/*
 * gdn.h — C ABI of libgdn: the per-chunk hot path of chunk-wise Gated DeltaNet
 * on NVIDIA B200 (sm_100a).
 *
 * The method: "When Good Enough Is Optimal: Multiplication-Only Matrix
 * Inversion Approximation for Quantized Gated DeltaNet" (arXiv 2606.06034),
 * as summarised on gist.science (sections "Énoncé du Problème",
 * "Méthodologie" §1-§3, "Adaptation à la Quantification").  Each chunk of k
 * tokens needs T = (I - A)^{-1} for a strictly lower-triangular A; T is
 * approximated with matrix products only (truncated Neumann series, a
 * structural band mask and a parallel residual correction) and then applied
 * to form the WY factors.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout.  Head-major and chunk-contiguous: K, V, Q, W, U, O are
 *   [B, H, T, d] row-major (d = 128); beta, g are [B, H, T] float32;
 *   A, T are [B, H, T/k, k, k] float32 row-major.  Chunk c of the flattened
 *   [B*H*T/k] sequence owns rows [c*k, (c+1)*k) of every [.., T, ..] array.
 *   nc = B*H*T/k is the number of chunks.
 * Pointers.  All data pointers are DEVICE pointers owned by the caller, who
 *   allocates them; the library never allocates device memory in a call.
 *   Every pointer must be 16-byte aligned (tensor-memory-access rule).
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  Every call is asynchronous on that stream; none synchronises,
 *   except gdn_get_status.
 * Errors.  Arguments are checked on the host before any launch; a failing
 *   check returns a negative code, launches nothing and records a message for
 *   gdn_last_error().  Device-side failures (a bounded wait that ran out) set a
 *   per-device status word read by gdn_get_status(); kernels never trap.
 * Values.  NaN/Inf inputs are not checked.  g must be the chunk-local
 *   cumulative sum of the per-token log-gates (g_i includes token i's gate);
 *   within a chunk g is then non-increasing, and exp(g_i - g_j) is evaluated
 *   only for i > j, so it never overflows.
 * Precision.  A and T are float32 in memory.  `dtype` fixes the type of
 *   K, V, Q, W, U, O.  bf16 data run their contractions on the tcgen05 tensor
 *   cores (bf16 x bf16 for K K^T and WY, fp16 x fp16 for the k x k chain, all
 *   accumulating in fp32); float32 data run on CUDA cores in fp32.
 */
#ifndef GDN_H
#define GDN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct gdn_shape {
    int64_t B, H, T;   /* batch, heads, tokens per sequence (T % k == 0)   */
    int32_t k;         /* chunk size: 32, 64, 128 or 256                    */
    int32_t d;         /* head dim d_k = d_v; 128 is the supported value    */
} gdn_shape;

typedef enum gdn_dtype { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/* Arithmetic of the k x k product chain in gdn_invert_neumann. */
typedef enum gdn_prec {
    GDN_PREC_F32 = 0,  /* float32 FMA on CUDA cores (k <= 128)               */
    GDN_PREC_F16 = 1   /* tcgen05 tensor cores, fp16 operands, fp32 accumulate */
} gdn_prec;

enum {
    GDN_OK = 0,
    GDN_ERR_ARG = -1,          /* null pointer, bad size, N/S out of range   */
    GDN_ERR_ALIGN = -2,        /* a pointer is not 16-byte aligned           */
    GDN_ERR_UNSUPPORTED = -3,  /* valid request this build does not serve    */
    GDN_ERR_CUDA = -4,         /* a CUDA runtime/driver call failed          */
    GDN_ERR_TIMEOUT = -5       /* device status: a bounded wait ran out      */
};

/*
 * A_ij = -beta_i (k_i . k_j) exp(g_i - g_j) for i > j, 0 for i <= j, per chunk.
 * The summary's problem statement ("Énoncé du Problème") fixes A as strictly
 * lower triangular; its entries are those of the gated delta-rule chunk
 * system.  In: K [B,H,T,d] (dtype), beta, g [B,H,T] f32.  Out: A [nc,k,k] f32.
 */
int gdn_build_A(const void* K, const float* beta, const float* g, float* A,
                gdn_shape s, gdn_dtype dtype, void* stream);

/*
 * Multiplication-only approximate inverse T ~ (I - A)^{-1} per chunk
 * ("Méthodologie" §1-§3): T0 = sum_{n=0}^{N} A^n (N >= 1 highest power), with
 * the band mask M_ij = [i - j <= N] applied to every power when mask != 0;
 * then, if S > 0, E = I - (I - A) T0 and T = T0 sum_{s=0}^{S} E^s (S >= 0).
 * In: A [nc,k,k] f32.  Out: T [nc,k,k] f32.  1 <= N <= k-1, 0 <= S <= 64.
 * GDN_PREC_F16 (tensor cores: fp16 operands, fp32 accumulation) serves
 * every k; GDN_PREC_F32 (fp32 on CUDA cores) serves k <= 128 and returns
 * GDN_ERR_UNSUPPORTED at k = 256.
 */
int gdn_invert_neumann(const float* A, float* T, gdn_shape s, int N, int mask,
                       int S, gdn_prec prec, void* stream);

/*
 * Sequential residual correction, the comparison point of "Méthodologie" §3
 * (the iterative update the method replaces by its parallel sum): T_0 is the
 * truncated series with the band mask as in gdn_invert_neumann, then M steps
 *   R_m = I - (I - A) T_m,   T_{m+1} = T_m + T_m R_m,
 * two dependent products per step.  In exact arithmetic T_M equals
 * gdn_invert_neumann with S = 2^M - 1.  Tensor cores (fp16 operands, fp32
 * accumulation), k in {32, 64, 128} (GDN_ERR_UNSUPPORTED at 256),
 * 0 <= M <= 6.  In: A [nc,k,k] f32.  Out: T [nc,k,k] f32.
 */
int gdn_invert_newton(const float* A, float* T, gdn_shape s, int N, int mask, int M,
                      void* stream);

/*
 * Exact T = (I - A)^{-1} by 2 x 2 block decomposition, the other comparison
 * point of "Énoncé du Problème" (block inversion): the 16 x 16 diagonal
 * blocks by substitution, then per doubling level T <- T + T (A_L T) with
 * A_L = A on that level's off-diagonal blocks (T10 = T11 A10 T00).  Tensor
 * cores with fp16 operands and fp32 accumulation, like GDN_PREC_F16.
 * k in {32, 64} (GDN_ERR_UNSUPPORTED above).  In: A [nc,k,k] f32.  Out: T f32.
 */
int gdn_invert_blocked(const float* A, float* T, gdn_shape s, void* stream);

/*
 * Exact T = (I - A)^{-1} by forward substitution ("Énoncé du Problème": the
 * k-1 sequential row steps the method replaces).  fp32 on CUDA cores.
 * In: A [nc,k,k] f32.  Out: T [nc,k,k] f32.
 */
int gdn_invert_fwdsub(const float* A, float* T, gdn_shape s, void* stream);

/*
 * WY factors W = T diag(beta) K and U = T diag(beta) V per chunk.  If g is
 * non-NULL, W is the gated factor T diag(beta * exp(g)) K used by the chunk
 * recurrence (U unchanged).  In: T [nc,k,k] f32, K, V [B,H,T,d] (dtype),
 * beta, g [B,H,T] f32.  Out: W, U [B,H,T,d] (dtype).
 */
int gdn_wy(const float* T, const void* K, const void* V, const float* beta,
           const float* g, void* W, void* U, gdn_shape s, gdn_dtype dtype,
           void* stream);

/*
 * INT8 truncated Neumann series ("Adaptation à la Quantification"): A and every
 * power held as int8 codes with one symmetric fp32 scale per chunk and power,
 * int32 accumulation on the tensor cores, band mask applied to each power
 * before it is quantised, dequantised T0 = I + sum_n s_n q_n in fp32.  The
 * fixed float32 operation order (IEEE, round-to-nearest-even, no FMA) is:
 *   P1 = M.A; a = max|P1|; q1 = clamp(rint(P1 * (127/a)), +-127); s1 = a/127;
 *   acc_n = q_{n-1} q1 (masked); m = max|acc_n|;
 *   q_n = clamp(rint(float(acc_n) * (127/float(m))), +-127);
 *   s_n = (s_{n-1} * s1) * (float(m)/127); zero maxima give q = 0, s = 0;
 *   T0 = I + s_1 q_1 + ... + s_N q_N, summed left to right.
 * In: A [nc,k,k] f32.  Out: T [nc,k,k] f32.  Optional debug outputs (NULL to
 * skip): q [nc,N,k,k] int8, acc [nc,N,k,k] int32 (slot 0 zero), scale [nc,N]
 * f32.  k = 64, 1 <= N <= 8.
 */
int gdn_invert_neumann_i8(const float* A, float* T, int N, int mask,
                          int8_t* q_dbg, int32_t* acc_dbg, float* scale_dbg,
                          gdn_shape s, void* stream);

/*
 * INT8 series followed by the parallel residual correction with every product
 * in int8 codes ("Adaptation à la Quantification": N = 3 compensated by S = 8;
 * "Méthodologie" §3 for E and T = T0 sum_{s<=S} E^s).  After the series of
 * gdn_invert_neumann_i8, with the same quantisation rules (codes(x): per-chunk
 * a = max|x|, q = clamp(rint(x * (127/a)), +-127), s = a/127; float32, no FMA):
 *   X = T0 - I;  E = (A - X) + (s_A * s_X) * float(q_A q_X)   (whole A, no mask);
 *   q_E1 = codes(E); q_E,s, s_E,s for s = 2..S requantised as the powers of A;
 *   Gm = s_E1 q_E1 + ... + s_E,S q_E,S (left to right);
 *   T = (T0 + Gm) + (s_X * s_G) * float(q_X q_G),  q_G = codes(Gm).
 * In: A [nc,k,k] f32.  Out: T [nc,k,k] f32.  k = 64, 1 <= N <= 8, 1 <= S <= 64.
 */
int gdn_invert_neumann_i8_residual(const float* A, float* T, int N, int mask, int S,
                                   gdn_shape s, void* stream);

/*
 * INT16 truncated Neumann series ("Adaptation à la Quantification", the INT16
 * operating point): as gdn_invert_neumann_i8 with codes in [-32767, 32767].
 * Products of two code matrices reach 2^36, so accumulators are exact int64
 * and every scale operation is IEEE binary64 (round to nearest even, no FMA):
 *   P1 = M.A; a = max|P1|; q1 = clamp(rint(double(P1) * (32767/double(a))), +-32767);
 *   s1 = double(a)/32767; acc_n = q_{n-1} q1 (masked); m = max|acc_n|;
 *   q_n = clamp(rint(double(acc_n) * (32767/double(m))), +-32767);
 *   s_n = (s_{n-1} * s1) * (double(m)/32767); zero maxima give q = 0, s = 0;
 *   T0 = I + s_1 q_1 + ... + s_N q_N summed left to right in binary64, then
 *   rounded once to float32.
 * In: A [nc,k,k] f32.  Out: T [nc,k,k] f32.  Optional debug outputs (NULL to
 * skip): q [nc,N,k,k] int16, acc [nc,N,k,k] int64 (slot 0 zero), scale
 * [nc,N] f64.  k = 64, 1 <= N <= 8.
 */
int gdn_invert_neumann_i16(const float* A, float* T, int N, int mask, int16_t* q_dbg,
                           int64_t* acc_dbg, double* scale_dbg, gdn_shape s, void* stream);

/*
 * INT16 series followed by the parallel residual correction with every product
 * in int16 codes ("Adaptation à la Quantification": the INT16 operating point,
 * N = 3 compensated by S = 8; "Méthodologie" §3 for E and T = T0 sum_{s<=S} E^s).
 * The steps of gdn_invert_neumann_i8_residual under the rules of
 * gdn_invert_neumann_i16 (codes in [-32767, 32767], exact int64 products, every
 * scale and sum in IEEE binary64, no FMA):
 *   T0 = I + s_1 q_1 + ... + s_N q_N (binary64, not rounded);  X = T0 - I;
 *   E = (A - X) + (s_A * s_X) * double(q_A q_X)   (whole A, no mask);
 *   q_E1 = codes(E); q_E,s, s_E,s for s = 2..S requantised as the powers of A;
 *   Gm = s_E1 q_E1 + ... + s_E,S q_E,S (left to right);
 *   T = (T0 + Gm) + (s_X * s_G) * double(q_X q_G),  q_G = codes(Gm), then
 *   rounded once to float32.
 * In: A [nc,k,k] f32.  Out: T [nc,k,k] f32.  k = 64, 1 <= N <= 8,
 * 1 <= S <= 64.  Errors as gdn_invert_neumann_i16.
 */
int gdn_invert_neumann_i16_residual(const float* A, float* T, int N, int mask, int S,
                                    gdn_shape s, void* stream);

/*
 * Fused per-chunk pipeline: A from K, beta, g; T by the Neumann + mask +
 * residual method (as gdn_invert_neumann); then W, U (gated W if gated != 0).
 * Only K, V, beta, g are read and only W, U (and T when T_out is non-NULL)
 * written.  bf16: tensor-core path; f32: CUDA-core path (k <= 128).
 */
int gdn_chunk_wy_fused(const void* K, const void* V, const float* beta,
                       const float* g, int N, int mask, int S, int gated,
                       void* W, void* U, float* T_out, gdn_shape s,
                       gdn_dtype dtype, void* stream);

/*
 * gdn_chunk_wy_fused with its prologue fused in: the steps just before A in a
 * layer.  K_raw rows are L2-normalised, k_i <- k_i / ||k_i|| (norm in fp32, the
 * result rounded to bf16; an all-zero row stays zero), and loggate holds each
 * token's own log-gate, summed chunk-locally into g (g_i includes token i),
 * inside the kernel before K K^T.  Everything else is gdn_chunk_wy_fused.
 * Optional outputs (NULL to skip): K_out [B,H,T,d] bf16, the normalised keys;
 * g_out [B,H,T] f32, the cumulative log-gates (what a later scan reads).
 * bf16 data, k in {32, 64, 128}.
 */
int gdn_chunk_wy_fused_raw(const void* K_raw, const void* V, const float* beta,
                           const float* loggate, int N, int mask, int S, int gated, void* W,
                           void* U, float* T_out, void* K_out, float* g_out, gdn_shape s,
                           gdn_dtype dtype, void* stream);

/*
 * Full chunk-wise Gated DeltaNet forward.  Per chunk: V~ = U - W_g S0^T,
 * O = diag(exp g) Q S0^T + (Q K^T . Gamma . L) V~,
 * S' = exp(g_last) S0 + V~^T diag(exp(g_last - g)) K, with
 * Gamma_ij = exp(g_i - g_j) and L the lower triangle with diagonal.  T per
 * chunk comes from the Neumann method (exact = 0) or forward substitution
 * (exact = 1).  In: Q, K, V [B,H,T,d] (dtype), beta, g [B,H,T] f32, S0
 * [B,H,d,d] f32 (d_v x d_k, NULL = zero).  Out: O [B,H,T,d] (dtype),
 * S_final [B,H,d,d] f32.  `workspace` is caller-owned device memory of at
 * least gdn_forward_workspace_bytes(s, dtype) bytes (W_g and U for every
 * chunk in dtype, then A and T in f32); its contents on entry do not matter.
 * k = 64.  The inter-chunk scan splits the d_v rows of the state across CTAs
 * (rows of S never mix), each CTA walking its head's chunks in order; for
 * bf16 data the output pass then forms O for every chunk in parallel on the
 * tensor cores (two chunks per 128-row tile).
 */
int gdn_forward(const void* Q, const void* K, const void* V, const float* beta,
                const float* g, const float* S0, int N, int mask, int S,
                int exact, void* O, float* S_final, void* workspace,
                int64_t workspace_bytes, gdn_shape s, gdn_dtype dtype,
                void* stream);
int64_t gdn_forward_workspace_bytes(gdn_shape s, gdn_dtype dtype);

/*
 * gdn_forward with its prologue: the steps just before the chunk system in a
 * layer (the gist.science summary's Problem Statement places the inversion
 * inside this layer).  Q_raw and K_raw rows are L2-normalised in the kernels,
 * q <- q / ||q||, k <- k / ||k|| (norms in fp32; an all-zero row stays zero;
 * the keys are rounded to bf16 like gdn_chunk_wy_fused_raw's, the queries'
 * scale is applied to each output row in fp32), and loggate holds each
 * token's own log-gate, summed chunk-locally.  The truncated series (exact =
 * 0 of gdn_forward) gives T.  In: Q_raw, K_raw, V [B,H,T,d] bf16, beta,
 * loggate [B,H,T] f32, S0 as in gdn_forward.  Out: O, S_final as in
 * gdn_forward.  `workspace` holds at least
 * gdn_forward_raw_workspace_bytes(s, dtype) bytes: gdn_forward's scratch,
 * then the normalised keys (bf16) and the cumulative log-gates (f32).
 * bf16 data, k = 64; GDN_ERR_UNSUPPORTED otherwise.
 */
int gdn_forward_raw(const void* Q_raw, const void* K_raw, const void* V, const float* beta,
                    const float* loggate, const float* S0, int N, int mask, int S,
                    void* O, float* S_final, void* workspace, int64_t workspace_bytes,
                    gdn_shape s, gdn_dtype dtype, void* stream);
int64_t gdn_forward_raw_workspace_bytes(gdn_shape s, gdn_dtype dtype);

/*
 * gdn_forward without a workspace argument: it allocates nothing.  The pages
 * have no counterpart to this call; it exists for callers that may not
 * allocate device memory while they run (for example a plug-in inside a
 * serving process that owns the whole GPU memory pool and hands out no
 * allocator, or a deployment whose memory budget is fixed at start-up), for
 * whom a cudaMalloc mid-request is forbidden or would synchronise the device.
 * The scratch (W_g, U, A, T) lives in a 64 MiB device array inside the
 * library, held on every GPU that loads it until the library is unloaded.
 * Problems needing more than that (gdn_forward_workspace_bytes(s, dtype) >
 * 64 MiB: more than 1024 chunks of 64 bf16 tokens, or 682 chunks of 64 fp32
 * tokens) return GDN_ERR_ARG.  All calls
 * on a device share the array and leave their data in it; nothing needs to
 * start at zero, but calls whose kernels may overlap on the GPU race on it, so
 * order them on one stream.  The first call on each device (made with that
 * device current) looks up the array's address: make it before any stream
 * capture.  The address is kept for the life of the process, so a device
 * reset (cudaDeviceReset) invalidates it: reload the library after one.
 * Arguments and results are otherwise those of gdn_forward.
 */
int gdn_forward_static(const void* Q, const void* K, const void* V,
                       const float* beta, const float* g, const float* S0,
                       int N, int mask, int S, int exact, void* O,
                       float* S_final, gdn_shape s, gdn_dtype dtype,
                       void* stream);

/*
 * Decode: the gated delta rule advanced token by token from a carried state,
 * as in the technical summary of "A Persistent-State Dataflow Accelerator for
 * Memory-Bound Linear Attention Decode on FPGA" (§1-§2).  For every batch b,
 * value head h and token t = 0 .. n-1, with query/key head j = h / (Hv / Hk)
 * (consecutive value heads share one query and one key):
 *   S <- a_t S (I - b_t k_t k_t^T) + b_t v_t k_t^T,   o_t = S q_t,
 *   a_t = exp(loggate_t)   (the token's own log-gate, not a cumulative sum).
 * In: Q, K [B, Hk, n, d] (dtype), V [B, Hv, n, d] (dtype), beta, loggate
 * [B, Hv, n] f32.  In/out: S [B, Hv, d, d] f32 (d_v x d_k, row-major),
 * updated in place.  Out: O [B, Hv, n, d] (dtype).  d = 128, Hv a multiple of
 * Hk, B <= 65535.  The state is read once and written once per call whatever
 * n is (n = 1 is one decode step).  B, Hv or n = 0: nothing happens.  Errors
 * as for every call; S is untouched on a nonzero return.
 */
int gdn_decode(const void* Q, const void* K, const void* V, const float* beta,
               const float* loggate, float* S, void* O, int64_t B, int64_t Hk, int64_t Hv,
               int64_t n, int32_t d, gdn_dtype dtype, void* stream);

/*
 * Streams: every entry point enqueues its kernels on `stream` (NULL = the
 * legacy default stream) and returns without synchronising; none allocates
 * device memory (gdn_forward takes a caller workspace).  The first call in a
 * process sets kernel attributes and looks up the status word; bench.py
 * makes it eagerly before it captures gdn_decode steps into a CUDA graph.
 */
/* The status word's address is looked up once per host thread and device and
 * kept; a device reset (cudaDeviceReset) invalidates it, as it does the
 * static scratch of gdn_forward_static: reload the library after one. */
/* Synchronises `stream`, returns the device status word of the current
 * device (GDN_OK, GDN_ERR_TIMEOUT, or GDN_ERR_CUDA when a kernel found its
 * shared memory misaligned) and clears it. */
int gdn_get_status(void* stream);

/*
 * Test hook for the bounded device waits; the pages have no counterpart.
 * Arms the next gdn_chunk_wy_fused call made on this host thread (bf16 data,
 * tensor-core path) so that one load of tile `tile` (token rows
 * [128 tile, 128 tile + 128) of the flattened [B*H*T] axis) is never issued:
 * K with beta and g when `load` = 0 (waited for at the start of the tile), V
 * when `load` = 1 (waited for before WY); every wait of that launch is bounded
 * by `timeout_ms` instead of 2 s.
 * The wait for that tile then runs out: the CTA that owns it sets
 * GDN_ERR_TIMEOUT in the status word, finishes the barrier sequence of the
 * tile it is on without starting further products, copies or stores, waits
 * (bounded) for its own work in flight, frees its tensor memory and returns;
 * the other CTAs finish normally.  That call's outputs are undefined; the
 * call after it runs normally.  Returns GDN_OK, or GDN_ERR_ARG for a negative
 * tile, a load other than 0 or 1, or timeout_ms outside (0, 2000].
 */
int gdn_debug_arm_wait_expiry(int tile, int load, double timeout_ms);

/* Message for the most recent nonzero return on this host thread. */
const char* gdn_last_error(void);

/* Number of kernels this library launched on this host thread since load. */
int64_t gdn_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* GDN_H */
