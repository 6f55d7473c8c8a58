// tc.h — internal launchers of the tcgen05 (tensor-core) kernels of libgdn.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

int* status_ptr();     // device address of the status word (api.cu)
bool tc_available();     // true when this build carries the sm_100a tensor-core kernels
bool tc_i8_available();  // true when the INT8 tensor-core kernel is built

cudaError_t launch_build_A_tc(const void* K, const float* beta, const float* g, float* A,
                              int64_t nc, int k, cudaStream_t st);
// k = 256, bf16 K: three 128 x 128 blocks of K K^T per chunk
cudaError_t launch_build_A256_tc(const void* K, const float* beta, const float* g, float* A,
                                 int64_t nc, cudaStream_t st);
cudaError_t launch_neumann_tc(const float* A, float* T, int64_t nc, int k, int N, int mask, int S,
                              cudaStream_t st);
// exact inverse by 2 x 2 block decomposition (16 x 16 diagonal blocks by
// substitution, then T <- T + T (A_L T) per doubling level); k in {32, 64}
cudaError_t launch_blockinv_tc(const float* A, float* T, int64_t nc, int k, cudaStream_t st);
// truncated series, then M sequential correction steps T <- T + T (I - (I - A) T)
cudaError_t launch_newton_tc(const float* A, float* T, int64_t nc, int k, int N, int mask, int M,
                             cudaStream_t st);
// k = 256: truncated series (Horner, by 128 x 128 blocks) and residual, one chunk per CTA
cudaError_t launch_neumann256_tc(const float* A, float* T, int64_t nc, int N, int mask, int S,
                                cudaStream_t st);
cudaError_t launch_wy_tc(const float* T, const void* K, const void* V, const float* beta,
                         const float* g, void* W, void* U, int64_t nc, int k, cudaStream_t st);
// S > 0: the residual correction in int8 products follows (debug outputs still
// describe the series)
cudaError_t launch_neumann_i8_tc(const float* A, float* T, int N, int mask, int8_t* q,
                                 int32_t* acc, float* sc, int64_t nc, cudaStream_t st, int S = 0);
// the fused step with its prologue: K rows L2-normalised in shared memory and
// the per-token log-gates summed chunk-locally; optional outputs of both
cudaError_t launch_fused_raw_tc(const void* K, const void* V, const float* beta,
                                const float* loggate, int N, int mask, int S, int gated, void* W,
                                void* U, float* Tout, void* Kout, float* gout, int64_t nc, int k,
                                cudaStream_t st);
// INT16 series (k = 64): int16 codes through unsigned-byte products, int64 accumulators;
// S > 0: the residual correction in int16 products follows
cudaError_t launch_neumann_i16_tc(const float* A, float* T, int N, int mask, int16_t* q,
                                  int64_t* acc, double* sc, int64_t nc, cudaStream_t st,
                                  int S = 0);
cudaError_t launch_fused_tc(const void* K, const void* V, const float* beta, const float* g,
                            int N, int mask, int S, int gated, void* W, void* U, float* Tout,
                            int64_t nc, int k, cudaStream_t st);
// the chunk-wise forward's output pass (k = 64, bf16): O = s (diag(gamma) Q S_c^T +
// (Q K^T . Gamma . L) V~) from the chunks' start states Sst (fp16 [nchunks][128][128])
// and V~ (fp16); s = 1 / ||q|| when normalize_q, else 1
cudaError_t launch_output_tc(const void* Q, const void* K, const void* Vt, const float* g,
                             const void* Sst, void* O, int64_t nchunks, bool normalize_q,
                             cudaStream_t st);
// tests of the bounded waits: the next launch_fused_tc on this host thread
// leaves tile `tile`'s K (v = 0) or V (v = 1) load unissued and bounds every
// wait by `timeout_ns`
void arm_wait_expiry(int tile, int v, unsigned long long timeout_ns);

}  // namespace gdn
