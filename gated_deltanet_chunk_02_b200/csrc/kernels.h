// kernels.h — internal launchers of libgdn (host side, not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

// CUDA-core kernels (simt.cu); k in {32, 64, 128} unless stated.
cudaError_t launch_build_A_simt(const void* K, const float* beta, const float* g, float* A,
                                int64_t nc, int k, bool bf16, cudaStream_t st);  // k <= 256
cudaError_t launch_neumann_simt(const float* A, float* T, int64_t nc, int k, int N, int mask,
                                int S, cudaStream_t st);
cudaError_t launch_wy_simt(const float* T, const void* K, const void* V, const float* beta,
                           const float* g, void* W, void* U, int64_t nc, int k, bool bf16,
                           cudaStream_t st);
cudaError_t launch_fused_simt(const void* K, const void* V, const float* beta, const float* g,
                              int N, int mask, int S, int gated, void* W, void* U, float* Tout,
                              int64_t nc, int k, bool bf16, cudaStream_t st);
cudaError_t launch_fwdsub(const float* A, float* T, int64_t nc, int k, cudaStream_t st);  // k <= 256
cudaError_t launch_neumann_i8_simt(const float* A, float* T, int N, int mask, int8_t* q,
                                   int32_t* acc, float* sc, int64_t nc, cudaStream_t st);

// Inter-chunk state scan of the forward (scan.cu); k = 64, d = 128.
// bf16: U is overwritten by V~ (fp16) and Sstates ([B*H*nchunk][d][d] fp16) by
// the chunks' start states; f32 uses neither.
// normalize_q (bf16): the query rows come raw and are L2-normalised in the output pass.
cudaError_t launch_scan(const void* Q, const void* K, const void* Wg, void* U, const float* g,
                        const float* S0, void* O, float* Sfin, void* Sstates, int64_t BH,
                        int64_t nchunk, bool bf16, cudaStream_t st, bool normalize_q = false);

// Decode steps (decode.cu); d = 128, S [B][Hv][d][d] fp32 updated in place.
cudaError_t launch_decode(const void* Q, const void* K, const void* V, const float* beta,
                          const float* loggate, float* S, void* O, int64_t B, int64_t Hk,
                          int64_t Hv, int64_t n, bool bf16, cudaStream_t st);

}  // namespace gdn
