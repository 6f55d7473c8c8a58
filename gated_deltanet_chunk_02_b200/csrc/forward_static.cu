// forward_static.cu — gdn_forward_static: the full forward with its scratch
// (W_g and U for every chunk, then A and T) in a fixed device array that the
// library owns, instead of a caller-provided workspace.
//
// Who needs this: callers that are not allowed to allocate device memory
// while they run.  Typical cases are plug-ins hosted by a serving process that
// owns the whole GPU memory pool and hands plug-ins no allocator, and
// fixed-budget deployments that reserve every byte at start-up; for them a
// cudaMalloc in the middle of a request is either forbidden or would
// synchronise the device and fragment the host's pool.  This entry point
// allocates nothing: the scratch is the array below, loaded with the library.
//
// Limits and sharing:
//  * the array holds kStaticScratchBytes (64 MiB) on every GPU that loads the
//    library, for as long as the library stays loaded;
//  * a call needs nc * (2 * k * d * elem + 2 * k * k * 4) bytes of it
//    (elem = 2 for bf16, 4 for f32) and is rejected with GDN_ERR_ARG when that
//    exceeds the array: at k = 64 a chunk needs 64 KiB (bf16) or 96 KiB (f32),
//    so the array holds 1024 bf16 chunks or 682 f32 chunks;
//  * every call on a device uses the same array and leaves its contents
//    behind; the forward overwrites every byte it reads before reading it, so
//    nothing has to start at zero;
//  * calls whose kernels overlap on the GPU (different streams without an
//    ordering between them) race on the array: serialise them.
//
// Set-up: the first call on each device (with that device current) looks up
// the array's device address with cudaGetSymbolAddress; make that first call
// before any stream capture.  The address is cached for the life of the
// process: a device reset (cudaDeviceReset) invalidates it, and the library
// must be reloaded after one.
#include <mutex>

#include "../../include/gdn.h"
#include "common.cuh"

namespace gdn {
void record_error(int code, const char* msg);   // api.cu: gdn_last_error() text
}  // namespace gdn

namespace {

constexpr int64_t kStaticScratchBytes = 64ll << 20;
__device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_lock;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once).
int scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        gdn::record_error(GDN_ERR_CUDA, cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        gdn::record_error(GDN_ERR_UNSUPPORTED, "device ordinal beyond the static scratch table");
        return GDN_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> hold(g_lock);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) {
            gdn::record_error(GDN_ERR_CUDA, cudaGetErrorString(e));
            return GDN_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return GDN_OK;
}

}  // namespace

extern "C" {

int gdn_forward_static(const void* Q, const void* K, const void* V, const float* beta,
                       const float* g, const float* S0, int N, int mask, int S, int exact,
                       void* O, float* S_final, gdn_shape s, gdn_dtype dtype, void* stream) {
    const int64_t need = gdn_forward_workspace_bytes(s, dtype);
    if (need < 0) {
        gdn::record_error(GDN_ERR_ARG, "gdn_forward_static: invalid shape or dtype");
        return GDN_ERR_ARG;
    }
    if (need > kStaticScratchBytes) {
        gdn::record_error(GDN_ERR_ARG,
                          "gdn_forward_static: this problem needs more scratch than the 64 MiB "
                          "static array; use gdn_forward with a workspace");
        return GDN_ERR_ARG;
    }
    if (need == 0) {
        return gdn_forward(Q, K, V, beta, g, S0, N, mask, S, exact, O, S_final, nullptr, 0, s,
                           dtype, stream);
    }
    void* ws = nullptr;
    const int rc = scratch_address(&ws);
    if (rc != GDN_OK) return rc;
    return gdn_forward(Q, K, V, beta, g, S0, N, mask, S, exact, O, S_final, ws,
                       kStaticScratchBytes, s, dtype, stream);
}

}  // extern "C"
