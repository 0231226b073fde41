// moe_static.cu -- moe_expert_ffn_static: the expert FFN with its scratch in a
// fixed device array owned by the library instead of a caller-supplied workspace.
//
// Some callers cannot hand the library a workspace: an op hosted by an inference
// engine that owns every device allocation and gives its ops no allocator, or a
// serving loop that must not allocate device memory once it has started.  For
// them this entry point keeps the FFN's only scratch -- the SwiGLU activations H
// between the two GEMMs, plus a status word -- in a file-scope __device__ array of
// MOE_STATIC_SCRATCH_BYTES bytes.  Every GPU that loads the library holds that
// array until the process exits.
//
// The array's name is only a host-side stand-in in host code, never a device
// address, so the address is looked up with cudaGetSymbolAddress once per device
// (on the first call made while that device is current) and cached.  The cache
// belongs to the device's primary context, the one the runtime API uses: after
// cudaDeviceReset the module is loaded again and the cached address is stale, so a
// process that resets a device must not call this entry point on it again.
#include <cuda_runtime.h>

#include <mutex>

#include "moe_internal.h"

namespace moe {
namespace {

constexpr size_t kStatusBytes = 256;

static __device__ __align__(256) unsigned char g_ffn_scratch[MOE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_ffn_scratch on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_ffn_scratch);
        if (err != cudaSuccess) return err;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_expert_ffn_static(const void* x_perm, const int32_t* offsets,
                                            const void* W1, const void* W3, const void* W2,
                                            int rows, int d, int h, int E, moe_dtype dt,
                                            float* y_perm, cudaStream_t stream) {
    // The same argument checks as moe_expert_ffn (which also takes a single expert),
    // then the scratch limit in place of the workspace size.
    if (rows < 0 || rows % 2 != 0) return MOE_ERR_INVALID_ARG;
    moe_status st = check_shape(rows / 2, d, h, E, 2, dt, true, /*routed=*/false);
    if (st != MOE_OK) return st;
    // H [rows, h] must fit behind the status word.
    const size_t h_bytes = static_cast<size_t>(rows) * h * dtype_bytes(dt);
    if (h_bytes > MOE_STATIC_SCRATCH_BYTES - kStatusBytes) return MOE_ERR_WORKSPACE;
    if (rows == 0) return MOE_OK;
    if (!ptrs_ok({x_perm, offsets, W1, W3, W2, y_perm})) return MOE_ERR_INVALID_ARG;

    void* base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return MOE_ERR_CUDA;
    uint32_t* status = static_cast<uint32_t*>(base);
    void* H = static_cast<char*>(base) + kStatusBytes;
    // The array keeps whatever the previous call left; only the status word has to
    // start at zero (H is fully written by the first GEMM before the second reads it).
    if (cudaMemsetAsync(status, 0, sizeof(uint32_t), stream) != cudaSuccess) return MOE_ERR_CUDA;

    cudaError_t err;
    if (dt == MOE_BF16) {
        err = launch_ffn_bf16(x_perm, offsets, W1, W3, W2, rows, d, h, E, H, y_perm, nullptr, 0,
                              /*reduce=*/true, nullptr, status, stream);
        if (err == cudaErrorInvalidValue) return MOE_ERR_INVALID_ARG;
    } else {
        err = launch_ffn_f32(static_cast<const float*>(x_perm), offsets,
                             static_cast<const float*>(W1), static_cast<const float*>(W3),
                             static_cast<const float*>(W2), rows, d, h, E,
                             static_cast<float*>(H), y_perm, stream);
    }
    if (err != cudaSuccess) return MOE_ERR_CUDA;
    if (debug_sync_enabled()) {
        if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
        uint32_t flags = 0;
        if (cudaMemcpy(&flags, status, sizeof(flags), cudaMemcpyDeviceToHost) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (flags & MOE_DEV_FLAG_TIMEOUT) return MOE_ERR_TIMEOUT;
    }
    return MOE_OK;
}
