// ffn_f32.cu -- the per-expert SwiGLU FFN in plain fp32 on CUDA cores (no TF32).
//
// notion notes "Mixtral of Experts", "Implementation" (SwiGLU expert function);
// atlas "Mixtral", "Design overview".  Used for the fp32 layer, whose tolerance
// (1e-5 relative) rules out tensor-core TF32.  One warp per output element: lanes
// stride over the reduction dimension with coalesced loads, then a shuffle tree.
//   pass 1: H[r, j] = silu(x_r . W1[e, j]) * (x_r . W3[e, j])
//   pass 2: Y[r, c] = H[r] . W2[e, c]
// where e is the group that owns grouped row r.
#include "moe_internal.h"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kFfnThreads = 256;

__device__ __forceinline__ int group_of(const int* s_off, int E, int r) {
    int e = 0;
    while (e + 1 < E && r >= s_off[e + 1]) ++e;
    return e;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

__global__ void __launch_bounds__(kFfnThreads)
    ffn1_f32_kernel(const float* __restrict__ xp, const int32_t* __restrict__ offsets,
                    const float* __restrict__ W1, const float* __restrict__ W3, int rows, int d,
                    int h, int E, int cap, float* __restrict__ H) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ int s_off[kMaxExperts + 1];
    if (threadIdx.x <= E) s_off[threadIdx.x] = offsets[threadIdx.x];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const size_t nwarps = static_cast<size_t>(gridDim.x) * (blockDim.x >> 5);
    const size_t total = static_cast<size_t>(rows) * h;
    for (size_t o = blockIdx.x * static_cast<size_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
         o < total; o += nwarps) {
        const int r = static_cast<int>(o / h);
        const int j = static_cast<int>(o - static_cast<size_t>(r) * h);
        const int e = group_of(s_off, E, r);
        if (r - s_off[e] >= cap) continue;  // beyond the expert's capacity (warp-uniform)
        const float* xr = xp + static_cast<size_t>(r) * d;
        const float* w1 = W1 + (static_cast<size_t>(e) * h + j) * d;
        const float* w3 = W3 + (static_cast<size_t>(e) * h + j) * d;
        float a = 0.f, b = 0.f;
        for (int i = lane; i < d; i += 32) {
            const float xv = xr[i];
            a = fmaf(xv, w1[i], a);
            b = fmaf(xv, w3[i], b);
        }
        a = warp_sum(a);
        b = warp_sum(b);
        if (lane == 0) H[o] = a / (1.0f + expf(-a)) * b;
    }
}

__global__ void __launch_bounds__(kFfnThreads)
    ffn2_f32_kernel(const float* __restrict__ H, const int32_t* __restrict__ offsets,
                    const float* __restrict__ W2, int rows, int d, int h, int E, int cap,
                    float* __restrict__ Y) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ int s_off[kMaxExperts + 1];
    if (threadIdx.x <= E) s_off[threadIdx.x] = offsets[threadIdx.x];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const size_t nwarps = static_cast<size_t>(gridDim.x) * (blockDim.x >> 5);
    const size_t total = static_cast<size_t>(rows) * d;
    for (size_t o = blockIdx.x * static_cast<size_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
         o < total; o += nwarps) {
        const int r = static_cast<int>(o / d);
        const int c = static_cast<int>(o - static_cast<size_t>(r) * d);
        const int e = group_of(s_off, E, r);
        if (r - s_off[e] >= cap) continue;
        const float* hr = H + static_cast<size_t>(r) * h;
        const float* w2 = W2 + (static_cast<size_t>(e) * d + c) * h;
        float acc = 0.f;
        for (int j = lane; j < h; j += 32) acc = fmaf(hr[j], w2[j], acc);
        acc = warp_sum(acc);
        if (lane == 0) Y[o] = acc;
    }
}

}  // namespace

cudaError_t launch_ffn_f32(const float* x_perm, const int32_t* offsets, const float* W1,
                           const float* W3, const float* W2, int rows, int d, int h, int E,
                           float* H, float* Y, cudaStream_t s, cudaEvent_t between, int cap) {
    const int warps = kFfnThreads / 32;
    const size_t max_blocks = static_cast<size_t>(device_sm_count()) * 16;
    size_t b1 = (static_cast<size_t>(rows) * h + warps - 1) / warps;
    size_t b2 = (static_cast<size_t>(rows) * d + warps - 1) / warps;
    b1 = b1 > max_blocks ? max_blocks : (b1 < 1 ? 1 : b1);
    b2 = b2 > max_blocks ? max_blocks : (b2 < 1 ? 1 : b2);
    cudaError_t err = launch_k(ffn1_f32_kernel, static_cast<unsigned>(b1), kFfnThreads, 0, s,
                               x_perm, offsets, W1, W3, rows, d, h, E, cap, H);
    if (err != cudaSuccess) return err;
    if (between && (err = cudaEventRecord(between, s)) != cudaSuccess) return err;
    return launch_k(ffn2_f32_kernel, static_cast<unsigned>(b2), kFfnThreads, 0, s, H, offsets,
                    W2, rows, d, h, E, cap, Y);
}

}  // namespace moe
