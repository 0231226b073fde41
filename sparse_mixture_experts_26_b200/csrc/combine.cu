// combine.cu -- weighted un-permute of the expert outputs.
//
// crackai "Mixtral of Experts", "Top-2 Routing in Detail":
// y = w_1 Expert_{i1}(x) + w_2 Expert_{i2}(x); notion notes "Mixtral of Experts",
// "Implementation", eq. y.  Each output element is w0*Y[r0] + w1*Y[r1] evaluated in
// fp32 (slot 0 first, one fused multiply-add for slot 1) and rounded once to the
// output dtype.  Pure streaming: reads 2 fp32 rows, writes 1 row per token.  When
// the expert outputs arrive as split-K partial sums, each row is first summed over
// the partials in a fixed order, so the result does not depend on scheduling.
#include <cuda_bf16.h>

#include "moe_internal.h"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kCombineThreads = 256;

__device__ __forceinline__ void store4(float* y, size_t i, float4 v) {
    reinterpret_cast<float4*>(y)[i] = v;
}
__device__ __forceinline__ void store4(__nv_bfloat16* y, size_t i, float4 v) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&lo);
    u.y = *reinterpret_cast<uint32_t*>(&hi);
    reinterpret_cast<uint2*>(y)[i] = u;
}

// Row r of the in-order sum of nsplit arrays split_stride4 float4s apart.  The first
// kDecodeSplitK partials are all loaded before the first add, so their loads overlap.
__device__ __forceinline__ void add4(float4& a, const float4& b) {
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
}
__device__ __forceinline__ float4 split_sum(const float4* __restrict__ Y, int nsplit,
                                           size_t split_stride4, size_t at) {
    float4 p[kDecodeSplitK];
#pragma unroll
    for (int i = 0; i < kDecodeSplitK; ++i)
        if (i < nsplit) p[i] = Y[static_cast<size_t>(i) * split_stride4 + at];
    float4 a = p[0];
#pragma unroll
    for (int i = 1; i < kDecodeSplitK; ++i)
        if (i < nsplit) add4(a, p[i]);
    for (int i = kDecodeSplitK; i < nsplit; ++i)
        add4(a, Y[static_cast<size_t>(i) * split_stride4 + at]);
    return a;
}

// kSplit: the expert outputs arrive as split-K partials (small batches).  The
// single-array form keeps its register count low, so that enough warps stay resident
// to stream large batches at full bandwidth.
template <typename Tout, bool kSplit>
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const float4* __restrict__ Y, int nsplit, size_t split_stride4,
                   const int32_t* __restrict__ inv, const float* __restrict__ w, int T, int d4,
                   Tout* __restrict__ y, const int32_t* __restrict__ idx,
                   const int32_t* __restrict__ offsets, int E, int cap, uint8_t* layout_out,
                   int layout_value) {
    pdl_wait();
    pdl_launch_dependents();
    if (layout_out && blockIdx.x == 0 && threadIdx.x == 0)
        *layout_out = static_cast<uint8_t>(layout_value);
    const size_t n = static_cast<size_t>(T) * d4;
    const unsigned P = 2u * static_cast<unsigned>(T);
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const size_t t = i / d4;
        const size_t c = i - t * d4;
        const unsigned r0 = static_cast<unsigned>(inv[2 * t]);
        const unsigned r1 = static_cast<unsigned>(inv[2 * t + 1]);
        float w0 = w[2 * t], w1 = w[2 * t + 1];
        if (cap != INT_MAX) {
            // a pair `cap` or more rows into its expert's group was dropped
            const unsigned e0 = static_cast<unsigned>(idx[2 * t]);
            const unsigned e1 = static_cast<unsigned>(idx[2 * t + 1]);
            if (e0 >= static_cast<unsigned>(E) || static_cast<int>(r0) - offsets[e0] >= cap) w0 = 0.f;
            if (e1 >= static_cast<unsigned>(E) || static_cast<int>(r1) - offsets[e1] >= cap) w1 = 0.f;
        }
        // inv_perm entries outside [0, 2T) would come from an invalid permutation;
        // they contribute nothing instead of reading out of bounds.
        // dropped pairs (w == 0) are not read: their rows were never written
        const size_t at0 = static_cast<size_t>(r0) * d4 + c;
        const size_t at1 = static_cast<size_t>(r1) * d4 + c;
        const bool use0 = r0 < P && w0 != 0.f, use1 = r1 < P && w1 != 0.f;
        float4 a = make_float4(0, 0, 0, 0), b = a;
        if constexpr (kSplit) {
            if (use0) a = split_sum(Y, nsplit, split_stride4, at0);
            if (use1) b = split_sum(Y, nsplit, split_stride4, at1);
        } else {
            if (use0) a = Y[at0];
            if (use1) b = Y[at1];
        }
        float4 o;
        o.x = fmaf(w1, b.x, w0 * a.x);
        o.y = fmaf(w1, b.y, w0 * a.y);
        o.z = fmaf(w1, b.z, w0 * a.z);
        o.w = fmaf(w1, b.w, w0 * a.w);
        store4(y, i, o);
    }
}

__global__ void __launch_bounds__(kCombineThreads)
    sum_splits_kernel(const float4* __restrict__ parts, int nsplit, size_t n4,
                      float4* __restrict__ Y) {
    pdl_wait();
    pdl_launch_dependents();
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
         i += static_cast<size_t>(gridDim.x) * blockDim.x)
        Y[i] = split_sum(parts, nsplit, n4, i);
}

unsigned grid_for(size_t n) {
    size_t blocks = (n + kCombineThreads - 1) / kCombineThreads;
    const size_t cap = static_cast<size_t>(device_sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return static_cast<unsigned>(blocks);
}

}  // namespace

cudaError_t launch_sum_splits(const float* parts, int nsplit, size_t n, float* Y,
                              cudaStream_t s) {
    const size_t n4 = n / 4;
    return launch_k(sum_splits_kernel, grid_for(n4), kCombineThreads, 0, s,
                    reinterpret_cast<const float4*>(parts), nsplit, n4,
                    reinterpret_cast<float4*>(Y));
}

cudaError_t launch_combine(const float* Y, int nsplit, size_t split_stride,
                           const int32_t* inv_perm, const float* w, int T, int d, moe_dtype dt,
                           void* y, cudaStream_t s, const int32_t* idx, const int32_t* offsets,
                           int E, int cap, uint8_t* layout_out, uint8_t layout_flags) {
    if (cap != INT_MAX && (!idx || !offsets)) return cudaErrorInvalidValue;
    if (nsplit < 1 || nsplit > kLayoutSplitMask) return cudaErrorInvalidValue;
    const int lv = nsplit | layout_flags;
    const int d4 = d / 4;
    const unsigned blocks = grid_for(static_cast<size_t>(T) * d4);
    const float4* Y4 = reinterpret_cast<const float4*>(Y);
    if (dt == MOE_BF16) {
        auto* yb = static_cast<__nv_bfloat16*>(y);
        if (nsplit > 1)
            return launch_k(combine_kernel<__nv_bfloat16, true>, blocks, kCombineThreads, 0, s, Y4,
                            nsplit, split_stride / 4, inv_perm, w, T, d4, yb, idx, offsets, E,
                            cap, layout_out, lv);
        return launch_k(combine_kernel<__nv_bfloat16, false>, blocks, kCombineThreads, 0, s, Y4,
                        nsplit, split_stride / 4, inv_perm, w, T, d4, yb, idx, offsets, E, cap,
                        layout_out, lv);
    }
    if (nsplit != 1) return cudaErrorInvalidValue;  // split-K partials are bf16-path only
    return launch_k(combine_kernel<float, false>, blocks, kCombineThreads, 0, s, Y4, nsplit,
                    split_stride / 4, inv_perm, w, T, d4, static_cast<float*>(y), idx, offsets, E,
                    cap, layout_out, lv);
}

}  // namespace moe
