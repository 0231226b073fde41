// route.cu -- router logits, top-2 selection and the two-way softmax.
//
// crackai "Mixtral of Experts", "Top-2 Routing in Detail": gate_logits = x . W_gate;
// notion notes "Mixtral of Experts", "Sparse gating", eq. G(x) = Softmax(TopK(x . W_g)).
//
// One warp per token.  Each lane reads 16-byte vectors of the token's row and
// accumulates all E logits in fp64: a bf16 x bf16 (or fp32 x fp32) product is exact
// in fp64, so the logits carry only the rounding of the fp64 sum and the top-2
// choice does not depend on the reduction order except at ties closer than ~1e-16
// relative.  W_g (d x E) is staged in shared memory once per block when it fits.
// The kernel is bound by reading x once (2*d bytes per token).
#include <cuda_bf16.h>

#include <cfloat>

#include "moe_internal.h"

namespace moe {
namespace {

template <typename Tin>
__device__ __forceinline__ double to_f64(Tin v);
template <>
__device__ __forceinline__ double to_f64<float>(float v) {
    return static_cast<double>(v);
}
template <>
__device__ __forceinline__ double to_f64<__nv_bfloat16>(__nv_bfloat16 v) {
    return static_cast<double>(__bfloat162float(v));
}

constexpr int kRouteThreads = 256;

template <typename Tin, int MAXE, bool WG_IN_SMEM>
__global__ void __launch_bounds__(kRouteThreads)
    route_kernel(const Tin* __restrict__ x, const Tin* __restrict__ Wg, int T, int d, int E,
                 int32_t* __restrict__ idx, float* __restrict__ w) {
    extern __shared__ __align__(16) unsigned char route_smem[];
    const Tin* wg = Wg;
    if (WG_IN_SMEM) {
        Tin* s = reinterpret_cast<Tin*>(route_smem);
        const int n = d * E;
        // 16-byte copies (d*E*sizeof(Tin) is a multiple of 16 since d % 8 == 0 and
        // sizeof(Tin) * 8 >= 16).
        const int nvec = n * static_cast<int>(sizeof(Tin)) / 16;
        for (int i = threadIdx.x; i < nvec; i += blockDim.x)
            reinterpret_cast<uint4*>(s)[i] = reinterpret_cast<const uint4*>(Wg)[i];
        __syncthreads();
        wg = s;
    }
    constexpr int V = 16 / sizeof(Tin);  // elements per 16-byte vector
    const int lane = threadIdx.x & 31;
    const int warps_per_block = blockDim.x >> 5;
    const int gwarp = blockIdx.x * warps_per_block + (threadIdx.x >> 5);
    const int nwarps = gridDim.x * warps_per_block;

    for (int t = gwarp; t < T; t += nwarps) {
        double acc[MAXE];
#pragma unroll
        for (int e = 0; e < MAXE; ++e) acc[e] = 0.0;
        const Tin* xt = x + static_cast<size_t>(t) * d;
        for (int i0 = lane * V; i0 < d; i0 += 32 * V) {
            Tin xv[V];
            *reinterpret_cast<uint4*>(xv) = *reinterpret_cast<const uint4*>(xt + i0);
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const double xd = to_f64(xv[v]);
                const Tin* row = wg + static_cast<size_t>(i0 + v) * E;
#pragma unroll
                for (int e = 0; e < MAXE; ++e)
                    if (e < E) acc[e] = fma(xd, to_f64(row[e]), acc[e]);
            }
        }
#pragma unroll
        for (int e = 0; e < MAXE; ++e) {
            if (e < E) {
                double s = acc[e];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
                acc[e] = s;
            }
        }
        if (lane == 0) {
            // (logit desc, index asc): strict comparisons keep the first maximum.
            double b1 = acc[0];
            int i1 = 0;
#pragma unroll
            for (int e = 1; e < MAXE; ++e)
                if (e < E && acc[e] > b1) {
                    b1 = acc[e];
                    i1 = e;
                }
            double b2 = -DBL_MAX;
            int i2 = -1;
#pragma unroll
            for (int e = 0; e < MAXE; ++e)
                if (e < E && e != i1 && (i2 < 0 || acc[e] > b2)) {
                    b2 = acc[e];
                    i2 = e;
                }
            const float w1 = static_cast<float>(1.0 / (1.0 + exp(b2 - b1)));
            idx[2 * t] = i1;
            idx[2 * t + 1] = i2;
            w[2 * t] = w1;
            w[2 * t + 1] = 1.0f - w1;  // exact (Sterbenz): the pair sums to 1 in float
        }
    }
}

template <typename Tin, int MAXE>
cudaError_t launch_route_t(const void* x, const void* Wg, int T, int d, int E, int32_t* idx,
                           float* w, cudaStream_t s) {
    const size_t wg_bytes = static_cast<size_t>(d) * E * sizeof(Tin);
    const int warps = kRouteThreads / 32;
    int blocks = (T + warps - 1) / warps;
    const int cap = device_sm_count() * 4;
    if (blocks > cap) blocks = cap;
    if (wg_bytes <= 64 * 1024) {
        auto k = route_kernel<Tin, MAXE, true>;
        if (wg_bytes > 48 * 1024)
            cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(wg_bytes));
        k<<<blocks, kRouteThreads, wg_bytes, s>>>(static_cast<const Tin*>(x),
                                                   static_cast<const Tin*>(Wg), T, d, E, idx, w);
    } else {
        route_kernel<Tin, MAXE, false><<<blocks, kRouteThreads, 0, s>>>(
            static_cast<const Tin*>(x), static_cast<const Tin*>(Wg), T, d, E, idx, w);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const void* x, const void* Wg, int T, int d, int E, moe_dtype dt,
                         int32_t* idx, float* w, cudaStream_t s) {
    if (dt == MOE_BF16) {
        return E <= 8 ? launch_route_t<__nv_bfloat16, 8>(x, Wg, T, d, E, idx, w, s)
                      : launch_route_t<__nv_bfloat16, kMaxExperts>(x, Wg, T, d, E, idx, w, s);
    }
    return E <= 8 ? launch_route_t<float, 8>(x, Wg, T, d, E, idx, w, s)
                  : launch_route_t<float, kMaxExperts>(x, Wg, T, d, E, idx, w, s);
}

}  // namespace moe
