// route.cu -- router logits, top-2 selection and the two-way softmax.
//
// crackai "Mixtral of Experts", "Top-2 Routing in Detail": gate_logits = x . W_gate;
// notion notes "Mixtral of Experts", "Sparse gating", eq. G(x) = Softmax(TopK(x . W_g)).
//
// A block takes TB tokens; its 8 warps split the model dimension d in
// interleaved 32-element chunks, so lanes read consecutive W_g rows (conflict-free,
// coalesced) and each converted weight row is reused for all tokens of the block.
// Every logit is accumulated in fp64: a bf16 x bf16 (or fp32 x fp32) product is
// exact in fp64, so the logits carry only the rounding of the fp64 sums and the
// top-2 choice does not depend on the summation order except at ties closer than
// ~1e-16 relative.  Warp partials are combined by a shuffle tree and then across
// warps in a fixed order, so the result is deterministic.  The kernel reads x once
// (2*d bytes per token); W_g (d*E elements) comes from L2 once per block.
#include <cuda_bf16.h>

#include <cfloat>

#include "moe_internal.h"
#include "sm100_ptx.cuh"

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
constexpr int kRouteWarps = kRouteThreads / 32;
// Loads of kUnroll loop iterations are issued before any of them is used, so each
// warp keeps several memory requests in flight instead of waiting on one at a time.
constexpr int kUnroll = 4;

__device__ __forceinline__ void widen_bf16x8(const uint4& u, double (&wv)[8]) {
    const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        wv[2 * j] = static_cast<double>(__uint_as_float(q[j] << 16));
        wv[2 * j + 1] = static_cast<double>(__uint_as_float(q[j] & 0xffff0000u));
    }
}

// W_g row i (E entries) as fp64, generic E.
template <typename Tin, int MAXE>
__device__ __forceinline__ void load_wrow(const Tin* __restrict__ Wg, int i, int E,
                                          double (&wv)[MAXE]) {
    const Tin* row = Wg + static_cast<size_t>(i) * E;
#pragma unroll
    for (int e = 0; e < MAXE; ++e) wv[e] = e < E ? to_f64(row[e]) : 0.0;
}

// TB tokens per block; 8 warps split d in interleaved 32-element chunks.
template <typename Tin, int MAXE, int TB>
__global__ void __launch_bounds__(kRouteThreads)
    route_kernel(const Tin* __restrict__ x, const Tin* __restrict__ Wg, int T, int d, int E,
                 int32_t* __restrict__ idx, float* __restrict__ w) {
    __shared__ double part[kRouteWarps][TB][MAXE];
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * TB;
    const int ntok = min(TB, T - t0);

    double acc[TB][MAXE];
#pragma unroll
    for (int tb = 0; tb < TB; ++tb)
#pragma unroll
        for (int e = 0; e < MAXE; ++e) acc[tb][e] = 0.0;

    // Fast path: bf16 with exactly 8 experts (one 16-byte W_g row per element).
    constexpr bool kRow16 = (sizeof(Tin) == 2 && MAXE == 8);
    const bool row16 = kRow16 && E == 8;
    for (int i0 = warp * 32 + lane; i0 < d; i0 += kRouteThreads * kUnroll) {
        uint4 wq[kUnroll];
        Tin xv[kUnroll][TB];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = i0 + u * kRouteThreads;
            if (i < d) {
                if (row16) wq[u] = __ldg(reinterpret_cast<const uint4*>(Wg) + i);
#pragma unroll
                for (int tb = 0; tb < TB; ++tb)
                    if (tb < ntok) xv[u][tb] = x[static_cast<size_t>(t0 + tb) * d + i];
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = i0 + u * kRouteThreads;
            if (i < d) {
                double wv[MAXE];
                if constexpr (kRow16) {
                    if (row16)
                        widen_bf16x8(wq[u], reinterpret_cast<double(&)[8]>(wv));
                    else
                        load_wrow<Tin, MAXE>(Wg, i, E, wv);
                } else {
                    load_wrow<Tin, MAXE>(Wg, i, E, wv);
                }
#pragma unroll
                for (int tb = 0; tb < TB; ++tb) {
                    if (tb < ntok) {
                        const double xd = to_f64(xv[u][tb]);
#pragma unroll
                        for (int e = 0; e < MAXE; ++e) acc[tb][e] = fma(xd, wv[e], acc[tb][e]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int tb = 0; tb < TB; ++tb)
#pragma unroll
        for (int e = 0; e < MAXE; ++e) {
            double s = acc[tb][e];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            if (lane == 0) part[warp][tb][e] = s;
        }
    __syncthreads();
    if (threadIdx.x < ntok) {
        const int tb = threadIdx.x;
        double l[MAXE];
#pragma unroll
        for (int e = 0; e < MAXE; ++e) {
            double s = 0.0;
#pragma unroll
            for (int wi = 0; wi < kRouteWarps; ++wi) s += part[wi][tb][e];
            l[e] = s;
        }
        // (logit desc, index asc): strict comparisons keep the first maximum.
        double b1 = l[0];
        int i1 = 0;
#pragma unroll
        for (int e = 1; e < MAXE; ++e)
            if (e < E && l[e] > b1) {
                b1 = l[e];
                i1 = e;
            }
        double b2 = -DBL_MAX;
        int i2 = -1;
#pragma unroll
        for (int e = 0; e < MAXE; ++e)
            if (e < E && e != i1 && (i2 < 0 || l[e] > b2)) {
                b2 = l[e];
                i2 = e;
            }
        const float w1 = static_cast<float>(1.0 / (1.0 + exp(b2 - b1)));
        const int t = t0 + tb;
        idx[2 * t] = i1;
        idx[2 * t + 1] = i2;
        w[2 * t] = w1;
        w[2 * t + 1] = 1.0f - w1;  // exact (Sterbenz): the pair sums to 1 in float
    }
}

template <typename Tin, int MAXE, int TB>
cudaError_t launch_route_tb(const void* x, const void* Wg, int T, int d, int E, int32_t* idx,
                            float* w, cudaStream_t s) {
    const int blocks = (T + TB - 1) / TB;
    return launch_k(route_kernel<Tin, MAXE, TB>, blocks, kRouteThreads, 0, s,
                    static_cast<const Tin*>(x), static_cast<const Tin*>(Wg), T, d, E, idx, w);
}

// Large bf16 batches, E <= 8, d % 32 == 0: fp64 tensor-core MMA.
// mma.sync m8n8k4 .f64 computes D[8x8] += A[8x4] B[4x8] in fp64, so a warp turns 8
// tokens x 8 experts x 4 elements of the dot products into one instruction; every
// widened x value feeds 8 FMAs and every widened W_g value 8 tokens.  Lane (g, q)
// (g = lane/4, q = lane%4) supplies x[token g][8q + s] and W_g[8q + s][expert g] at
// step s of a 32-element K block (the K order inside the block is permuted
// consistently in A and B, which leaves the dot product unchanged), loading each as
// one 16-byte vector.  W_g is staged once per persistent block, transposed to
// [expert][d] in shared memory (64 KiB at d = 4096).  A block is 8 warps = 2 groups
// of 8 tokens x 4 K quarters; the quarters' partial logits are added in a fixed
// order, so results are deterministic.
constexpr int kMmaGroupsPerBlock = 2;
constexpr int kDmmaMinTokens = 512;  // the tensor-core kernel above this many tokens
constexpr int kMmaKSplit = kRouteWarps / kMmaGroupsPerBlock;  // 4

__device__ __forceinline__ void dmma_8x8x4(double& d0, double& d1, double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
                 : "+d"(d0), "+d"(d1)
                 : "d"(a), "d"(b));
}

__device__ __forceinline__ double bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ double bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// With `blk_counts` (zero on entry) the kernel also counts, for every kPermChunk-token
// chunk, the pairs sent to each expert -- the first step of the grouping, so that the
// permutation can skip its own count pass.  Integer atomics: the counts do not depend
// on the order in which they are added.
__global__ void __launch_bounds__(kRouteThreads)
    route_dmma_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ Wg,
                      int T, int d, int E, int32_t* __restrict__ idx, float* __restrict__ w,
                      int32_t* __restrict__ blk_counts) {
    extern __shared__ __align__(16) unsigned char route_smem[];
    __nv_bfloat16* wgT = reinterpret_cast<__nv_bfloat16*>(route_smem);  // [8][d]
    __shared__ double part[kRouteWarps][32][2];
    pdl_wait();
    pdl_launch_dependents();
    if (E == 8) {
        // one 16-byte W_g row (8 experts) per load; kStageUnroll rows per thread in
        // flight before any is stored, so the staging is not a chain of L2 round trips
        constexpr int kStageUnroll = 8;
        const uint4* wg4 = reinterpret_cast<const uint4*>(Wg);
        for (int r0 = threadIdx.x; r0 < d; r0 += kStageUnroll * blockDim.x) {
            uint4 v[kStageUnroll];
#pragma unroll
            for (int u = 0; u < kStageUnroll; ++u) {
                const int r = r0 + u * blockDim.x;
                v[u] = r < d ? __ldg(wg4 + r) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kStageUnroll; ++u) {
                const int r = r0 + u * blockDim.x;
                if (r < d) {
                    const uint32_t q[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        wgT[(2 * j) * d + r] = __ushort_as_bfloat16(static_cast<unsigned short>(q[j] & 0xffffu));
                        wgT[(2 * j + 1) * d + r] = __ushort_as_bfloat16(static_cast<unsigned short>(q[j] >> 16));
                    }
                }
            }
        }
    } else {
        for (int r = threadIdx.x; r < d; r += blockDim.x) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
                wgT[e * d + r] = e < E ? Wg[static_cast<size_t>(r) * E + e] : __float2bfloat16(0.f);
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int grp_in_block = warp / kMmaKSplit, ks = warp % kMmaKSplit;
    const int kq = d / kMmaKSplit;                 // multiple of 8 (d % 32 == 0)
    const int k_begin = ks * kq, k_end = k_begin + kq;
    const int ngroups = (T + 7) / 8;
    const uint4* wrow = reinterpret_cast<const uint4*>(wgT + g * d);
    for (int grp0 = blockIdx.x * kMmaGroupsPerBlock; grp0 < ngroups;
         grp0 += gridDim.x * kMmaGroupsPerBlock) {
        const int grp = grp0 + grp_in_block;
        const int t = grp * 8 + g;
        const bool valid = grp < ngroups && t < T;
        const uint4* xrow = reinterpret_cast<const uint4*>(x + static_cast<size_t>(valid ? t : 0) * d);
        double c0 = 0.0, c1 = 0.0;
        for (int k0 = k_begin; k0 < k_end; k0 += 32 * kUnroll) {
            uint4 xv[kUnroll], wv[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int kk = k0 + u * 32 + 8 * q;
                const bool in = kk < k_end;
                xv[u] = (valid && in) ? __ldg(xrow + kk / 8) : make_uint4(0, 0, 0, 0);
                wv[u] = in ? wrow[kk / 8] : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const uint32_t xa[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
                const uint32_t wa[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    dmma_8x8x4(c0, c1, bf16_lo(xa[j]), bf16_lo(wa[j]));
                    dmma_8x8x4(c0, c1, bf16_hi(xa[j]), bf16_hi(wa[j]));
                }
            }
        }
        // lane (g, q) holds logits of token g for experts 2q and 2q+1 (partial over ks)
        part[warp][lane][0] = c0;
        part[warp][lane][1] = c1;
        __syncthreads();
        if (ks == 0) {  // warp-uniform: all 32 lanes take part in the shuffles
            double v0 = 0.0, v1 = 0.0;
#pragma unroll
            for (int s2 = 0; s2 < kMmaKSplit; ++s2) {
                v0 += part[warp + s2][lane][0];
                v1 += part[warp + s2][lane][1];
            }
            double l[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                l[2 * j] = __shfl_sync(0xffffffffu, v0, (lane & ~3) + j, 32);
                l[2 * j + 1] = __shfl_sync(0xffffffffu, v1, (lane & ~3) + j, 32);
            }
            if (q == 0 && valid) {
                double b1 = l[0];
                int i1 = 0;
#pragma unroll
                for (int e = 1; e < 8; ++e)
                    if (e < E && l[e] > b1) {
                        b1 = l[e];
                        i1 = e;
                    }
                double b2 = -DBL_MAX;
                int i2 = -1;
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (e < E && e != i1 && (i2 < 0 || l[e] > b2)) {
                        b2 = l[e];
                        i2 = e;
                    }
                const float w1 = static_cast<float>(1.0 / (1.0 + exp(b2 - b1)));
                idx[2 * t] = i1;
                idx[2 * t + 1] = i2;
                w[2 * t] = w1;
                w[2 * t + 1] = 1.0f - w1;
                if (blk_counts) {
                    int32_t* c = blk_counts + static_cast<size_t>(t / kPermChunk) * E;
                    atomicAdd(c + i1, 1);
                    atomicAdd(c + i2, 1);
                }
            }
        }
        __syncthreads();
    }
}

// Batches of up to kDmmaMinTokens tokens: one token per block, so the work spreads
// over T SMs.  Larger bf16 batches (E <= 8, d % 32 == 0, W_g fits shared memory): the
// fp64 tensor-core kernel above, whose per-warp K loop only pays for its eight
// dependent load rounds when many tokens share a block (measured, B200: 21 vs 13 us
// for route + grouping at 96 tokens, 25.5 vs 17 us at 256, equal from 1024 on).
// Otherwise: one token per block.
template <typename Tin, int MAXE>
cudaError_t launch_route_t(const void* x, const void* Wg, int T, int d, int E, int32_t* idx,
                           float* w, cudaStream_t s, int32_t* blk_counts) {
    const size_t wgt_bytes = static_cast<size_t>(8) * d * 2;
    if (sizeof(Tin) == 2 && MAXE == 8 && T > kDmmaMinTokens && d % 32 == 0 &&
        wgt_bytes <= 96 * 1024) {
        auto kern = route_dmma_kernel;
        static PerDeviceOnce smem_once;
        if (const cudaError_t err = opt_in_smem(smem_once, kern, 96 * 1024); err != cudaSuccess)
            return err;
        const int blocks_needed = ((T + 7) / 8 + kMmaGroupsPerBlock - 1) / kMmaGroupsPerBlock;
        const int cap = 3 * device_sm_count();
        return launch_k(kern, blocks_needed < cap ? blocks_needed : cap, kRouteThreads, wgt_bytes,
                        s, static_cast<const __nv_bfloat16*>(x),
                        static_cast<const __nv_bfloat16*>(Wg), T, d, E, idx, w, blk_counts);
    }
    if (blk_counts) return cudaErrorInvalidValue;  // the histogram needs the kernel above
    return launch_route_tb<Tin, MAXE, 1>(x, Wg, T, d, E, idx, w, s);
}

}  // namespace

bool dmma_route_applies(int T, int d, int E, moe_dtype dt) {
    return dt == MOE_BF16 && E <= 8 && T > kDmmaMinTokens && d % 32 == 0 &&
           static_cast<size_t>(8) * d * 2 <= 96 * 1024;
}

cudaError_t launch_route(const void* x, const void* Wg, int T, int d, int E, moe_dtype dt,
                         int32_t* idx, float* w, cudaStream_t s, int32_t* blk_counts) {
    if (dt == MOE_BF16) {
        return E <= 8 ? launch_route_t<__nv_bfloat16, 8>(x, Wg, T, d, E, idx, w, s, blk_counts)
                      : launch_route_t<__nv_bfloat16, kMaxExperts>(x, Wg, T, d, E, idx, w, s,
                                                                   blk_counts);
    }
    return E <= 8 ? launch_route_t<float, 8>(x, Wg, T, d, E, idx, w, s, blk_counts)
                  : launch_route_t<float, kMaxExperts>(x, Wg, T, d, E, idx, w, s, blk_counts);
}

}  // namespace moe
