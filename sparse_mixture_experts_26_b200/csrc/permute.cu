// permute.cu -- group the (token, slot) pairs by expert and gather the token rows.
//
// ml-canon "52 Mixtral", "Questions worth asking": tokens spread unevenly over the
// experts and have to be gathered per expert and scattered back; notion notes
// "Mixtral of Experts", "Expert Parallelism": each expert's output is returned to
// the token's original location.
//
// The grouping is a deterministic, stable counting sort over the flattened index
// f = t*k + j, done in four launches with no atomics that decide an order:
//   1. count:  per block of kPermChunk tokens, how many pairs go to each expert (in
//              the layer, the fp64 tensor-core router counts them instead);
//   2. scan:   one block turns the per-block counts into group offsets and the base
//              row of every (block, expert);
//   3. rank:   each block walks its pairs in order, 256 at a time, ranking equal
//              experts with warp match/popc and a per-warp prefix, and writes
//              perm_token / inv_perm;
//   4. gather: each token row is read once (16-byte vectors) and written to its
//              two grouped rows.
// Batches of up to kPermSmallT tokens use one launch instead: every block redoes
// the (tiny) count / scan / rank in shared memory, block 0 publishes it, and each
// block gathers its share of the rows.
#include <cuda_bf16.h>

#include "moe_internal.h"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kPermThreads = 256;
constexpr int kPermWarps = kPermThreads / 32;
constexpr uint32_t kFlagBadIndex = 0x2u;
constexpr int kPermSmallT = kPermSmallTokens;

// Stable ranks of the pairs [f_begin, f_end) in order, 256 at a time: pair f of
// expert e gets row running[e] + (number of earlier pairs of e in this range);
// `emit(f, r)` is called for every valid pair.  running[] is advanced.
template <typename Emit>
__device__ __forceinline__ void rank_range(const int32_t* __restrict__ idx, int f_begin, int f_end,
                                           int E, int* running, int (*warp_cnt)[kMaxExperts],
                                           Emit emit) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned lanemask_lt = (1u << lane) - 1u;
    for (int base = f_begin; base < f_end; base += kPermThreads) {
        const int f = base + threadIdx.x;
        int e = -1;
        if (f < f_end) {
            e = idx[f];
            if (e < 0 || e >= E) e = -1;
        }
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int rank_in_warp = __popc(same & lanemask_lt);
        for (int i = lane; i < E; i += 32) warp_cnt[warp][i] = 0;
        __syncwarp();
        if (e >= 0 && (__ffs(same) - 1) == lane) warp_cnt[warp][e] = __popc(same);
        __syncthreads();
        if (e >= 0) {
            int before = 0;
            for (int w2 = 0; w2 < warp; ++w2) before += warp_cnt[w2][e];
            emit(f, running[e] + before + rank_in_warp);
        }
        __syncthreads();
        if (threadIdx.x < E) {
            int s = 0;
#pragma unroll
            for (int w2 = 0; w2 < kPermWarps; ++w2) s += warp_cnt[w2][threadIdx.x];
            running[threadIdx.x] += s;
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kPermThreads)
    perm_count_kernel(const int32_t* __restrict__ idx, int T, int k, int E,
                      int32_t* __restrict__ blk_counts, uint32_t* status) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ int cnt[kMaxExperts];
    if (threadIdx.x < kMaxExperts) cnt[threadIdx.x] = 0;
    __syncthreads();
    const int t0 = blockIdx.x * kPermChunk;
    const int t1 = min(T, t0 + kPermChunk);
    for (int f = t0 * k + threadIdx.x; f < t1 * k; f += blockDim.x) {
        const int e = idx[f];
        if (e >= 0 && e < E)
            atomicAdd(&cnt[e], 1);
        else if (status)
            atomicOr(status, kFlagBadIndex);
    }
    __syncthreads();
    if (threadIdx.x < E) blk_counts[blockIdx.x * E + threadIdx.x] = cnt[threadIdx.x];
}

// One block of 32 threads: thread e sums expert e's counts over blocks, thread 0
// scans over experts, then thread e writes the base row of each (block, e) and
// clears the counts it read, so that they are zero for a router that accumulates
// them in the next call.
__global__ void perm_scan_kernel(int32_t* __restrict__ blk_counts, int nblk, int E,
                                 int32_t* __restrict__ offsets, int32_t* __restrict__ blk_base) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ int tot[kMaxExperts];
    __shared__ int off[kMaxExperts + 1];
    const int e = threadIdx.x;
    if (e < E) {
        int s = 0;
        for (int b = 0; b < nblk; ++b) s += blk_counts[b * E + e];
        tot[e] = s;
    }
    __syncthreads();
    if (e == 0) {
        int s = 0;
        for (int g = 0; g < E; ++g) {
            off[g] = s;
            s += tot[g];
        }
        off[E] = s;
    }
    __syncthreads();
    if (e < E) offsets[e] = off[e];
    if (e == 0) offsets[E] = off[E];  // E may be 32: no thread E in a block of 32
    if (e < E) {
        int s = off[e];
        for (int b = 0; b < nblk; ++b) {
            blk_base[b * E + e] = s;
            s += blk_counts[b * E + e];
            blk_counts[b * E + e] = 0;
        }
    }
}

__global__ void __launch_bounds__(kPermThreads)
    perm_rank_kernel(const int32_t* __restrict__ idx, int T, int k, int E,
                     const int32_t* __restrict__ blk_base, int32_t* __restrict__ perm_token,
                     int32_t* __restrict__ inv_perm) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ int running[kMaxExperts];
    __shared__ int warp_cnt[kPermWarps][kMaxExperts];
    if (threadIdx.x < E) running[threadIdx.x] = blk_base[blockIdx.x * E + threadIdx.x];
    __syncthreads();
    const int f_begin = blockIdx.x * kPermChunk * k;
    const int f_end = min(T, (blockIdx.x + 1) * kPermChunk) * k;
    rank_range(idx, f_begin, f_end, E, running, warp_cnt, [&](int f, int r) {
        perm_token[r] = f / k;
        inv_perm[f] = r;
    });
}

// Whole permutation of a small batch in one launch (see the file comment).
__global__ void __launch_bounds__(kPermThreads)
    perm_small_kernel(const int32_t* __restrict__ idx, const uint4* __restrict__ x, int T, int k,
                      int E, int vec_per_row, int32_t* __restrict__ offsets,
                      int32_t* __restrict__ perm_token, int32_t* __restrict__ inv_perm,
                      uint4* __restrict__ x_perm, uint32_t* status) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ int cnt[kMaxExperts];
    __shared__ int running[kMaxExperts];
    __shared__ int warp_cnt[kPermWarps][kMaxExperts];
    __shared__ int s_inv[kPermSmallT * 2];
    const int P = T * k;
    const bool publish = blockIdx.x == 0;
    if (threadIdx.x < kMaxExperts) cnt[threadIdx.x] = 0;
    for (int f = threadIdx.x; f < P; f += blockDim.x) s_inv[f] = -1;
    __syncthreads();
    for (int f = threadIdx.x; f < P; f += blockDim.x) {
        const int e = idx[f];
        if (e >= 0 && e < E)
            atomicAdd(&cnt[e], 1);
        else if (publish && status)
            atomicOr(status, kFlagBadIndex);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int g = 0; g < E; ++g) {
            running[g] = acc;
            if (publish) offsets[g] = acc;
            acc += cnt[g];
        }
        if (publish) offsets[E] = acc;
    }
    __syncthreads();
    rank_range(idx, 0, P, E, running, warp_cnt, [&](int f, int r) {
        s_inv[f] = r;
        if (publish) {
            perm_token[r] = f / k;
            inv_perm[f] = r;
        }
    });
    // s_inv is complete (rank_range ends with a barrier); gather this block's tokens.
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        const unsigned r0 = static_cast<unsigned>(s_inv[2 * t]);
        const unsigned r1 = static_cast<unsigned>(s_inv[2 * t + 1]);
        for (int v = threadIdx.x; v < vec_per_row; v += blockDim.x) {
            const uint4 val = x[static_cast<size_t>(t) * vec_per_row + v];
            if (r0 < static_cast<unsigned>(P)) x_perm[static_cast<size_t>(r0) * vec_per_row + v] = val;
            if (r1 < static_cast<unsigned>(P)) x_perm[static_cast<size_t>(r1) * vec_per_row + v] = val;
        }
    }
}

// x_perm[inv[t, j]] = x[t] for j = 0, 1; 16-byte vectors, grid-stride.
__global__ void __launch_bounds__(kPermThreads)
    gather_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ inv, int T,
                       int vec_per_row, uint4* __restrict__ x_perm) {
    pdl_wait();
    pdl_launch_dependents();
    const size_t n = static_cast<size_t>(T) * vec_per_row;
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const size_t t = i / vec_per_row;
        const size_t v = i - t * vec_per_row;
        const uint4 val = x[i];
        const unsigned r0 = static_cast<unsigned>(inv[2 * t]);
        const unsigned r1 = static_cast<unsigned>(inv[2 * t + 1]);
        // Rows outside [0, 2T) only arise from invalid expert ids (flagged by the
        // count kernel); they are skipped rather than written out of bounds.
        if (r0 < 2u * T) x_perm[static_cast<size_t>(r0) * vec_per_row + v] = val;
        if (r1 < 2u * T) x_perm[static_cast<size_t>(r1) * vec_per_row + v] = val;
    }
}

}  // namespace

cudaError_t launch_permute(const int32_t* idx, const void* x, int T, int d, int E, moe_dtype dt,
                           int32_t* offsets, int32_t* perm_token, int32_t* inv_perm,
                           void* x_perm, int32_t* blk_counts, int32_t* blk_base,
                           uint32_t* status, cudaStream_t s, bool counts_ready) {
    const int k = 2;
    const int vec_per_row = static_cast<int>(d * dtype_bytes(dt) / 16);
    if (T <= kPermSmallT) {
        if (counts_ready) return cudaErrorInvalidValue;  // the one-launch form counts itself
        const int grid = T < 2 * device_sm_count() ? T : 2 * device_sm_count();
        return launch_k(perm_small_kernel, grid, kPermThreads, 0, s, idx,
                        static_cast<const uint4*>(x), T, k, E, vec_per_row, offsets, perm_token,
                        inv_perm, static_cast<uint4*>(x_perm), status);
    }
    const int nblk = perm_blocks(T);
    cudaError_t err = cudaSuccess;
    if (!counts_ready)  // otherwise the router has counted
        err = launch_k(perm_count_kernel, nblk, kPermThreads, 0, s, idx, T, k, E, blk_counts,
                       status);
    if (err == cudaSuccess)
        err = launch_k(perm_scan_kernel, 1, 32, 0, s, blk_counts, nblk, E, offsets, blk_base);
    if (err == cudaSuccess)
        err = launch_k(perm_rank_kernel, nblk, kPermThreads, 0, s, idx, T, k, E,
                       static_cast<const int32_t*>(blk_base), perm_token, inv_perm);
    if (err != cudaSuccess) return err;
    const size_t nvec = static_cast<size_t>(T) * vec_per_row;
    size_t blocks = (nvec + kPermThreads - 1) / kPermThreads;
    const size_t cap = static_cast<size_t>(device_sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return launch_k(gather_rows_kernel, static_cast<unsigned>(blocks), kPermThreads, 0, s,
                    static_cast<const uint4*>(x), static_cast<const int32_t*>(inv_perm), T,
                    vec_per_row, static_cast<uint4*>(x_perm));
}

}  // namespace moe
