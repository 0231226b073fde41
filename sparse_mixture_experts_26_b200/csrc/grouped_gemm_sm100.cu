// grouped_gemm_sm100.cu -- the per-expert SwiGLU FFN on 5th-generation tensor cores.
//
// notion notes "Mixtral of Experts", "Implementation": the expert function is the
// SwiGLU FFN; atlas "Mixtral", "Design overview": inner dimension 14336.  notion
// notes, "Architectural details" mention that single-GPU MoE runs with specialised
// sparse-matmul kernels (Megablocks); this is a grouped GEMM instead: every expert's
// rows are contiguous after the permutation, so each expert is one dense GEMM over
// its own rows, and all experts run in one persistent launch.
//
//   GEMM1 (+SwiGLU):  H[r, n] = silu(x_r . W1[e, n]) * (x_r . W3[e, n])   bf16 out
//   GEMM2:            Y[r, c] = H_r . W2[e, c]                            fp32 out
//
// Both are "TN" products with both operands K-major, the native tcgen05 layout:
//   A = grouped activations [rows, K], B = the expert's weight rows [N, K].
//
// Design (one CTA per SM, persistent, 6 warps):
//   warp 0      TMA producer: 128x64 A tile + (2 NO)x64 or (GEMM2) Wx64 B tile per
//               stage, a ring of shared-memory stages guarded by mbarriers.
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma
//               (M=128, N=2 NO or W, K=16; four per 64-wide K block) into one of
//               two fp32 accumulators 256 columns apart, and commits stage/accumulator
//               barriers.
//   warps 2-5   epilogue: tcgen05.ld the accumulator (one row per thread), apply
//               silu(a)*b (GEMM1) or nothing (GEMM2), store to global, release
//               the accumulator.  The other accumulator is being filled meanwhile.
// For GEMM1 the B tile stacks NO rows of W1 over the same NO rows of W3, so
// accumulator columns [0,NO) hold a and [NO,2 NO) hold b for the same outputs.  NO is
// 128, or 112 when h is a multiple of 112: a batch of 129..511 tokens has one or two
// 128-row blocks per expert, and with Mixtral's h = 14336 the 112 columns give
// 8 x 128 = 1024 tiles (6.9 rounds of 148 SMs, the last one full) instead of
// 8 x 112 = 896 (6.05 rounds, the 7th nearly empty); the smaller stage (44 KiB) also
// lets 5 stages fit instead of 4.  GEMM2's tile width W (256 down to 128 columns) is
// chosen on the device from the number of row blocks, so that the tiles fill whole
// rounds of the grid (gemm2_tile_width below).
//
// Tiles never mix experts' weights: a tile is (expert, 128-row block of that
// expert's rows, output-column block).  A row block may run past the expert's last
// row into the next expert (or past the end, where TMA fills zeros); those rows
// are computed but not stored.  Group sizes are read on the device, so the host
// never waits for the routing.  Every wait is bounded (see sm100_ptx.cuh).
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdio>
#include <mutex>

#include "moe_internal.h"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;        // rows per tile (TMEM lanes)
constexpr int kBK = 64;         // K per stage: one 128-byte swizzle atom of bf16
constexpr int kMmaN = 256;      // accumulator stride (columns) in TMEM
constexpr int kMaxStages = 5;
constexpr int kABytes = kBM * kBK * 2;      // 16 KiB
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr uint32_t kTmemCols = 2 * kMmaN;   // two accumulators: all 512 columns

enum Epilogue { kEpiSwiGLU = 0, kEpiStoreF32 = 1 };

// Shape of one instantiation: GEMM1 tiles cover NO outputs (B = NO W1 rows + NO W3
// rows), GEMM2 tiles up to 256 output columns (the stage holds 256 weight rows).
// Stages fill the shared memory.
template <int EPI, int NO>
struct GemmShape {
    static constexpr int kBRows = EPI == kEpiSwiGLU ? 2 * NO : 256;
    static constexpr int kBBytes = kBRows * kBK * 2;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = (227 * 1024 - 2048) / kStageBytes < kMaxStages
                                       ? (227 * 1024 - 2048) / kStageBytes
                                       : kMaxStages;
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 1024 /*book*/;
    static constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kBRows);
    static_assert(kBRows % 16 == 0 && kBRows <= 256, "MMA N");
    static_assert((NO * kBK * 2) % 1024 == 0, "W3 half of B must start on a swizzle atom");
};

struct GemmArgs {
    const int32_t* offsets;  // [E+1] group row offsets (device)
    int E;
    int rows;           // grouped rows (T*k)
    int K;              // reduction length
    int N;              // output columns
    int b_rows;         // rows of one expert in the flattened weight view [E*b_rows, K]
    int n_tiles;        // output-column tiles per row block
    void* out;          // H (bf16) or Y (fp32), row-major [rows, N]
    uint32_t* status;   // workspace status word
    int cap;            // rows kept per group (capacity; INT_MAX = no limit)
    float* a_out;       // KEEP: a = x W1^T, fp32 [rows, N]
    float* b_out;       // KEEP: b = x W3^T, fp32 [rows, N]
};

struct Bookkeeping {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int off[kMaxExperts + 1];        // sanitised group offsets
    int end[kMaxExperts];            // end of the rows kept in group g (capacity)
    int tile_start[kMaxExperts + 1]; // prefix sum of tiles per group
    int tile_n;                      // output columns per tile (GEMM2: chosen per launch)
    int n_tiles;                     // column tiles per row block
};
static_assert(sizeof(Bookkeeping) <= 1024, "bookkeeping must fit its reserve");

struct TileCoord {
    int e, row0, row_end, nt;
};

__device__ __forceinline__ TileCoord decode_tile(const Bookkeeping& bk, int E, int tile) {
    int g = 0;
    while (g + 1 < E && tile >= bk.tile_start[g + 1]) ++g;
    const int local = tile - bk.tile_start[g];
    const int m_tiles = (bk.end[g] - bk.off[g] + kBM - 1) / kBM;
    TileCoord c;
    c.e = g;
    c.row0 = bk.off[g] + (local % m_tiles) * kBM;  // row blocks inner: weight tile reuse
    c.nt = local / m_tiles;
    c.row_end = bk.end[g];
    return c;
}

// C pre-activations a and b of one row (fp32 bits), kept for the backward pass
// (columns past N are not written; N is a multiple of 8 and C of 16).
template <int C>
__device__ __forceinline__ void keep_pre_activations(const GemmArgs& args, int row, int col0,
                                                     const uint32_t (&a)[C],
                                                     const uint32_t (&b)[C]) {
    float* ar = args.a_out + static_cast<size_t>(row) * args.N;
    float* br = args.b_out + static_cast<size_t>(row) * args.N;
#pragma unroll
    for (int j = 0; j < C / 4; ++j) {
        const int col = col0 + 4 * j;
        if (col < args.N) {
            *reinterpret_cast<float4*>(ar + col) = make_float4(
                bits_f32(a[4 * j]), bits_f32(a[4 * j + 1]), bits_f32(a[4 * j + 2]), bits_f32(a[4 * j + 3]));
            *reinterpret_cast<float4*>(br + col) = make_float4(
                bits_f32(b[4 * j]), bits_f32(b[4 * j + 1]), bits_f32(b[4 * j + 2]), bits_f32(b[4 * j + 3]));
        }
    }
}

// silu(a) * b = a b / (1 + e^-a), with a correctly rounded reciprocal (cheaper than a
// division in the epilogue).
__device__ __forceinline__ float silu_mul(float a, float b) {
    return a * b * __frcp_rn(1.0f + __expf(-a));
}

// GEMM2's weight rows past the first 128 of a tile narrower than 256 columns: tensor
// maps with 32-, 64- and 96-row boxes (unused by GEMM1).
struct W2Tails {
    CUtensorMap box[3];
};

// GEMM2 tile width for `row_blocks` row blocks on `grid` CTAs: each CTA streams its
// tiles' A rows and weight rows from L2, so the time goes as the rounds of tiles a CTA
// runs times the rows one tile streams (128 + width); the narrowest tiles refill the
// rounds that 256-column tiles would leave half empty (e.g. 13 row blocks: 208 tiles
// of 256 columns, two rounds of 148 with 60 CTAs in the second, against 286 tiles of
// 192 columns in two full rounds).
__host__ __device__ inline int gemm2_tile_width(int row_blocks, int N, int grid) {
    int best = 256, best_cost = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 5; ++i) {
        const int w = 256 - 32 * i;  // constant after unrolling: no runtime division by w
        const int tiles = row_blocks * ((N + w - 1) / w);
        const int cost = (tiles + grid - 1) / grid * (128 + w);
        if (cost < best_cost) {
            best_cost = cost;
            best = w;
        }
    }
    return best;
}

// KEEP (kEpiSwiGLU only): also write the pre-activations a, b in fp32 (the training
// forward); a separate instance, so that the plain GEMM1 carries none of that code.
template <int EPI, int NO, bool KEEP = false>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1,
                        const __grid_constant__ W2Tails tails, const GemmArgs args) {
    using S = GemmShape<EPI, NO>;
    constexpr int kStages = S::kStages;
    constexpr int kBBytes = S::kBBytes;
    constexpr int kStageBytes = S::kStageBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages * kABytes;
    Bookkeeping& bk = *reinterpret_cast<Bookkeeping*>(smem + kStages * kStageBytes);
    volatile int* abort_flag = &bk.abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int E = args.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bk.full[s], 1);
            mbar_init(&bk.empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&bk.tmem_full[a], 1);
            mbar_init(&bk.tmem_empty[a], kEpiThreads);
        }
        mbar_init(&bk.drain, 1);
        bk.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB0);
        if (EPI == kEpiSwiGLU) tma_prefetch_desc(&tmB1);
    }
    if (warp == 1) tmem_alloc(&bk.tmem_base, kTmemCols);

    // The routing results come from the previous launch on the stream.
    pdl_wait();
    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        // Offsets are clamped to [0, rows] and made monotone so that nothing below
        // can address rows outside the buffers, whatever the device array holds.
        int prev = 0;
        for (int g = 0; g <= E; ++g) {
            int v = args.offsets[g];
            v = v < prev ? prev : (v > args.rows ? args.rows : v);
            bk.off[g] = v;
            prev = v;
        }
        int row_blocks = 0;
        for (int g = 0; g < E; ++g) {
            const int n = bk.off[g + 1] - bk.off[g];
            bk.end[g] = bk.off[g] + (n < args.cap ? n : args.cap);
            row_blocks += (bk.end[g] - bk.off[g] + kBM - 1) / kBM;
        }
        if (EPI == kEpiSwiGLU) {
            bk.tile_n = NO;
            bk.n_tiles = args.n_tiles;
        } else {
            const int w = gemm2_tile_width(row_blocks, args.N, static_cast<int>(gridDim.x));
            bk.tile_n = w;
            bk.n_tiles = (args.N + w - 1) / w;
        }
        bk.tile_start[0] = 0;
        for (int g = 0; g < E; ++g)
            bk.tile_start[g + 1] =
                bk.tile_start[g] + (bk.end[g] - bk.off[g] + kBM - 1) / kBM * bk.n_tiles;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = bk.tmem_base;
    const int total_tiles = bk.tile_start[E];
    const int tile_n = bk.tile_n;
    const int num_kb = (args.K + kBK - 1) / kBK;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t pending = 0, pending_phase = 0;
            bool ok = true;
            const uint64_t w_policy = l2_policy_evict_first();
            for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
                const TileCoord c = decode_tile(bk, E, tile);
                const int brow = c.e * args.b_rows + c.nt * tile_n;
                // GEMM2: 128 weight rows from the 128-row map, the rest of a narrower
                // tile from the map whose box is that many rows
                const CUtensorMap* tail = tile_n == 256 ? &tmB0
                                          : tile_n > 128 ? &tails.box[(tile_n - 128) / 32 - 1]
                                                         : nullptr;
                const uint32_t tx_bytes =
                    EPI == kEpiSwiGLU ? kStageBytes : kABytes + tile_n * kBK * 2;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait_bounded(&bk.empty[stage], phase ^ 1u, abort_flag,
                                           args.status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bk.full[stage], tx_bytes);
                    const int kc = kb * kBK;
                    uint8_t* a_dst = sA + stage * kABytes;
                    uint8_t* b_dst = sB + stage * kBBytes;
                    tma_load_2d(&tmA, &bk.full[stage], a_dst, kc, c.row0);
                    if (EPI == kEpiSwiGLU) {  // NO-row boxes: W1 rows, then W3 rows
                        // weights first out of L2 (the gathered rows are the reused
                        // operand): GEMM1 1.5-2% faster at 192-256 tokens, GEMM2 not
                        tma_load_2d_hint(&tmB0, &bk.full[stage], b_dst, kc, brow, w_policy);
                        tma_load_2d_hint(&tmB1, &bk.full[stage], b_dst + kBBytes / 2, kc, brow,
                                         w_policy);
                    } else {
                        tma_load_2d(&tmB0, &bk.full[stage], b_dst, kc, brow);
                        if (tail != nullptr)
                            tma_load_2d(tail, &bk.full[stage], b_dst + kBBytes / 2, kc, brow + 128);
                    }
                    pending |= 1u << stage;
                    pending_phase = (pending_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // Let copies already in flight land before the block can exit.
                for (int s = 0; s < kStages; ++s)
                    if (pending & (1u << s)) drain_wait(&bk.full[s], (pending_phase >> s) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true, issued = false;
            const uint32_t idesc = EPI == kEpiSwiGLU ? S::kIdesc : idesc_bf16_f32(kBM, tile_n);
            for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
                if (!mbar_wait_bounded(&bk.tmem_empty[acc], acc_phase ^ 1u, abort_flag,
                                       args.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kMmaN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait_bounded(&bk.full[stage], phase, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + stage * kABytes));
                    const uint64_t bd = sw128_kmajor_desc(smem_u32(sB + stage * kBBytes));
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        umma_bf16(d_tmem, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0);
                    umma_commit(&bk.empty[stage]);
                    issued = true;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(&bk.tmem_full[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (!ok && issued) {
                // Wait for the MMAs still reading shared memory / writing TMEM.
                umma_commit(&bk.drain);
                drain_wait(&bk.drain, 0);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int row_in_tile = q * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
            const TileCoord c = decode_tile(bk, E, tile);
            if (!mbar_wait_bounded(&bk.tmem_full[acc], acc_phase, abort_flag, args.status))
                break;
            tc_fence_after();
            const uint32_t tbase =
                tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kMmaN);
            const int row = c.row0 + row_in_tile;
            const bool valid = row < c.row_end;
            if (EPI == kEpiSwiGLU && NO % 32 != 0) {
                // a in columns [0, NO), b in [NO, 2 NO): 16-column chunks
                __nv_bfloat16* out =
                    static_cast<__nv_bfloat16*>(args.out) + static_cast<size_t>(row) * args.N;
                const int col0 = c.nt * NO;
#pragma unroll 1
                for (int ch = 0; ch < NO / 16; ++ch) {
                    uint32_t a[16], b[16];
                    tmem_ld_16cols(tbase + ch * 16, a);
                    tmem_ld_16cols(tbase + NO + ch * 16, b);
                    tmem_ld_wait();
                    uint32_t p[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        p[i] = pack_bf16x2(silu_mul(bits_f32(a[2 * i]), bits_f32(b[2 * i])),
                                           silu_mul(bits_f32(a[2 * i + 1]), bits_f32(b[2 * i + 1])));
                    if (KEEP && valid) keep_pre_activations<16>(args, row, col0 + ch * 16, a, b);
                    if (valid) {
#pragma unroll
                        for (int v = 0; v < 2; ++v) {
                            const int col = col0 + ch * 16 + v * 8;
                            if (col < args.N)
                                *reinterpret_cast<uint4*>(out + col) =
                                    make_uint4(p[4 * v], p[4 * v + 1], p[4 * v + 2], p[4 * v + 3]);
                        }
                    }
                }
            } else if (EPI == kEpiSwiGLU) {
                __nv_bfloat16* out =
                    static_cast<__nv_bfloat16*>(args.out) + static_cast<size_t>(row) * args.N;
                const int col0 = c.nt * NO;
#pragma unroll 1
                for (int ch = 0; ch < NO / 32; ++ch) {
                    uint32_t a[32], b[32];
                    tmem_ld_32cols(tbase + ch * 32, a);
                    tmem_ld_32cols(tbase + NO + ch * 32, b);
                    tmem_ld_wait();
                    uint32_t p[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        p[i] = pack_bf16x2(silu_mul(bits_f32(a[2 * i]), bits_f32(b[2 * i])),
                                           silu_mul(bits_f32(a[2 * i + 1]), bits_f32(b[2 * i + 1])));
                    if (KEEP && valid) keep_pre_activations<32>(args, row, col0 + ch * 32, a, b);
                    if (valid) {
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const int col = col0 + ch * 32 + v * 8;
                            if (col < args.N)
                                *reinterpret_cast<uint4*>(out + col) =
                                    make_uint4(p[4 * v], p[4 * v + 1], p[4 * v + 2], p[4 * v + 3]);
                        }
                    }
                }
            } else {
                float* out = static_cast<float*>(args.out) + static_cast<size_t>(row) * args.N;
                const int col0 = c.nt * tile_n;
#pragma unroll 1
                for (int ch = 0; ch < tile_n / 32; ++ch) {
                    uint32_t v[32];
                    tmem_ld_32cols(tbase + ch * 32, v);
                    tmem_ld_wait();
                    if (valid) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int col = col0 + ch * 32 + j * 4;
                            if (col < args.N)
                                *reinterpret_cast<float4*>(out + col) =
                                    make_float4(bits_f32(v[4 * j]), bits_f32(v[4 * j + 1]),
                                                bits_f32(v[4 * j + 2]), bits_f32(v[4 * j + 3]));
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&bk.tmem_empty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

template <int EPI, int NO = 128, bool KEEP = false>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const W2Tails& tails, const GemmArgs& args, int grid, cudaStream_t s) {
    auto kern = grouped_gemm_kernel<EPI, NO, KEEP>;
    constexpr int kSmemBytes = GemmShape<EPI, NO>::kSmemBytes;
    static PerDeviceOnce smem_once;
    if (const cudaError_t err = opt_in_smem(smem_once, kern, kSmemBytes); err != cudaSuccess)
        return err;
    return launch_k(kern, grid, kThreads, kSmemBytes, s, a, b0, b1, tails, args);
}

}  // namespace

// ---------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// fp32 tensor [batches, rows, cols] (row-major, contiguous) viewed as 3-D; box =
// box_cols x box_rows x 1 with 128-byte swizzle (box_cols * 4 must be 128 at most).
bool encode_f32_3d(CUtensorMap* map, const void* base, uint64_t batches, uint64_t rows,
                   uint64_t cols, uint32_t box_cols, uint32_t box_rows) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {cols, rows, batches};
    const cuuint64_t strides[2] = {cols * 4, rows * cols * 4};
    const cuuint32_t box[3] = {box_cols, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// Row-major bf16 matrix [rows, cols] viewed as a 2-D tensor; box = 64 columns (one
// 128-byte swizzle span) x box_rows rows, 128-byte swizzle, zero fill out of bounds.
bool encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}


cudaError_t launch_ffn_bf16(const void* x_perm, const int32_t* offsets, const void* W1,
                            const void* W3, const void* W2, int rows, int d, int h, int E,
                            void* H, float* Y, float* partials, int partial_cap, bool reduce,
                            FfnOut* out, uint32_t* status, cudaStream_t s,
                            cudaEvent_t between, uint32_t* counters, int cap, float* a_save,
                            float* b_save) {
    // Small batches stream the weights: the fused cooperative launch up to
    // kFusedMaxRows rows, the two-launch form (no co-residency needed) up to
    // kDecodeMaxRows; above that, or where neither applies, the grouped GEMMs below.
    const bool can_fuse = counters != nullptr && rows <= kFusedMaxRows;
    if (rows <= kDecodeMaxRows || can_fuse) {
        int ksplit = partials ? decode_ksplit(h, partial_cap) : 1;
        float* dst = ksplit > 1 ? partials : Y;
        cudaError_t err;
        err = cudaErrorNotSupported;
        if (can_fuse) {
            err = launch_ffn_bf16_decode_fused(x_perm, offsets, W1, W3, W2, rows, d, h, E, H, dst,
                                               ksplit, counters, status, s, cap, a_save, b_save);
            if (err == cudaErrorCooperativeLaunchTooLarge || err == cudaErrorNotSupported)
                cudaGetLastError();  // clear it: a path below needs no co-residency
            else if (err == cudaSuccess && between)
                err = cudaEventRecord(between, s);
        }
        const bool fallback =
            err == cudaErrorCooperativeLaunchTooLarge || err == cudaErrorNotSupported;
        if (fallback && rows <= kDecodeMaxRows)
            err = launch_ffn_bf16_decode(x_perm, offsets, W1, W3, W2, rows, d, h, E, H, dst,
                                         ksplit, status, s, between, cap);
        if (!fallback || rows <= kDecodeMaxRows) {
            if (err != cudaSuccess) return err;
            if (ksplit > 1 && reduce) {
                err = launch_sum_splits(partials, ksplit, static_cast<size_t>(rows) * d, Y, s);
                if (err != cudaSuccess) return err;
                ksplit = 1;
                dst = Y;
            }
            if (out) {
                *out = FfnOut{dst, ksplit};
                // only the fused launch keeps the pre-activations
                out->saved_ab = can_fuse && !fallback && a_save != nullptr && b_save != nullptr;
            }
            return cudaSuccess;
        }
        // 129..256 rows on a device that cannot co-schedule the fused launch: grouped GEMMs
    }
    if (out) *out = FfnOut{Y, 1};
    if (rows >= kPairMinRows && pair_gemm_enabled()) {
        // the CTA-pair GEMM1 can also keep the pre-activations for the backward pass
        if (out) out->saved_ab = a_save != nullptr && b_save != nullptr;
        return launch_ffn_bf16_pair(x_perm, offsets, W1, W3, W2, rows, d, h, E, H, Y, status, s,
                                    between, cap, a_save, b_save);
    }
    // GEMM1 tile width: 112 outputs where h is a multiple of 112 (see the file comment)
    const int no = h % 112 == 0 ? 112 : 128;
    CUtensorMap mx, mw1, mw3, mh, mw2;
    if (!encode_bf16_2d(&mx, x_perm, rows, d, kBM) ||
        !encode_bf16_2d(&mw1, W1, static_cast<uint64_t>(E) * h, d, no) ||
        !encode_bf16_2d(&mw3, W3, static_cast<uint64_t>(E) * h, d, no) ||
        !encode_bf16_2d(&mh, H, rows, h, kBM) ||
        !encode_bf16_2d(&mw2, W2, static_cast<uint64_t>(E) * d, h, 128))
        return cudaErrorInvalidValue;
    W2Tails tails;
    for (int i = 0; i < 3; ++i)
        if (!encode_bf16_2d(&tails.box[i], W2, static_cast<uint64_t>(E) * d, h, 32 * (i + 1)))
            return cudaErrorInvalidValue;

    const int sms = device_sm_count();
    // Upper bound on row blocks: sum_e ceil(n_e / 128) <= (rows + 127 E) / 128.
    const long long row_blocks = (static_cast<long long>(rows) + 127LL * E) / kBM;

    GemmArgs g1{offsets, E, rows, d, h, h, (h + no - 1) / no, H, status, cap};
    long long tiles1 = row_blocks * g1.n_tiles;
    int grid1 = static_cast<int>(tiles1 < sms ? (tiles1 < 1 ? 1 : tiles1) : sms);
    const bool keep = a_save != nullptr && b_save != nullptr;
    g1.a_out = a_save;
    g1.b_out = b_save;
    if (out) out->saved_ab = keep;
    cudaError_t err =
        keep ? (no == 112 ? launch_gemm<kEpiSwiGLU, 112, true>(mx, mw1, mw3, tails, g1, grid1, s)
                          : launch_gemm<kEpiSwiGLU, 128, true>(mx, mw1, mw3, tails, g1, grid1, s))
             : (no == 112 ? launch_gemm<kEpiSwiGLU, 112>(mx, mw1, mw3, tails, g1, grid1, s)
                          : launch_gemm<kEpiSwiGLU, 128>(mx, mw1, mw3, tails, g1, grid1, s));
    if (err != cudaSuccess) return err;
    if (between && (err = cudaEventRecord(between, s)) != cudaSuccess) return err;

    // GEMM2's tile width is chosen on the device from the row blocks (up to 32 tiles of
    // 128 columns per row block), so the grid covers the narrowest tiling
    GemmArgs g2{offsets, E, rows, h, d, d, (d + 127) / 128, Y, status, cap};
    long long tiles2 = row_blocks * g2.n_tiles;
    int grid2 = static_cast<int>(tiles2 < sms ? (tiles2 < 1 ? 1 : tiles2) : sms);
    return launch_gemm<kEpiStoreF32>(mh, mw2, mw2, tails, g2, grid2, s);
}

}  // namespace moe
