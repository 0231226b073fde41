// grouped_gemm_pair_sm100.cu -- the per-expert SwiGLU FFN for large batches on pairs of
// SMs (tcgen05 cta_group::2).
//
// Same computation as grouped_gemm_sm100.cu (notion notes "Mixtral of Experts",
// "Implementation": SwiGLU expert function; atlas "Mixtral", "Design overview"):
//   GEMM1 (+SwiGLU):  H[r, n] = silu(x_r . W1[e, n]) * (x_r . W3[e, n])   bf16 out
//   GEMM2:            Y[r, c] = H_r . W2[e, c]                            fp32 out
// but each tile is computed by a cluster of two CTAs on two SMs.  One thread of the
// leader CTA issues tcgen05.mma.cta_group::2 with M = 256 rows (128 from each CTA's
// shared memory) and N = 256 columns whose B operand is split between the CTAs
// (128 rows of B each); each CTA's tensor memory receives its 128 rows x 256
// columns.  Per SM this halves the B bytes staged per K block (32 KiB per stage
// instead of 48 KiB for the same math), which leaves room for 6 or 7 pipeline stages
// and cuts the L2->SM traffic by a third.
//
// GEMM1 covers 128 outputs n0 .. n0+127 per tile.  Each CTA stages 64 W1 rows and
// the same 64 W3 rows (the leader outputs n0 .. n0+63, the peer n0+64 .. n0+127), so
// accumulator columns [0,64) hold a = x.W1 and [64,128) b = x.W3 for the leader's
// outputs and [128,192) / [192,256) the same for the peer's: every thread finds the a
// and b of an output in its own TMEM lane, in both tile modes below.
//
// An expert's rows are covered by 256-row blocks; a last block with at most 128 rows
// is issued with M = 128 (64 rows per CTA) so that no more rows are wasted than with
// 128-row tiles.  In that mode the accumulator uses the "2x2" data-path layout:
// columns 0..127 of the tile in TMEM lanes 0..63 and columns 128..255 in lanes
// 64..127, both in the first 128 TMEM columns of the buffer.
//
// Pipeline depth: GEMM1 keeps 7 stages (224 KiB).  The fp32-output GEMMs (GEMM2 and
// the backward's dH and dX) keep 6 and use the rest for their store epilogue: each
// epilogue warp stages 32 rows x 32 columns of its accumulator rows in shared memory
// (128-byte swizzle) and one lane writes them with a TMA tensor store, so every row
// segment leaves as whole 128-byte lines instead of 16-byte pieces from 32 rows at a
// time.  A chunk whose 32 rows are not all inside the expert's group (the last block
// of a group, whose further rows belong to the next expert) is stored row by row.
// The backward SwiGLU step, whose half-tile epilogue exchanges b through shared
// memory, keeps 6 stages.
//
// Synchronisation: both CTAs' TMA loads count their bytes on the leader's "full"
// barrier; the leader's MMA completions are multicast to both CTAs' "empty" and
// "tmem_full" barriers; both CTAs' epilogues arrive on the leader's "tmem_empty"
// barrier.  Every wait is bounded; a CTA that gives up raises the status flag.
#include <cuda.h>
#include <cuda_bf16.h>

#include "moe_internal.h"
#include "sm100_ptx.cuh"

namespace moe {

// Defined in grouped_gemm_sm100.cu.
bool encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows);
bool encode_f32_3d(CUtensorMap* map, const void* base, uint64_t batches, uint64_t rows,
                   uint64_t cols, uint32_t box_cols, uint32_t box_rows);

namespace {

constexpr int kRowsPerCta = 128;
constexpr int kPairRows = 2 * kRowsPerCta;   // rows per full pair tile
constexpr int kBK = 64;
constexpr int kN = 256;                      // accumulator columns per tile
constexpr int kMaxStages = 7;
constexpr int kABytes = kRowsPerCta * kBK * 2;  // 16 KiB
constexpr int kBBytes = 128 * kBK * 2;          // 16 KiB: this CTA's half of B
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr uint32_t kTmemCols = 2 * kN;
constexpr uint32_t kIdescFull = idesc_bf16_f32(2 * kRowsPerCta, kN);
constexpr uint32_t kIdescHalf = idesc_bf16_f32(kRowsPerCta, kN);
constexpr int kXferBytes = 32 * 64 * 4;  // one 32-column chunk of b for 64 rows
constexpr int kXferBarrier = 1;
constexpr int kVoteBarrier = 2;  // epilogue vote after a bounded wait
constexpr uint16_t kBothCtas = 0x3;

// kEpiBwdSwiGLU (backward pass): the accumulator holds a = x.W1 and b = x.W3 as for
// kEpiSwiGLU; with g = dH of the same outputs the epilogue writes du = g b silu'(a)
// and dv = g silu(a) (bf16, row stride 2N: du in columns [0, N), dv in [N, 2N)).
enum Epilogue { kEpiSwiGLU = 0, kEpiStoreF32 = 1, kEpiBwdSwiGLU = 2 };

// fp32 store staging: per epilogue warp two 32 x 32 fp32 chunks (4 KiB each).
constexpr int kOutChunkBytes = 32 * 32 * 4;
constexpr int kOutBufs = 2;
constexpr int kOutStageBytes = (kEpiThreads / 32) * kOutBufs * kOutChunkBytes;

// Pipeline depth and shared memory of each epilogue kind.
__host__ __device__ constexpr int stages_of(int epi) { return epi == kEpiSwiGLU ? 7 : 6; }
__host__ __device__ constexpr int smem_bytes_of(int epi) {
    return stages_of(epi) * kStageBytes + 1024 /*align*/ + 1024 /*bookkeeping*/ +
           (epi == kEpiBwdSwiGLU ? kXferBytes : epi == kEpiStoreF32 ? kOutStageBytes : 0);
}
static_assert(smem_bytes_of(kEpiStoreF32) <= 227 * 1024, "shared memory per CTA");
static_assert(smem_bytes_of(kEpiSwiGLU) <= 227 * 1024, "shared memory per CTA");
static_assert(smem_bytes_of(kEpiBwdSwiGLU) <= 227 * 1024, "shared memory per CTA");
// B operand: K-major weight rows (the forward), or MN-major (weights [K, N] read as
// 64 x 64 boxes; backward dH = dY W2), optionally taken from W1 for k < h and from W3
// for k >= h (backward dX = [du dv] [W1; W3]).
enum BOperand { kBKMajor = 0, kBMn = 1, kBMnSplit = 2 };
constexpr int kBoxMn = kMnBoxBytes;  // one 64 x 64 bf16 box of an MN-major operand

struct PairArgs {
    const int32_t* offsets;
    int E;
    int rows;
    int K;
    int N;        // output columns
    int b_rows;   // rows of one expert in the flattened weight view
    int n_tiles;  // column tiles per row block
    void* out;
    uint32_t* status;
    int cap;      // rows kept per group (capacity; INT_MAX = no limit)
    int h;             // kBMnSplit: the K index where W3 takes over from W1
    const float* dH;   // kEpiBwdSwiGLU: dH fp32 [rows, N]
    int group;         // row blocks whose A rows stay in L2 together (tile order)
    // kEpiSwiGLU with KEEP: the pre-activations a = x W1^T and b = x W3^T, fp32
    // [rows, N] each, kept for the backward pass
    float* a_out;
    float* b_out;
    // optional: the launch does nothing when bit 7 of this device byte is set (the
    // backward's recompute of a and b, when the forward kept them)
    const uint8_t* skip_flag;
};

struct PairBook {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int off[kMaxExperts + 1];
    int end[kMaxExperts];
    int tile_start[kMaxExperts + 1];
};
static_assert(sizeof(PairBook) <= 1024, "bookkeeping reserve");

struct PairTile {
    int e, row0, row_end, nt;
    bool half;
};

// Tile order inside an expert: row blocks in groups of `group` (the last group may be
// smaller); a group's tiles run column tile by column tile with its row blocks
// innermost.  Concurrent pairs then share each weight tile (read from DRAM once) and
// a group's A rows (sized on the host to fit L2 with room to spare) are read from DRAM
// once for all column tiles; an expert with at most `group` row blocks runs in plain
// column-major order.
__device__ __forceinline__ PairTile decode_pair_tile(const PairBook& bk, int E, int tile,
                                                    int n_tiles, int group) {
    int g = 0;
    while (g + 1 < E && tile >= bk.tile_start[g + 1]) ++g;
    const int local = tile - bk.tile_start[g];
    const int blocks = (bk.end[g] - bk.off[g] + kPairRows - 1) / kPairRows;
    const int full = blocks / group;                // complete row-block groups
    const int per_full = group * n_tiles;
    int rb, nt;
    if (local < full * per_full) {
        const int r = local % per_full;
        rb = (local / per_full) * group + r % group;
        nt = r / group;
    } else {
        const int rem = blocks - full * group;      // > 0 here
        const int r = local - full * per_full;
        rb = full * group + r % rem;
        nt = r / rem;
    }
    PairTile t;
    t.e = g;
    t.row0 = bk.off[g] + rb * kPairRows;
    t.nt = nt;
    t.row_end = bk.end[g];
    t.half = t.row_end - t.row0 <= kRowsPerCta;
    return t;
}

// silu(a) * b = a b / (1 + e^-a), with a correctly rounded reciprocal instead of a
// division: the division's slow path (one warp per scheduler, no latency hiding) made
// the epilogue, not the tensor cores, set GEMM1's pace at full clock.
__device__ __forceinline__ float silu_mul(float a, float b) {
    return a * b * __frcp_rn(1.0f + __expf(-a));
}

// du = g b silu'(a), dv = g silu(a) for one output of the backward SwiGLU step.
__device__ __forceinline__ void bwd_swiglu(float a, float b, float g, float& du, float& dv) {
    const float s = __frcp_rn(1.0f + __expf(-a));
    du = g * b * (s * (1.0f + a * (1.0f - s)));
    dv = g * (a * s);
}

// The 32 pre-activations a and b of one row that a GEMM1 epilogue chunk holds, kept in
// fp32 for the backward pass (columns past N are not written).
__device__ __forceinline__ void store_pre_activations(const PairArgs& args, int row, int col0,
                                                      const uint32_t (&a)[32],
                                                      const uint32_t (&b)[32]) {
    float* ar = args.a_out + static_cast<size_t>(row) * args.N;
    float* br = args.b_out + static_cast<size_t>(row) * args.N;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int col = col0 + 4 * j;
        if (col < args.N) {
            *reinterpret_cast<float4*>(ar + col) = make_float4(
                bits_f32(a[4 * j]), bits_f32(a[4 * j + 1]), bits_f32(a[4 * j + 2]), bits_f32(a[4 * j + 3]));
            *reinterpret_cast<float4*>(br + col) = make_float4(
                bits_f32(b[4 * j]), bits_f32(b[4 * j + 1]), bits_f32(b[4 * j + 2]), bits_f32(b[4 * j + 3]));
        }
    }
}

// KEEP (kEpiSwiGLU only): also write the pre-activations a, b (moe_layer_forward_train);
// a separate instance, so that the plain GEMM1 carries none of that code.
template <int EPI, int BOP = kBKMajor, bool KEEP = false>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmB0,
                             const __grid_constant__ CUtensorMap tmB1,
                             const __grid_constant__ CUtensorMap tmOut, const PairArgs args) {
    constexpr int kStages = stages_of(EPI);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages * kABytes;
    PairBook& bk = *reinterpret_cast<PairBook*>(smem + kStages * kStageBytes);
    // exchange buffer of the backward SwiGLU half-tile epilogue (kEpiBwdSwiGLU), or the
    // fp32 store staging (kEpiStoreF32)
    float* xfer = reinterpret_cast<float*>(smem + kStages * kStageBytes + 1024);
    uint8_t* out_stage = smem + kStages * kStageBytes + 1024;
    volatile int* abort_flag = &bk.abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int E = args.E;
    const uint32_t rank = cluster_ctarank();  // 0 = leader, 1 = peer
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    // Both CTAs of every pair read the same byte, so a skipped launch leaves together
    // before any barrier, cluster synchronisation or tensor-memory allocation.
    if (args.skip_flag != nullptr && (*args.skip_flag & 0x80u) != 0) return;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bk.full[s], 1);
            mbar_init(&bk.empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&bk.tmem_full[a], 1);
            mbar_init(&bk.tmem_empty[a], 2 * kEpiThreads);
        }
        mbar_init(&bk.drain, 1);
        bk.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB0);
        if (EPI != kEpiStoreF32 || BOP == kBMnSplit) tma_prefetch_desc(&tmB1);
        if (EPI == kEpiStoreF32) tma_prefetch_desc(&tmOut);
    }
    if (warp == 1) tmem_alloc_pair(&bk.tmem_base, kTmemCols);

    pdl_wait();
    if (threadIdx.x == 0) {
        int prev = 0;
        for (int g = 0; g <= E; ++g) {
            int v = args.offsets[g];
            v = v < prev ? prev : (v > args.rows ? args.rows : v);
            bk.off[g] = v;
            prev = v;
        }
        bk.tile_start[0] = 0;
        for (int g = 0; g < E; ++g) {
            const int n = bk.off[g + 1] - bk.off[g];
            bk.end[g] = bk.off[g] + (n < args.cap ? n : args.cap);
            bk.tile_start[g + 1] = bk.tile_start[g] +
                                   (bk.end[g] - bk.off[g] + kPairRows - 1) / kPairRows *
                                       args.n_tiles;
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers are initialised before either signals the other
    tc_fence_after();

    const uint32_t tmem_base = bk.tmem_base;
    const int total = bk.tile_start[E];
    const int num_kb = (args.K + kBK - 1) / kBK;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t pending = 0, pending_phase = 0;
            bool ok = true, issued = false;
            // kEpiBwdSwiGLU: B = [128 W1 rows (leader) | the same 128 W3 rows (peer)]
            constexpr bool kStacked = EPI == kEpiBwdSwiGLU;
            const CUtensorMap* tmB = (kStacked && !leader) ? &tmB1 : &tmB0;
            for (int tile = pair; ok && tile < total; tile += npairs) {
                const PairTile t = decode_pair_tile(bk, E, tile, args.n_tiles, args.group);
                const int a_row = t.row0 + static_cast<int>(rank) * (t.half ? 64 : kRowsPerCta);
                const int b_row =
                    EPI == kEpiSwiGLU
                        ? t.e * args.b_rows + t.nt * 128 + static_cast<int>(rank) * 64
                        : t.e * args.b_rows + t.nt * (kStacked ? 128 : 256) +
                              (kStacked ? 0 : static_cast<int>(rank) * 128);
                const int b_col = t.nt * 256 + static_cast<int>(rank) * 128;  // MN-major B
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait_bounded(&bk.empty[stage], phase ^ 1u, abort_flag,
                                           args.status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full_leader = map_to_cta(smem_u32(&bk.full[stage]), 0);
                    if (leader) mbar_arrive_expect_tx(&bk.full[stage], 2 * kStageBytes);
                    const int kc = kb * kBK;
                    tma_load_2d_pair(&tmA, full_leader, sA + stage * kABytes, kc, a_row);
                    if (EPI == kEpiSwiGLU) {
                        // 64 W1 rows, then the same 64 W3 rows (64-row boxes)
                        tma_load_2d_pair(&tmB0, full_leader, sB + stage * kBBytes, kc, b_row);
                        tma_load_2d_pair(&tmB1, full_leader, sB + stage * kBBytes + kBBytes / 2,
                                         kc, b_row);
                    } else if (BOP == kBKMajor) {
                        tma_load_2d_pair(tmB, full_leader, sB + stage * kBBytes, kc, b_row);
                    } else {
                        const CUtensorMap* mb = &tmB0;
                        int krow = t.e * args.b_rows + kc;
                        if (BOP == kBMnSplit) {
                            const bool second = kc >= args.h;
                            mb = second ? &tmB1 : &tmB0;
                            krow = t.e * args.h + (second ? kc - args.h : kc);
                        }
                        tma_load_2d_pair(mb, full_leader, sB + stage * kBBytes, b_col, krow);
                        tma_load_2d_pair(mb, full_leader, sB + stage * kBBytes + kBoxMn,
                                         b_col + 64, krow);
                    }
                    issued = true;
                    pending |= 1u << stage;
                    pending_phase = (pending_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok && issued) {
                if (leader) {
                    for (int s = 0; s < kStages; ++s)
                        if (pending & (1u << s)) drain_wait(&bk.full[s], (pending_phase >> s) & 1u);
                } else {
                    // The peer's copies complete on the leader's barriers; give them
                    // time to land before this CTA's shared memory can be released.
                    short_pause_ns(2000000ull);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (lane == 0 && leader) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true, issued = false;
            for (int tile = pair; ok && tile < total; tile += npairs) {
                const PairTile t = decode_pair_tile(bk, E, tile, args.n_tiles, args.group);
                constexpr uint32_t kBT = BOP == kBKMajor ? 0u : (1u << 16);  // B MN-major
                const uint32_t idesc = (t.half ? kIdescHalf : kIdescFull) | kBT;
                if (!mbar_wait_bounded(&bk.tmem_empty[acc], acc_phase ^ 1u, abort_flag,
                                       args.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait_bounded(&bk.full[stage], phase, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + stage * kABytes));
                    const uint32_t bs = smem_u32(sB + stage * kBBytes);
                    const uint64_t bd = BOP == kBKMajor ? sw128_kmajor_desc(bs) : sw128_mn_desc(bs);
                    constexpr uint64_t kBStep = BOP == kBKMajor ? kKDescStep : kMnDescStep;
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        umma_bf16_pair(d_tmem, ad + 2 * k, bd + kBStep * k, idesc, (kb | k) != 0);
                    umma_commit_pair(&bk.empty[stage], kBothCtas);
                    issued = true;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit_pair(&bk.tmem_full[acc], kBothCtas);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (!ok && issued) {
                umma_commit_pair(&bk.drain, 0x1);
                drain_wait(&bk.drain, 0);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        uint8_t* wstage = out_stage + q * kOutBufs * kOutChunkBytes;  // this warp's staging
        int obuf = 0;
        const uint32_t empty_leader0 = map_to_cta(smem_u32(&bk.tmem_empty[0]), 0);
        const uint32_t empty_leader1 = map_to_cta(smem_u32(&bk.tmem_empty[1]), 0);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = pair; tile < total; tile += npairs) {
            const PairTile t = decode_pair_tile(bk, E, tile, args.n_tiles, args.group);
            if (!bar_all(mbar_wait_bounded(&bk.tmem_full[acc], acc_phase, abort_flag, args.status),
                         kVoteBarrier, kEpiThreads))
                break;
            tc_fence_after();
            const uint32_t tlane = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(acc * kN);
            if (!t.half) {
                const int row = t.row0 + static_cast<int>(rank) * kRowsPerCta + q * 32 + lane;
                const bool valid = row < t.row_end;
                if (EPI == kEpiSwiGLU) {
                    __nv_bfloat16* out =
                        static_cast<__nv_bfloat16*>(args.out) + static_cast<size_t>(row) * args.N;
                    const int col0 = t.nt * 128;
                    // chunk c: outputs col0 + 32c .. +31, a in accumulator column
                    // (c / 2) * 128 + (c % 2) * 32, b 64 columns further
#pragma unroll 1
                    for (int ch = 0; ch < 4; ++ch) {
                        const uint32_t ca = static_cast<uint32_t>((ch >> 1) * 128 + (ch & 1) * 32);
                        uint32_t a[32], b[32];
                        tmem_ld_32cols(tlane + ca, a);
                        tmem_ld_32cols(tlane + ca + 64, b);
                        tmem_ld_wait();
                        uint32_t p[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            p[i] = pack_bf16x2(silu_mul(bits_f32(a[2 * i]), bits_f32(b[2 * i])),
                                               silu_mul(bits_f32(a[2 * i + 1]), bits_f32(b[2 * i + 1])));
                        if (valid) {
#pragma unroll
                            for (int v = 0; v < 4; ++v) {
                                const int col = col0 + ch * 32 + v * 8;
                                if (col < args.N)
                                    *reinterpret_cast<uint4*>(out + col) =
                                        make_uint4(p[4 * v], p[4 * v + 1], p[4 * v + 2], p[4 * v + 3]);
                            }
                            if (KEEP)
                                store_pre_activations(args, row, col0 + ch * 32, a, b);
                        }
                    }
                } else if (EPI == kEpiBwdSwiGLU) {
                    // du, dv for this row's 128 outputs (N = h is a multiple of 64)
                    const int N = args.N;
                    __nv_bfloat16* duv =
                        static_cast<__nv_bfloat16*>(args.out) + static_cast<size_t>(row) * 2 * N;
                    const float* g = args.dH + static_cast<size_t>(row) * N;
                    const int col0 = t.nt * 128;
#pragma unroll 1
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t a[32], b[32];
                        tmem_ld_32cols(tlane + ch * 32, a);
                        tmem_ld_32cols(tlane + 128 + ch * 32, b);
                        tmem_ld_wait();
                        const int c0 = col0 + ch * 32;
                        if (valid && c0 < N) {
                            float gv[32];
#pragma unroll
                            for (int v = 0; v < 8; ++v) {
                                const float4 t4 = *reinterpret_cast<const float4*>(g + c0 + 4 * v);
                                gv[4 * v] = t4.x;
                                gv[4 * v + 1] = t4.y;
                                gv[4 * v + 2] = t4.z;
                                gv[4 * v + 3] = t4.w;
                            }
                            uint32_t pu[16], pv[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                float u0, v0, u1, v1;
                                bwd_swiglu(bits_f32(a[2 * i]), bits_f32(b[2 * i]), gv[2 * i], u0, v0);
                                bwd_swiglu(bits_f32(a[2 * i + 1]), bits_f32(b[2 * i + 1]),
                                           gv[2 * i + 1], u1, v1);
                                pu[i] = pack_bf16x2(u0, u1);
                                pv[i] = pack_bf16x2(v0, v1);
                            }
#pragma unroll
                            for (int v = 0; v < 4; ++v) {
                                *reinterpret_cast<uint4*>(duv + c0 + 8 * v) =
                                    make_uint4(pu[4 * v], pu[4 * v + 1], pu[4 * v + 2], pu[4 * v + 3]);
                                *reinterpret_cast<uint4*>(duv + N + c0 + 8 * v) =
                                    make_uint4(pv[4 * v], pv[4 * v + 1], pv[4 * v + 2], pv[4 * v + 3]);
                            }
                        }
                    }
                } else {
                    float* out = static_cast<float*>(args.out) + static_cast<size_t>(row) * args.N;
                    const int col0 = t.nt * 256;
                    const int wrow0 = t.row0 + static_cast<int>(rank) * kRowsPerCta + q * 32;
                    const bool whole = wrow0 + 32 <= t.row_end;  // all 32 rows in the group
#pragma unroll 1
                    for (int ch = 0; ch < 8; ++ch) {
                        uint32_t v[32];
                        tmem_ld_32cols(tlane + ch * 32, v);
                        tmem_ld_wait();
                        if (col0 + ch * 32 >= args.N) continue;
                        if (whole) {
                            // TMA store of 32 rows x 32 columns (columns past N are outside
                            // the tensor and not written)
                            uint8_t* st = wstage + obuf * kOutChunkBytes;
                            if (lane == 0) bulk_wait_group_read<kOutBufs - 1>();
                            __syncwarp();
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                *reinterpret_cast<uint4*>(st + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                                    make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                tma_store_3d(&tmOut, st, col0 + ch * 32, wrow0, 0);
                                bulk_commit_group();
                            }
                            if (++obuf == kOutBufs) obuf = 0;
                        } else if (valid) {
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
            } else {
                // 64 rows per CTA; lanes 0..63 hold tile columns 0..127 and lanes 64..127
                // hold columns 128..255, both in TMEM columns 0..127 of the buffer.
                const int m = (q & 1) * 32 + lane;
                const int row = t.row0 + static_cast<int>(rank) * 64 + m;
                const bool valid = row < t.row_end;
                const bool upper = q >= 2;  // holds tile columns 128..255
                if (EPI == kEpiSwiGLU) {
                    // lanes 0..63 hold the leader's 64 outputs (a in columns 0..63, b in
                    // 64..127), lanes 64..127 the peer's: each thread writes 64 outputs
                    __nv_bfloat16* out =
                        static_cast<__nv_bfloat16*>(args.out) + static_cast<size_t>(row) * args.N;
                    const int col0 = t.nt * 128 + (upper ? 64 : 0);
#pragma unroll 1
                    for (int ch = 0; ch < 2; ++ch) {
                        uint32_t a[32], b[32];
                        tmem_ld_32cols(tlane + ch * 32, a);
                        tmem_ld_32cols(tlane + 64 + ch * 32, b);
                        tmem_ld_wait();
                        if (valid) {
                            uint32_t p[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                p[i] = pack_bf16x2(silu_mul(bits_f32(a[2 * i]), bits_f32(b[2 * i])),
                                                   silu_mul(bits_f32(a[2 * i + 1]),
                                                            bits_f32(b[2 * i + 1])));
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const int col = col0 + ch * 32 + u * 8;
                                if (col < args.N)
                                    *reinterpret_cast<uint4*>(out + col) =
                                        make_uint4(p[4 * u], p[4 * u + 1], p[4 * u + 2], p[4 * u + 3]);
                            }
                            if (KEEP)
                                store_pre_activations(args, row, col0 + ch * 32, a, b);
                        }
                    }
                } else if (EPI == kEpiBwdSwiGLU) {
                    const int N = args.N;
                    __nv_bfloat16* duv =
                        static_cast<__nv_bfloat16*>(args.out) + static_cast<size_t>(row) * 2 * N;
                    const float* g = args.dH + static_cast<size_t>(row) * N;
                    const int col0 = t.nt * 128;
#pragma unroll 1
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t v[32];
                        tmem_ld_32cols(tlane + ch * 32, v);
                        tmem_ld_wait();
                        if (upper) {  // b for rows m, columns ch*32 .. ch*32+31
#pragma unroll
                            for (int j = 0; j < 32; ++j) xfer[j * 64 + m] = bits_f32(v[j]);
                        }
                        asm volatile("bar.sync %0, %1;" ::"r"(kXferBarrier), "r"(kEpiThreads)
                                     : "memory");
                        const int c0 = col0 + ch * 32;
                        if (!upper && valid && c0 < N) {
                            uint32_t pu[16], pv[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                float u0, v0, u1, v1;
                                bwd_swiglu(bits_f32(v[2 * i]), xfer[(2 * i) * 64 + m],
                                           g[c0 + 2 * i], u0, v0);
                                bwd_swiglu(bits_f32(v[2 * i + 1]), xfer[(2 * i + 1) * 64 + m],
                                           g[c0 + 2 * i + 1], u1, v1);
                                pu[i] = pack_bf16x2(u0, u1);
                                pv[i] = pack_bf16x2(v0, v1);
                            }
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                *reinterpret_cast<uint4*>(duv + c0 + 8 * u) =
                                    make_uint4(pu[4 * u], pu[4 * u + 1], pu[4 * u + 2], pu[4 * u + 3]);
                                *reinterpret_cast<uint4*>(duv + N + c0 + 8 * u) =
                                    make_uint4(pv[4 * u], pv[4 * u + 1], pv[4 * u + 2], pv[4 * u + 3]);
                            }
                        }
                        asm volatile("bar.sync %0, %1;" ::"r"(kXferBarrier), "r"(kEpiThreads)
                                     : "memory");
                    }
                } else {
                    float* out = static_cast<float*>(args.out) + static_cast<size_t>(row) * args.N;
                    const int col0 = t.nt * 256 + (upper ? 128 : 0);
#pragma unroll 1
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t v[32];
                        tmem_ld_32cols(tlane + ch * 32, v);
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
            }
            tc_fence_before();
            mbar_arrive_cluster(acc == 0 ? empty_leader0 : empty_leader1);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (EPI == kEpiStoreF32 && lane == 0)
            bulk_wait_group<0>();  // every tensor store complete before the block exits
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the leader's MMAs into this CTA's TMEM are done on both sides
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

template <int EPI, int BOP = kBKMajor, bool KEEP = false>
cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const CUtensorMap& o, const PairArgs& args, int npairs, cudaStream_t s) {
    auto kern = grouped_gemm_pair_kernel<EPI, BOP, KEEP>;
    constexpr int kSmemBytes = smem_bytes_of(EPI);
    // Row blocks per tile-order group: A rows of at most ~64 MB (a half of L2) per group.
    PairArgs a2 = args;
    const long long a_block_bytes = static_cast<long long>(kPairRows) * args.K * 2;
    const long long g = (64LL << 20) / (a_block_bytes > 0 ? a_block_bytes : 1);
    a2.group = static_cast<int>(g < 1 ? 1 : (g > 1024 ? 1024 : g));
    static PerDeviceOnce smem_once;
    if (const cudaError_t err = opt_in_smem(smem_once, kern, kSmemBytes); err != cudaSuccess)
        return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * npairs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, kern, a, b0, b1, o, a2);
    return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace

// Large-batch expert FFN on CTA pairs (both GEMMs).
cudaError_t launch_ffn_bf16_pair(const void* x_perm, const int32_t* offsets, const void* W1,
                                 const void* W3, const void* W2, int rows, int d, int h, int E,
                                 void* H, float* Y, uint32_t* status, cudaStream_t s,
                                 cudaEvent_t between, int cap, float* a_out, float* b_out) {
    CUtensorMap mx, mw1, mw3, mh, mw2, my;
    if (!encode_f32_3d(&my, Y, 1, rows, d, 32, 32) ||
        !encode_bf16_2d(&mx, x_perm, rows, d, kRowsPerCta) ||
        !encode_bf16_2d(&mw1, W1, static_cast<uint64_t>(E) * h, d, 64) ||
        !encode_bf16_2d(&mw3, W3, static_cast<uint64_t>(E) * h, d, 64) ||
        !encode_bf16_2d(&mh, H, rows, h, kRowsPerCta) ||
        !encode_bf16_2d(&mw2, W2, static_cast<uint64_t>(E) * d, h, 128))
        return cudaErrorInvalidValue;
    const int max_pairs = device_sm_count() / 2;
    const long long blocks = (static_cast<long long>(rows) + (kPairRows - 1LL) * E) / kPairRows;
    PairArgs g1{offsets, E, rows, d, h, h, (h + 127) / 128, H, status, cap};
    g1.a_out = a_out;
    g1.b_out = b_out;
    long long t1 = blocks * g1.n_tiles;
    const int grid1 = static_cast<int>(t1 < max_pairs ? (t1 < 1 ? 1 : t1) : max_pairs);
    cudaError_t err = a_out != nullptr
                          ? launch_pair<kEpiSwiGLU, kBKMajor, true>(mx, mw1, mw3, mx, g1, grid1, s)
                          : launch_pair<kEpiSwiGLU>(mx, mw1, mw3, mx, g1, grid1, s);
    if (err != cudaSuccess) return err;
    if (between && (err = cudaEventRecord(between, s)) != cudaSuccess) return err;
    PairArgs g2{offsets, E, rows, h, d, d, (d + 255) / 256, Y, status, cap};
    long long t2 = blocks * g2.n_tiles;
    return launch_pair<kEpiStoreF32>(
        mh, mw2, mw2, my, g2, static_cast<int>(t2 < max_pairs ? (t2 < 1 ? 1 : t2) : max_pairs), s);
}

// Backward row-grouped GEMMs on CTA pairs (the backward pass is described in
// backward_sm100.cu): mode 0  dH = dY W2_e (B = W2 read MN-major), fp32 [rows, h];
// mode 1  du, dv from a = x W1_e^T, b = x W3_e^T and dH (B = [W1 | W3] rows, as GEMM1),
// bf16 [rows, 2h]; mode 2  dX = [du dv] [W1_e; W3_e] (B MN-major, W1 for k < h, then
// W3), fp32 [rows, d].  A maps have 128-row boxes, MN-major B maps 64 x 64 boxes.
cudaError_t launch_bwd_rows_pair(int mode, const CUtensorMap& a, const CUtensorMap& b0,
                                 const CUtensorMap& b1, const int32_t* offsets, int E, int rows,
                                 int d, int h, void* out, const float* dH, uint32_t* status,
                                 int cap, cudaStream_t s, const uint8_t* skip_flag) {
    const int max_pairs = device_sm_count() / 2;
    const long long blocks = (static_cast<long long>(rows) + (kPairRows - 1LL) * E) / kPairRows;
    auto grid = [&](long long tiles) {
        return static_cast<int>(tiles < max_pairs ? (tiles < 1 ? 1 : tiles) : max_pairs);
    };
    if (mode == 0) {
        CUtensorMap mo;  // dH [rows, h] fp32
        if (!encode_f32_3d(&mo, out, 1, rows, h, 32, 32)) return cudaErrorInvalidValue;
        PairArgs g{offsets, E, rows, d, h, d, (h + 255) / 256, out, status, cap, h, nullptr};
        return launch_pair<kEpiStoreF32, kBMn>(a, b0, b0, mo, g, grid(blocks * g.n_tiles), s);
    }
    if (mode == 1) {
        PairArgs g{offsets, E, rows, d, h, h, (h + 127) / 128, out, status, cap, h, dH};
        g.skip_flag = skip_flag;
        return launch_pair<kEpiBwdSwiGLU, kBKMajor>(a, b0, b1, a, g, grid(blocks * g.n_tiles), s);
    }
    CUtensorMap mo;  // dX [rows, d] fp32
    if (!encode_f32_3d(&mo, out, 1, rows, d, 32, 32)) return cudaErrorInvalidValue;
    PairArgs g{offsets, E, rows, 2 * h, d, h, (d + 255) / 256, out, status, cap, h, nullptr};
    return launch_pair<kEpiStoreF32, kBMnSplit>(a, b0, b1, mo, g, grid(blocks * g.n_tiles), s);
}

}  // namespace moe
