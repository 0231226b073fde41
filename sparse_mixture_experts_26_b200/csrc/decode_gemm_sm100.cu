// decode_gemm_sm100.cu -- the expert FFN for small batches, where streaming the
// touched experts' weights from HBM is the whole cost.
//
// crackai "Mixtral of Experts", "Key Takeaways": active parameters set the compute,
// total parameters set the memory; ml-canon "52 Mixtral", "Questions worth asking":
// all experts must sit in memory although only two run per token.  With a handful of
// tokens per expert the layer reads every touched expert's W1, W3 and W2 once and
// does almost no arithmetic per byte, so this path is built to keep HBM busy:
//
// * swap-AB: weight rows are the MMA's M operand (128 rows per instruction) and the
//   expert's few token rows are the N operand (NT = 16/32/64 columns), so the token
//   tile is tiny and nearly every byte moved is a weight byte;
// * every MMA row is a real weight row.  The tensor core re-reads its whole 128-row
//   A operand from shared memory for every K=16 step, so a tile with unused rows
//   costs as much MMA time as a full one (measured: half-empty tiles halved the
//   streaming rate);
// * gate/up GEMM: a tile is 64 rows of W1 stacked over the same 64 rows of W3
//   (rows 0..63 and 64..127 of the A tile), so the accumulator holds a = x.W1 and
//   b = x.W3 for the same 64 outputs in lanes j and 64+j; the epilogue exchanges
//   them through shared memory and writes silu(a)*b.  h/64 tiles per expert;
// * down GEMM: a tile is 128 rows of W2 over one of `ksplit` equal K ranges; each
//   K range writes its own fp32 partial output, summed later in a fixed order
//   (deterministic split-K), so that d/128 * ksplit units spread evenly over the
//   SMs (8 experts x 32 x 4 = 1024 units = 6.9 rounds of 148);
// * a deep ring of ~18 KiB stages keeps ~200 KiB of weight reads in flight per SM;
//   weight loads carry an evict-first L2 hint so the small token tiles stay cached.
// Every wait is bounded (see sm100_ptx.cuh).
#include <cuda.h>
#include <cuda_bf16.h>

#include "moe_internal.h"
#include "sm100_ptx.cuh"

namespace moe {

// Defined in grouped_gemm_sm100.cu.
bool encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows);

namespace {

constexpr int kBK = 64;          // one 128-byte swizzle span of bf16 along K
constexpr int kM = 128;          // MMA rows = weight rows per tile
constexpr int kThreads = 192;    // TMA warp, MMA warp, 4 epilogue warps
constexpr int kEpiThreads = 128;
constexpr int kXferBarrier = 1;  // named barrier id for the epilogue exchange
constexpr int kVoteBarrier = 2;  // epilogue vote after a bounded wait

enum DecodeMode { kSwiGLU = 0, kDown = 1 };

struct DecodeArgs {
    const int32_t* offsets;  // [E+1] group offsets (device)
    int E;
    int rows;        // grouped rows
    int K;           // reduction length
    int N;           // output columns (h for GEMM1, d for GEMM2)
    int w_rows;      // weight rows of one expert in the flattened view (= N)
    int n_wblocks;   // ceil(N / rows-per-tile)
    int ksplit;      // K ranges per tile (down GEMM), 1 for gate/up
    void* out;       // H bf16 [rows, N], or ksplit fp32 partials [ksplit][rows][N]
    uint32_t* status;
    int cap;         // rows kept per group (capacity; INT_MAX = no limit)
};

template <int MODE, int NT>
struct DecodeCfg {
    static constexpr int kJ = (MODE == kSwiGLU) ? kM / 2 : kM;  // output rows per tile
    static constexpr int kAStage = kM * 128;                      // 16 KiB
    static constexpr int kBStage = NT * 128;
    static constexpr int kStageTx = kAStage + kBStage;
    static constexpr int kStages = (200 * 1024) / (kAStage + kBStage);
    // TMEM columns: 128 (8, 4 or 2 accumulators of 16, 32 or 64 token columns), or two
    // accumulators of 128 token columns
    static constexpr uint32_t kTmemCols = NT <= 64 ? 128 : 2 * NT;
    static constexpr int kAcc = kTmemCols / NT;  // accumulators in flight
    // token columns the gate/up epilogue exchanges through shared memory at a time
    static constexpr int kXferCols = NT <= 64 ? NT : 32;
    static constexpr int kXferBytes = (MODE == kSwiGLU) ? kM * kXferCols * 4 : 0;
    static constexpr int kSmem =
        kStages * (kAStage + kBStage) + 1024 /*align*/ + 2048 /*bookkeeping*/ + kXferBytes;
    static constexpr uint32_t kIdesc = idesc_bf16_f32(kM, NT);
    static_assert(kBStage % 1024 == 0, "1 KiB-aligned stages");
    static_assert(NT % 16 == 0 && NT >= 16 && NT <= 128, "N must be 16..128, multiple of 16");
    static_assert(kStages >= 4 && kStages <= 16, "stage count");
    static_assert(kSmem <= 232448, "shared memory");
};

template <int NACC>
struct DecodeBook {
    uint64_t full[16];
    uint64_t empty[16];
    uint64_t tmem_full[NACC];
    uint64_t tmem_empty[NACC];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int off[kMaxExperts + 1];
    int end[kMaxExperts];
    int tile_start[kMaxExperts + 1];
};

struct Tile {
    int e, row0, nvalid, wb, ks;
};

template <int NACC>
__device__ __forceinline__ Tile decode_tile(const DecodeBook<NACC>& bk, int E, int nwb,
                                            int ksplit, int NTc, int tile) {
    int g = 0;
    while (g + 1 < E && tile >= bk.tile_start[g + 1]) ++g;
    int local = tile - bk.tile_start[g];
    Tile t;
    t.e = g;
    t.ks = local % ksplit;  // K ranges innermost, then weight blocks, then token chunks
    local /= ksplit;
    const int chunk = local / nwb;
    t.wb = local - chunk * nwb;
    t.row0 = bk.off[g] + chunk * NTc;
    const int left = bk.end[g] - t.row0;
    t.nvalid = left < NTc ? left : NTc;
    return t;
}

template <int NT>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[NT]);

template <>
__device__ __forceinline__ void tmem_ld_cols<16>(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_cols<32>(uint32_t taddr, uint32_t (&r)[32]) {
    tmem_ld_32cols(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_ld_cols<64>(uint32_t taddr, uint32_t (&r)[64]) {
    tmem_ld_32cols(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
    tmem_ld_32cols(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
}

template <int MODE, int NT>
__global__ void __launch_bounds__(kThreads, 1)
    decode_gemm_kernel(const __grid_constant__ CUtensorMap tmW0,
                       const __grid_constant__ CUtensorMap tmW1,
                       const __grid_constant__ CUtensorMap tmX, const DecodeArgs args) {
    using C = DecodeCfg<MODE, NT>;
    constexpr int NACC = C::kAcc;
    constexpr int J = C::kJ;
    using Book = DecodeBook<NACC>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;                                   // kStages * 16 KiB
    uint8_t* sB = smem + C::kStages * C::kAStage;         // kStages * kBStage
    Book& bk = *reinterpret_cast<Book*>(sB + C::kStages * C::kBStage);
    float* xfer = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(&bk) + 2048);
    static_assert(sizeof(Book) <= 2048, "bookkeeping reserve");
    volatile int* abort_flag = &bk.abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int E = args.E;
    const int ksplit = args.ksplit;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bk.full[s], 1);
            mbar_init(&bk.empty[s], 1);
        }
        for (int a = 0; a < NACC; ++a) {
            mbar_init(&bk.tmem_full[a], 1);
            mbar_init(&bk.tmem_empty[a], kEpiThreads);
        }
        mbar_init(&bk.drain, 1);
        bk.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW0);
        if (MODE == kSwiGLU) tma_prefetch_desc(&tmW1);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) tmem_alloc(&bk.tmem_base, C::kTmemCols);

    pdl_wait();
    pdl_launch_dependents();
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
            const int chunks = (bk.end[g] - bk.off[g] + NT - 1) / NT;
            bk.tile_start[g + 1] = bk.tile_start[g] + chunks * args.n_wblocks * ksplit;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = bk.tmem_base;
    const int total = bk.tile_start[E];
    const int num_kb = (args.K + kBK - 1) / kBK;
    const int kb_per_split = (num_kb + ksplit - 1) / ksplit;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t evict_first = l2_policy_evict_first();
            int stage = 0;
            uint32_t phase = 0, pending = 0, pending_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
                const Tile t = decode_tile(bk, E, args.n_wblocks, ksplit, NT, tile);
                const int wrow = t.e * args.w_rows + t.wb * J;
                const int kb0 = t.ks * kb_per_split;
                const int kb1 = min(num_kb, kb0 + kb_per_split);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(&bk.empty[stage], phase ^ 1u, abort_flag,
                                           args.status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bk.full[stage], C::kStageTx);
                    const int kc = kb * kBK;
                    uint8_t* a = sA + stage * C::kAStage;
                    tma_load_2d_hint(&tmW0, &bk.full[stage], a, kc, wrow, evict_first);
                    if (MODE == kSwiGLU)
                        tma_load_2d_hint(&tmW1, &bk.full[stage], a + J * 128, kc, wrow,
                                         evict_first);
                    tma_load_2d(&tmX, &bk.full[stage], sB + stage * C::kBStage, kc, t.row0);
                    pending |= 1u << stage;
                    pending_phase = (pending_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                for (int s = 0; s < C::kStages; ++s)
                    if (pending & (1u << s)) drain_wait(&bk.full[s], (pending_phase >> s) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true, issued = false;
            for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
                const Tile t = decode_tile(bk, E, args.n_wblocks, ksplit, NT, tile);
                const int kb0 = t.ks * kb_per_split;
                const int kb1 = min(num_kb, kb0 + kb_per_split);
                if (!mbar_wait_bounded(&bk.tmem_empty[acc], acc_phase ^ 1u, abort_flag,
                                       args.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * NT);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(&bk.full[stage], phase, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + stage * C::kAStage));
                    const uint64_t bd = sw128_kmajor_desc(smem_u32(sB + stage * C::kBStage));
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        umma_bf16(d_tmem, ad + 2 * k, bd + 2 * k, C::kIdesc,
                                  (kb > kb0 || k > 0) ? 1u : 0u);
                    umma_commit(&bk.empty[stage]);
                    issued = true;
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(&bk.tmem_full[acc]);
                if (++acc == NACC) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            if (!ok && issued) {
                umma_commit(&bk.drain);
                drain_wait(&bk.drain, 0);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        // Accumulator lane r = weight row r of the tile; column c = token c.
        const int q = warp & 3;
        const int r = q * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const Tile t = decode_tile(bk, E, args.n_wblocks, ksplit, NT, tile);
            if (!bar_all(mbar_wait_bounded(&bk.tmem_full[acc], acc_phase, abort_flag, args.status),
                         kVoteBarrier, kEpiThreads))
                break;
            tc_fence_after();
            uint32_t v[NT];
            tmem_ld_cols<NT>(tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                 static_cast<uint32_t>(acc * NT),
                             v);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&bk.tmem_empty[acc]);
            if (MODE == kSwiGLU) {
                // lanes J..2J-1 hold b for rows 0..J-1: pass all through shared memory
#pragma unroll
                for (int c = 0; c < NT; ++c) xfer[c * kM + r] = __uint_as_float(v[c]);
                asm volatile("bar.sync %0, %1;" ::"r"(kXferBarrier), "r"(kEpiThreads) : "memory");
                if (r < J) {
                    const int col = t.wb * J + r;
                    if (col < args.N) {
                        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.out);
#pragma unroll
                        for (int c = 0; c < NT; ++c) {
                            if (c < t.nvalid) {
                                const float a = xfer[c * kM + r];
                                const float b = xfer[c * kM + J + r];
                                out[static_cast<size_t>(t.row0 + c) * args.N + col] =
                                    __float2bfloat16_rn(a * b * __frcp_rn(1.0f + __expf(-a)));
                            }
                        }
                    }
                }
                asm volatile("bar.sync %0, %1;" ::"r"(kXferBarrier), "r"(kEpiThreads) : "memory");
            } else {
                const int col = t.wb * J + r;
                if (col < args.N) {
                    float* out = static_cast<float*>(args.out) +
                                 static_cast<size_t>(t.ks) * args.rows * args.N;
#pragma unroll
                    for (int c = 0; c < NT; ++c)
                        if (c < t.nvalid)
                            out[static_cast<size_t>(t.row0 + c) * args.N + col] =
                                __uint_as_float(v[c]);
                }
            }
            if (++acc == NACC) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

template <int MODE, int NT>
cudaError_t launch_decode(const CUtensorMap& w0, const CUtensorMap& w1, const CUtensorMap& x,
                          const DecodeArgs& args, int grid, cudaStream_t s) {
    using C = DecodeCfg<MODE, NT>;
    auto kern = decode_gemm_kernel<MODE, NT>;
    static PerDeviceOnce smem_once;
    if (const cudaError_t err = opt_in_smem(smem_once, kern, C::kSmem); err != cudaSuccess)
        return err;
    return launch_k(kern, grid, kThreads, C::kSmem, s, w0, w1, x, args);
}

// ---------------------------------------------------------------- fused gate/up + down
// One persistent cooperative launch runs both GEMMs.  Its unit list is all gate/up
// tiles (expert, token chunk, 64-row block of W1/W3), then all down units (expert,
// token chunk, 128-row block of W2, K range), experts in order.  A down unit needs
// only the H columns of its own K range, i.e. the gate/up tiles with the same expert
// and h-blocks in that range; each such tile bumps ready[e][ks] after its H stores
// are visible, and the down unit's producer waits (bounded) for the count before it
// loads H.  SMs that run out of gate/up tiles start streaming W2 at once, so neither
// the gate/up tail nor the launch boundary leaves HBM idle.  The readers of a
// counter also count themselves and the last one resets both counters to zero, so
// every launch starts from zeroed counters (repeated launches and graph replays).
struct FusedArgs {
    const int32_t* offsets;
    int E;
    int rows;
    int d;
    int h;
    int n_hb;      // 64-row W1/W3 blocks per expert: ceil(h / 64)
    int n_db;      // 128-row W2 blocks per expert: ceil(d / 128)
    int ksplit;    // K ranges of the down projection
    void* H;       // bf16 [rows, h]
    float* Ypart;  // ksplit fp32 partials [ksplit][rows][d]
    uint32_t* ready;    // [E][ksplit]
    uint32_t* readers;  // [E][ksplit]
    uint32_t* status;
    int cap;            // rows kept per group (capacity; INT_MAX = no limit)
    // optional: the pre-activations a = x W1^T and b = x W3^T, fp32 [rows, h] each,
    // kept for the backward pass (moe_layer_forward_train); nullptr: not written
    float* a_out;
    float* b_out;
};

template <int NACC>
struct FusedBook {
    uint64_t full[16];
    uint64_t empty[16];
    uint64_t tmem_full[NACC];
    uint64_t tmem_empty[NACC];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int off[kMaxExperts + 1];
    int end[kMaxExperts];         // end of the rows kept in group g (capacity)
    int start1[kMaxExperts + 1];  // gate/up tiles before expert g
    int start2[kMaxExperts + 1];  // down units before expert g
    int ntr;                      // token rows per tile in this launch (<= NT)
    int stages;                   // stages the ring holds at that tile size
};

struct FusedUnit {
    bool down;
    int e, row0, nvalid, chunks, blk, ks, kb0, kb1;
};

template <int NACC>
__device__ __forceinline__ FusedUnit fused_unit(const FusedBook<NACC>& bk, const FusedArgs& a,
                                                int NTc, int num_kb1, int kps, int num_kb2,
                                                int u) {
    FusedUnit f;
    const int n1 = bk.start1[a.E];
    int g = 0, local;
    if (u < n1) {
        while (g + 1 < a.E && u >= bk.start1[g + 1]) ++g;
        local = u - bk.start1[g];
        f.down = false;
        f.ks = 0;
        f.chunks = (bk.end[g] - bk.off[g] + NTc - 1) / NTc;
        // token chunks innermost: the chunks of one weight block run on neighbouring
        // CTAs at the same time, so the weights cross HBM once
        f.blk = local / f.chunks;
        const int chunk = local - f.blk * f.chunks;
        f.row0 = bk.off[g] + chunk * NTc;
        f.kb0 = 0;
        f.kb1 = num_kb1;
    } else {
        const int v = u - n1;
        while (g + 1 < a.E && v >= bk.start2[g + 1]) ++g;
        local = v - bk.start2[g];
        f.down = true;
        f.chunks = (bk.end[g] - bk.off[g] + NTc - 1) / NTc;
        const int chunk = local % f.chunks;
        local /= f.chunks;
        f.ks = local % a.ksplit;
        f.blk = local / a.ksplit;
        f.row0 = bk.off[g] + chunk * NTc;
        f.kb0 = f.ks * kps;
        f.kb1 = min(num_kb2, f.kb0 + kps);
    }
    f.e = g;
    const int left = bk.end[g] - f.row0;
    f.nvalid = left < NTc ? left : NTc;
    return f;
}

// Token operands of the fused launch, each as tensor maps whose boxes hold 16, 32, 64
// and 128 rows (at most NT).  The launch reads the group sizes first and takes the
// smallest token tile that holds its largest group (every group is then one chunk);
// the stage ring is cut into as many stages as fit at that tile size (128 rows: 6,
// 64: 8, 32: 10, 16: 12 of the same ~200 KiB), so a batch whose groups are small keeps
// more weight bytes in flight per SM, which is what sets the streaming rate here.
struct TokMaps {
    CUtensorMap m[4];
};
constexpr int kTokBoxes = 4;
__host__ __device__ constexpr int tok_box_rows(int i, int NT) {
    return (16 << i) < NT ? (16 << i) : NT;
}
__device__ __forceinline__ int tok_box_index(int n) {
    return n <= 16 ? 0 : n <= 32 ? 1 : n <= 64 ? 2 : 3;
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    decode_ffn_fused_kernel(const __grid_constant__ CUtensorMap tmW1,
                            const __grid_constant__ CUtensorMap tmW3,
                            const __grid_constant__ TokMaps tmX,
                            const __grid_constant__ CUtensorMap tmW2,
                            const __grid_constant__ TokMaps tmH, const FusedArgs args) {
    using C = DecodeCfg<kSwiGLU, NT>;  // the ring's size and the accumulators
    constexpr int NACC = C::kAcc;
    constexpr int J1 = kM / 2;         // 64 output columns of H per gate/up tile
    constexpr int kRingBytes = C::kStages * (C::kAStage + C::kBStage);
    using Book = FusedBook<NACC>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    Book& bk = *reinterpret_cast<Book*>(smem + kRingBytes);
    float* xfer = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(&bk) + 2048);
    static_assert(sizeof(Book) <= 2048, "bookkeeping reserve");
    volatile int* abort_flag = &bk.abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int E = args.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 16; ++s) {  // every stage the ring can be cut into
            mbar_init(&bk.full[s], 1);
            mbar_init(&bk.empty[s], 1);
        }
        for (int a = 0; a < NACC; ++a) {
            mbar_init(&bk.tmem_full[a], 1);
            mbar_init(&bk.tmem_empty[a], kEpiThreads);
        }
        mbar_init(&bk.drain, 1);
        bk.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW1);
        tma_prefetch_desc(&tmW3);
        tma_prefetch_desc(&tmW2);
        for (int i = 0; i < kTokBoxes; ++i) {
            tma_prefetch_desc(&tmX.m[i]);
            tma_prefetch_desc(&tmH.m[i]);
        }
    }
    if (warp == 1) tmem_alloc(&bk.tmem_base, C::kTmemCols);

    pdl_wait();
    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        int prev = 0;
        for (int g = 0; g <= E; ++g) {
            int v = args.offsets[g];
            v = v < prev ? prev : (v > args.rows ? args.rows : v);
            bk.off[g] = v;
            prev = v;
        }
        int max_n = 1;
        for (int g = 0; g < E; ++g) {
            const int n = bk.off[g + 1] - bk.off[g];
            bk.end[g] = bk.off[g] + (n < args.cap ? n : args.cap);
            max_n = bk.end[g] - bk.off[g] > max_n ? bk.end[g] - bk.off[g] : max_n;
        }
        const int ntr = tok_box_rows(tok_box_index(max_n), NT);
        const int st = kRingBytes / (C::kAStage + ntr * 128);
        bk.ntr = ntr;
        bk.stages = st < 16 ? st : 16;
        bk.start1[0] = 0;
        bk.start2[0] = 0;
        for (int g = 0; g < E; ++g) {
            const int chunks = (bk.end[g] - bk.off[g] + ntr - 1) / ntr;
            bk.start1[g + 1] = bk.start1[g] + chunks * args.n_hb;
            bk.start2[g + 1] = bk.start2[g] + chunks * args.n_db * args.ksplit;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // the ring at this launch's tile size: A slots, then B slots of ntr rows
    const int ntr = bk.ntr, n_stages = bk.stages;
    const int b_slot = ntr * 128;
    uint8_t* sB = smem + n_stages * C::kAStage;
    const int tok_map = tok_box_index(ntr);
    const uint32_t tmem_base = bk.tmem_base;
    const int total = bk.start1[E] + bk.start2[E];
    const int num_kb1 = (args.d + kBK - 1) / kBK;
    const int num_kb2 = (args.h + kBK - 1) / kBK;
    const int kps = (num_kb2 + args.ksplit - 1) / args.ksplit;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t evict_first = l2_policy_evict_first();
            int stage = 0;
            uint32_t phase = 0, pending = 0, pending_phase = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < total; u += gridDim.x) {
                const FusedUnit f = fused_unit(bk, args, ntr, num_kb1, kps, num_kb2, u);
                if (f.down) {
                    // wait until every gate/up tile of this K range has published its H
                    const uint32_t need = static_cast<uint32_t>(f.chunks * (f.kb1 - f.kb0));
                    const uint32_t* rdy = args.ready + f.e * args.ksplit + f.ks;
                    if (!flag_wait_bounded(rdy, need, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_global();
                    // the last reader of this counter resets it for the next launch
                    uint32_t* rd = args.readers + f.e * args.ksplit + f.ks;
                    if (atomicAdd(rd, 1u) + 1u == static_cast<uint32_t>(f.chunks * args.n_db)) {
                        *const_cast<uint32_t*>(rdy) = 0u;
                        *rd = 0u;
                    }
                }
                const int wrow = f.down ? f.e * args.d + f.blk * kM : f.e * args.h + f.blk * J1;
                for (int kb = f.kb0; kb < f.kb1; ++kb) {
                    if (!mbar_wait_bounded(&bk.empty[stage], phase ^ 1u, abort_flag,
                                           args.status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bk.full[stage], C::kAStage + b_slot);
                    const int kc = kb * kBK;
                    uint8_t* a = sA + stage * C::kAStage;
                    uint8_t* b = sB + stage * b_slot;
                    if (f.down) {
                        tma_load_2d_hint(&tmW2, &bk.full[stage], a, kc, wrow, evict_first);
                        tma_load_2d(&tmH.m[tok_map], &bk.full[stage], b, kc, f.row0);
                    } else {
                        tma_load_2d_hint(&tmW1, &bk.full[stage], a, kc, wrow, evict_first);
                        tma_load_2d_hint(&tmW3, &bk.full[stage], a + J1 * 128, kc, wrow,
                                         evict_first);
                        tma_load_2d(&tmX.m[tok_map], &bk.full[stage], b, kc, f.row0);
                    }
                    pending |= 1u << stage;
                    pending_phase = (pending_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == n_stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                for (int s2 = 0; s2 < n_stages; ++s2)
                    if (pending & (1u << s2)) drain_wait(&bk.full[s2], (pending_phase >> s2) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true, issued = false;
            for (int u = blockIdx.x; ok && u < total; u += gridDim.x) {
                const FusedUnit f = fused_unit(bk, args, ntr, num_kb1, kps, num_kb2, u);
                if (!mbar_wait_bounded(&bk.tmem_empty[acc], acc_phase ^ 1u, abort_flag,
                                       args.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * NT);
                const uint32_t idesc = idesc_bf16_f32(kM, ntr);
                for (int kb = f.kb0; kb < f.kb1; ++kb) {
                    if (!mbar_wait_bounded(&bk.full[stage], phase, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + stage * C::kAStage));
                    const uint64_t bd = sw128_kmajor_desc(smem_u32(sB + stage * b_slot));
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        umma_bf16(d_tmem, ad + 2 * k, bd + 2 * k, idesc,
                                  (kb > f.kb0 || k > 0) ? 1u : 0u);
                    umma_commit(&bk.empty[stage]);
                    issued = true;
                    if (++stage == n_stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(&bk.tmem_full[acc]);
                if (++acc == NACC) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            if (!ok && issued) {
                umma_commit(&bk.drain);
                drain_wait(&bk.drain, 0);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int r = q * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int u = blockIdx.x; u < total; u += gridDim.x) {
            const FusedUnit f = fused_unit(bk, args, ntr, num_kb1, kps, num_kb2, u);
            if (!bar_all(mbar_wait_bounded(&bk.tmem_full[acc], acc_phase, abort_flag, args.status),
                         kVoteBarrier, kEpiThreads))
                break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                  static_cast<uint32_t>(acc * NT);
            if constexpr (NT <= 64) {
                uint32_t v[NT];
                tmem_ld_cols<NT>(tacc, v);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&bk.tmem_empty[acc]);
                if (!f.down) {
#pragma unroll
                    for (int c = 0; c < NT; ++c) xfer[c * kM + r] = __uint_as_float(v[c]);
                    asm volatile("bar.sync %0, %1;" ::"r"(kXferBarrier), "r"(kEpiThreads) : "memory");
                    if (r < J1) {
                        const int col = f.blk * J1 + r;
                        if (col < args.h) {
                            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.H);
#pragma unroll
                            for (int c = 0; c < NT; ++c) {
                                if (c < f.nvalid) {
                                    const float a = xfer[c * kM + r];
                                    const float b = xfer[c * kM + J1 + r];
                                    const size_t at = static_cast<size_t>(f.row0 + c) * args.h + col;
                                    out[at] = __float2bfloat16_rn(a * b * __frcp_rn(1.0f + __expf(-a)));
                                    if (args.a_out != nullptr) {
                                        args.a_out[at] = a;
                                        args.b_out[at] = b;
                                    }
                                }
                            }
                        }
                        __threadfence();  // H stores visible at device scope before the count
                    }
                    asm volatile("bar.sync %0, %1;" ::"r"(kXferBarrier), "r"(kEpiThreads) : "memory");
                    if (r == 0) {
                        fence_proxy_async_global();
                        atomicAdd(args.ready + f.e * args.ksplit + f.blk / kps, 1u);
                    }
                } else {
                    const int col = f.blk * kM + r;
                    if (col < args.d) {
                        float* out = args.Ypart + static_cast<size_t>(f.ks) * args.rows * args.d;
#pragma unroll
                        for (int c = 0; c < NT; ++c)
                            if (c < f.nvalid)
                                out[static_cast<size_t>(f.row0 + c) * args.d + col] =
                                    __uint_as_float(v[c]);
                    }
                }
            } else {
                // 128 token columns: drain the accumulator 32 columns at a time (the
                // exchange buffer holds 32 columns); chunks past the last row are skipped.
                constexpr int kC = C::kXferCols;
                if (!f.down) {
                    for (int c0 = 0; c0 < NT && c0 < f.nvalid; c0 += kC) {
                        uint32_t v[kC];
                        tmem_ld_32cols(tacc + c0, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int c = 0; c < kC; ++c) xfer[c * kM + r] = __uint_as_float(v[c]);
                        asm volatile("bar.sync %0, %1;" ::"r"(kXferBarrier), "r"(kEpiThreads)
                                     : "memory");
                        if (r < J1) {
                            const int col = f.blk * J1 + r;
                            if (col < args.h) {
                                __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.H);
#pragma unroll
                                for (int c = 0; c < kC; ++c) {
                                    if (c0 + c < f.nvalid) {
                                        const float a = xfer[c * kM + r];
                                        const float b = xfer[c * kM + J1 + r];
                                        const size_t at =
                                            static_cast<size_t>(f.row0 + c0 + c) * args.h + col;
                                        out[at] = __float2bfloat16_rn(a * b * __frcp_rn(1.0f + __expf(-a)));
                                        if (args.a_out != nullptr) {
                                            args.a_out[at] = a;
                                            args.b_out[at] = b;
                                        }
                                    }
                                }
                            }
                        }
                        asm volatile("bar.sync %0, %1;" ::"r"(kXferBarrier), "r"(kEpiThreads)
                                     : "memory");
                    }
                    tc_fence_before();
                    mbar_arrive(&bk.tmem_empty[acc]);
                    if (r < J1) __threadfence();  // H stores visible before the count
                    asm volatile("bar.sync %0, %1;" ::"r"(kXferBarrier), "r"(kEpiThreads) : "memory");
                    if (r == 0) {
                        fence_proxy_async_global();
                        atomicAdd(args.ready + f.e * args.ksplit + f.blk / kps, 1u);
                    }
                } else {
                    const int col = f.blk * kM + r;
                    float* out = args.Ypart + static_cast<size_t>(f.ks) * args.rows * args.d;
                    for (int c0 = 0; c0 < NT && c0 < f.nvalid; c0 += kC) {
                        uint32_t v[kC];
                        tmem_ld_32cols(tacc + c0, v);
                        tmem_ld_wait();
                        if (col < args.d) {
#pragma unroll
                            for (int c = 0; c < kC; ++c)
                                if (c0 + c < f.nvalid)
                                    out[static_cast<size_t>(f.row0 + c0 + c) * args.d + col] =
                                        __uint_as_float(v[c]);
                        }
                    }
                    tc_fence_before();
                    mbar_arrive(&bk.tmem_empty[acc]);
                }
            }
            if (++acc == NACC) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

template <int NT>
cudaError_t launch_ffn_fused_nt(const void* x_perm, const int32_t* offsets, const void* W1,
                                const void* W3, const void* W2, int rows, int d, int h, int E,
                                void* H, float* Ypart, int ksplit, uint32_t* counters,
                                uint32_t* status, cudaStream_t s, int cap, float* a_out,
                                float* b_out) {
    CUtensorMap mw1, mw3, mw2;
    TokMaps mx, mh;
    if (!encode_bf16_2d(&mw1, W1, static_cast<uint64_t>(E) * h, d, kM / 2) ||
        !encode_bf16_2d(&mw3, W3, static_cast<uint64_t>(E) * h, d, kM / 2) ||
        !encode_bf16_2d(&mw2, W2, static_cast<uint64_t>(E) * d, h, kM))
        return cudaErrorInvalidValue;
    for (int i = 0; i < kTokBoxes; ++i)
        if (!encode_bf16_2d(&mx.m[i], x_perm, rows, d, tok_box_rows(i, NT)) ||
            !encode_bf16_2d(&mh.m[i], H, rows, h, tok_box_rows(i, NT)))
            return cudaErrorInvalidValue;
    using C = DecodeCfg<kSwiGLU, NT>;
    auto kern = decode_ffn_fused_kernel<NT>;
    static PerDeviceOnce smem_once;
    if (const cudaError_t err = opt_in_smem(smem_once, kern, C::kSmem); err != cudaSuccess)
        return err;
    FusedArgs a{offsets, E, rows, d, h, (h + 63) / 64, (d + kM - 1) / kM, ksplit, H, Ypart,
                counters, counters + E * ksplit, status, cap, a_out, b_out};
    const int sms = device_sm_count();
    const long long chunks = static_cast<long long>(rows) / NT + E;
    const long long units = chunks * (a.n_hb + static_cast<long long>(a.n_db) * ksplit);
    // Every CTA must be resident at once (down units wait for other CTAs' tiles), so
    // the launch is cooperative: one CTA per SM at most.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(units < sms ? units : sms));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, kern, mw1, mw3, mx, mw2, mh, a);
    return err != cudaSuccess ? err : cudaGetLastError();
}

template <int NT>
cudaError_t launch_ffn_decode_nt(const void* x_perm, const int32_t* offsets, const void* W1,
                                 const void* W3, const void* W2, int rows, int d, int h, int E,
                                 void* H, float* Yout, int ksplit, uint32_t* status,
                                 cudaStream_t s, cudaEvent_t between, int cap) {
    constexpr int J1 = DecodeCfg<kSwiGLU, NT>::kJ, J2 = DecodeCfg<kDown, NT>::kJ;
    CUtensorMap mw1, mw3, mx, mw2, mh;
    if (!encode_bf16_2d(&mw1, W1, static_cast<uint64_t>(E) * h, d, J1) ||
        !encode_bf16_2d(&mw3, W3, static_cast<uint64_t>(E) * h, d, J1) ||
        !encode_bf16_2d(&mx, x_perm, rows, d, NT) ||
        !encode_bf16_2d(&mw2, W2, static_cast<uint64_t>(E) * d, h, J2) ||
        !encode_bf16_2d(&mh, H, rows, h, NT))
        return cudaErrorInvalidValue;
    const int sms = device_sm_count();
    // Units per launch are at most (rows/NT + E) * weight blocks * K ranges.
    const long long chunks = static_cast<long long>(rows) / NT + E;
    DecodeArgs a1{offsets, E, rows, d, h, h, (h + J1 - 1) / J1, 1, H, status, cap};
    const long long t1 = chunks * a1.n_wblocks;
    cudaError_t err = launch_decode<kSwiGLU, NT>(mw1, mw3, mx, a1,
                                                  static_cast<int>(t1 < sms ? t1 : sms), s);
    if (err != cudaSuccess) return err;
    if (between && (err = cudaEventRecord(between, s)) != cudaSuccess) return err;
    DecodeArgs a2{offsets, E, rows, h, d, d, (d + J2 - 1) / J2, ksplit, Yout, status, cap};
    const long long t2 = chunks * a2.n_wblocks * ksplit;
    return launch_decode<kDown, NT>(mw2, mw2, mh, a2, static_cast<int>(t2 < sms ? t2 : sms), s);
}

}  // namespace

cudaError_t launch_ffn_bf16_decode_fused(const void* x_perm, const int32_t* offsets,
                                         const void* W1, const void* W3, const void* W2, int rows,
                                         int d, int h, int E, void* H, float* Ypart, int ksplit,
                                         uint32_t* counters, uint32_t* status, cudaStream_t s,
                                         int cap, float* a_out, float* b_out) {
    const int T = rows / 2;
    if (T <= 16)
        return launch_ffn_fused_nt<16>(x_perm, offsets, W1, W3, W2, rows, d, h, E, H, Ypart,
                                       ksplit, counters, status, s, cap, a_out, b_out);
    if (T <= 32)
        return launch_ffn_fused_nt<32>(x_perm, offsets, W1, W3, W2, rows, d, h, E, H, Ypart,
                                       ksplit, counters, status, s, cap, a_out, b_out);
    if (T <= 64)
        return launch_ffn_fused_nt<64>(x_perm, offsets, W1, W3, W2, rows, d, h, E, H, Ypart,
                                       ksplit, counters, status, s, cap, a_out, b_out);
    return launch_ffn_fused_nt<128>(x_perm, offsets, W1, W3, W2, rows, d, h, E, H, Ypart, ksplit,
                                    counters, status, s, cap, a_out, b_out);
}

cudaError_t launch_ffn_bf16_decode(const void* x_perm, const int32_t* offsets, const void* W1,
                                   const void* W3, const void* W2, int rows, int d, int h, int E,
                                   void* H, float* Yout, int ksplit, uint32_t* status,
                                   cudaStream_t s, cudaEvent_t between, int cap) {
    const int T = rows / 2;  // a group holds each token at most once
    if (T <= 16)
        return launch_ffn_decode_nt<16>(x_perm, offsets, W1, W3, W2, rows, d, h, E, H, Yout,
                                        ksplit, status, s, between, cap);
    if (T <= 32)
        return launch_ffn_decode_nt<32>(x_perm, offsets, W1, W3, W2, rows, d, h, E, H, Yout,
                                        ksplit, status, s, between, cap);
    return launch_ffn_decode_nt<64>(x_perm, offsets, W1, W3, W2, rows, d, h, E, H, Yout, ksplit,
                                    status, s, between, cap);
}

}  // namespace moe
