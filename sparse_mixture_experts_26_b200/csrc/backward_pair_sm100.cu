// backward_pair_sm100.cu -- the weight-gradient GEMMs of the backward pass on pairs of
// SMs (tcgen05 cta_group::2), for reductions over many rows per expert.
//
// Same computation as bwd_wgrad_kernel in backward_sm100.cu (the exact derivative of
// the layer; crackai "Mixtral of Experts", "Key Takeaways": the router and experts are
// learned jointly):  out[e][m][n] = sum over the rows r of expert e of A[r, m] B[r, n],
// with dW2 = dY^T H and [dW1; dW3] = [du dv]^T x.  A tile is 256 output rows (m) x 256
// output columns (n), computed by a cluster of two CTAs: each CTA stages its own 128
// columns of A and its own 128 columns of B per 64-row K block (both MN-major boxes),
// and one thread of the leader issues tcgen05.mma.cta_group::2 (M = 256 from the two
// A halves, N = 256 from the two B halves); each CTA's TMEM receives its 128 rows.
// Per SM a stage is 32 KiB instead of 48 KiB for the same math, which leaves room for
// 7 stages.
//
// A reduction starts and ends at arbitrary rows, so the rows of an expert's last,
// partial K block that belong to the next expert must be zero before the MMA reads
// them.  Whole K blocks take the plain pair path: both CTAs' TMA loads count their
// bytes on the leader's "full" barrier.  A partial block's loads complete instead on
// a barrier of each CTA's own ("landed"); a fix-up warp in each CTA waits there,
// clears the rows in its own tiles and makes the writes visible to the tensor core
// (fence.proxy.async); the peer's then arrives on the leader's "fixed" barrier, and
// the leader's, once both are done, arrives on "full".  (A handshake on every block
// instead measured 2-4x slower: a cluster-scope arrive per block serialises the
// pipeline.)  The leader's MMA completions are multicast to both CTAs' "empty" and
// "tmem_full" barriers; both epilogues arrive on the leader's "tmem_empty".
//
// The epilogue stores straight from registers: each warp reads its TMEM lanes in the
// 16x256b shape, where four consecutive threads hold eight consecutive columns of a
// row, so every store instruction writes whole 32-byte sectors.  (Staging 32 x 32
// chunks in shared memory for TMA tensor stores, as the single-SM kernel does, was
// slower here -- the stores queued behind the operand loads on the TMA path: dW1+dW3
// 1.66 -> 1.62 ms with real data, 1.43 -> 1.25 ms at full clock -- and its 32 KiB of
// staging now holds a 7th input stage.)  Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>

#include "moe_internal.h"
#include "sm100_ptx.cuh"

namespace moe {

namespace {

constexpr int kRows = 128;                  // output rows per CTA (TMEM lanes)
constexpr int kBK = 64;                     // K rows per stage
constexpr int kN = 256;                     // output columns per tile
constexpr int kStages = 7;
constexpr int kBox = kMnBoxBytes;           // one 64-column x 64-row bf16 box: 8 KiB
constexpr int kABytes = 2 * kBox;           // this CTA's 128 columns of A
constexpr int kBBytes = 2 * kBox;           // this CTA's 128 columns of B
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 224;  // TMA, MMA, 4 epilogue warps, fix-up warp
constexpr int kEpiThreads = 128;
constexpr uint32_t kTmemCols = 2 * kN;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 1024 /*book*/;
static_assert(kSmemBytes <= 232448, "shared memory");
constexpr int kVoteBarrier = 2;
constexpr uint16_t kBothCtas = 0x3;
// M = 256 (two CTAs), N = 256, both operands MN-major.
constexpr uint32_t kIdesc = idesc_bf16_f32_major(2 * kRows, kN, true, true);

struct Book {
    uint64_t landed[kStages];    // partial blocks: this CTA's loads are in shared memory
    uint64_t fixed[kStages];     // leader, partial blocks: the peer cleared its rows
    uint64_t full[kStages];      // leader: both CTAs' stages are ready for the MMA
    uint64_t empty[kStages];     // the MMAs reading a stage are done (multicast)
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];      // leader: both epilogues drained the accumulator
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int off[kMaxExperts + 1];
    int end[kMaxExperts];
    int poff[kMaxExperts + 1];  // first row of each expert in a padded operand
};
static_assert(sizeof(Book) <= 1024, "bookkeeping reserve");

struct PArgs {
    const int32_t* offsets;
    int E;
    int rows;
    int M;
    int N;
    int m_pairs;     // ceil(M / 256)
    int n_tiles;     // ceil(N / 256)
    int split;       // output rows m < split go to out0, the rest to out1
    float* out0;
    float* out1;
    uint32_t* status;
    int cap;
    // 1: the operand (A or B) is a padded copy whose expert e starts at row poff[e]
    // and has zero rows up to the next multiple of 64.  With either set, every K
    // block takes the plain pair path (no partial blocks to clear).
    int pad_a, pad_b;
};

// Bounded wait with cluster-scope acquire: pairs with the peer's cluster-scope release
// arrive, so the peer's shared-memory writes before it are ordered before what follows.
__device__ __forceinline__ bool wait_cluster_bounded(uint64_t* bar, uint32_t parity,
                                                     volatile int* abort_flag, uint32_t* status) {
    auto try_wait = [&]() {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        return done != 0;
    };
    if (try_wait()) return true;
    const unsigned long long t0 = global_timer_ns();
    while (!try_wait()) {
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > kWaitTimeoutNs) {
            *abort_flag = 1;
            if (status) atomicOr(status, 1u);  // MOE_DEV_FLAG_TIMEOUT
            return false;
        }
    }
    return true;
}

__global__ void __launch_bounds__(kThreads, 1)
    bwd_wgrad_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                          const __grid_constant__ CUtensorMap tmB, const PArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages * kABytes;
    Book& bk = *reinterpret_cast<Book*>(smem + kStages * kStageBytes);
    volatile int* abort_flag = &bk.abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int E = args.E;
    const uint32_t rank = cluster_ctarank();  // 0 = leader, 1 = peer
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bk.landed[s], 1);
            mbar_init(&bk.fixed[s], 1);
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
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) tmem_alloc_pair(&bk.tmem_base, kTmemCols);
    if (threadIdx.x == 0) {
        int prev = 0;
        for (int g = 0; g <= E; ++g) {
            int v = args.offsets[g];
            v = v < prev ? prev : (v > args.rows ? args.rows : v);
            bk.off[g] = v;
            prev = v;
        }
        bk.poff[0] = 0;
        for (int g = 0; g < E; ++g) {
            const int n = bk.off[g + 1] - bk.off[g];
            bk.end[g] = bk.off[g] + (n < args.cap ? n : args.cap);
            bk.poff[g + 1] = bk.poff[g] + (n + kBK - 1) / kBK * kBK;
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers are initialised before either signals the other
    tc_fence_after();

    const uint32_t tmem_base = bk.tmem_base;
    const bool padded = (args.pad_a | args.pad_b) != 0;
    const int per_e = args.m_pairs * args.n_tiles;
    const int total = E * per_e;

    auto tile_of = [&](int tile, int& e, int& mp, int& nt, int& r0, int& n_rows) {
        e = tile / per_e;
        const int local = tile - e * per_e;
        nt = local % args.n_tiles;  // column blocks innermost
        mp = local / args.n_tiles;
        r0 = bk.off[e];
        n_rows = bk.end[e] - bk.off[e];
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, lpar = 0;     // ring phase; parity of each landed[s]
            uint32_t pend_full = 0, pend_full_ph = 0, pend_land = 0, pend_land_ph = 0;
            bool ok = true, issued = false;
            for (int tile = pair; ok && tile < total; tile += npairs) {
                int e, mp, nt, r0, n_rows;
                tile_of(tile, e, mp, nt, r0, n_rows);
                const int nkb = (n_rows + kBK - 1) / kBK;
                const int mcol = mp * 2 * kRows + static_cast<int>(rank) * kRows;
                const int ncol = nt * kN + static_cast<int>(rank) * (kN / 2);
                const int ra0 = args.pad_a ? bk.poff[e] : r0;  // first K row of A, of B
                const int rb0 = args.pad_b ? bk.poff[e] : r0;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait_bounded(&bk.empty[stage], phase ^ 1u, abort_flag,
                                           args.status)) {
                        ok = false;
                        break;
                    }
                    const int r = r0 + kb * kBK;
                    const int ra = ra0 + kb * kBK, rb = rb0 + kb * kBK;
                    uint8_t* a = sA + stage * kABytes;
                    uint8_t* b = sB + stage * kBBytes;
                    const uint32_t bit = 1u << stage;
                    if (!padded && n_rows - kb * kBK < kBK) {
                        // partial block: land locally, the fix-up warp takes over
                        mbar_arrive_expect_tx(&bk.landed[stage], kStageBytes);
                        tma_load_2d(&tmA, &bk.landed[stage], a, mcol, r);
                        tma_load_2d(&tmA, &bk.landed[stage], a + kBox, mcol + 64, r);
                        tma_load_2d(&tmB, &bk.landed[stage], b, ncol, r);
                        tma_load_2d(&tmB, &bk.landed[stage], b + kBox, ncol + 64, r);
                        pend_land |= bit;
                        pend_land_ph = (pend_land_ph & ~bit) | (lpar & bit);
                        lpar ^= bit;
                    } else {
                        const uint32_t full_leader = map_to_cta(smem_u32(&bk.full[stage]), 0);
                        if (leader) mbar_arrive_expect_tx(&bk.full[stage], 2 * kStageBytes);
                        tma_load_2d_pair(&tmA, full_leader, a, mcol, ra);
                        tma_load_2d_pair(&tmA, full_leader, a + kBox, mcol + 64, ra);
                        tma_load_2d_pair(&tmB, full_leader, b, ncol, rb);
                        tma_load_2d_pair(&tmB, full_leader, b + kBox, ncol + 64, rb);
                        pend_full |= bit;
                        pend_full_ph = (pend_full_ph & ~bit) | (phase << stage);
                    }
                    issued = true;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok && issued) {
                // let copies in flight land before this CTA's shared memory is released
                for (int s = 0; s < kStages; ++s)
                    if (pend_land & (1u << s)) drain_wait(&bk.landed[s], (pend_land_ph >> s) & 1u);
                if (leader) {
                    for (int s = 0; s < kStages; ++s)
                        if (pend_full & (1u << s)) drain_wait(&bk.full[s], (pend_full_ph >> s) & 1u);
                } else if (pend_full) {
                    short_pause_ns(2000000ull);  // its pair copies count on the leader's barriers
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
                int e, mp, nt, r0, n_rows;
                tile_of(tile, e, mp, nt, r0, n_rows);
                const int nkb = (n_rows + kBK - 1) / kBK;
                if (nkb == 0) continue;  // zero tile: written by the epilogues alone
                if (!mbar_wait_bounded(&bk.tmem_empty[acc], acc_phase ^ 1u, abort_flag,
                                       args.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kN);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait_bounded(&bk.full[stage], phase, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_mn_desc(smem_u32(sA + stage * kABytes));
                    const uint64_t bd = sw128_mn_desc(smem_u32(sB + stage * kBBytes));
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        umma_bf16_pair(d_tmem, ad + kMnDescStep * k, bd + kMnDescStep * k, kIdesc,
                                       (kb | k) != 0);
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
    } else if (warp == 6) {
        // ------------------------------------------- fix-up of partial K blocks (both)
        int stage = 0;
        uint32_t lpar = 0, fpar = 0;  // parity of each landed[s] / fixed[s]
        const uint32_t cap_rows = args.cap != INT_MAX ? 1u : 0u;
        bool ok = true;
        for (int tile = pair; ok && tile < total; tile += npairs) {
            int e, mp, nt, r0, n_rows;
            tile_of(tile, e, mp, nt, r0, n_rows);
            const int nkb = (n_rows + kBK - 1) / kBK;
            for (int kb = 0; kb < nkb; ++kb) {
                const int kv = n_rows - kb * kBK;  // rows of this block inside the group
                if (!padded && kv < kBK) {
                    const uint32_t bit = 1u << stage;
                    int got = 1;
                    if (lane == 0)
                        got = mbar_wait_bounded(&bk.landed[stage], (lpar >> stage) & 1u,
                                                abort_flag, args.status);
                    lpar ^= bit;
                    ok = __shfl_sync(0xffffffffu, got, 0) != 0;
                    if (!ok) break;
                    // rows kv..63 belong to the next group: clear them in this CTA's A
                    // boxes (and B boxes when a capacity may have left rows unwritten)
                    uint8_t* a = sA + stage * kABytes;
                    uint8_t* b = sB + stage * kBBytes;
                    const int nz = (kBK - kv) * 8;
                    const int boxes = cap_rows ? 4 : 2;
                    for (int i = lane; i < boxes * nz; i += 32) {
                        const int box = i / nz, c = i - box * nz;
                        uint8_t* base = box < 2 ? a + box * kBox : b + (box - 2) * kBox;
                        *reinterpret_cast<uint4*>(base + kv * 128 + c * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        if (!leader) {
                            mbar_arrive_cluster(map_to_cta(smem_u32(&bk.fixed[stage]), 0));
                        } else {
                            got = wait_cluster_bounded(&bk.fixed[stage], (fpar >> stage) & 1u,
                                                       abort_flag, args.status);
                            if (got) mbar_arrive(&bk.full[stage]);
                        }
                    }
                    fpar ^= bit;
                    ok = __shfl_sync(0xffffffffu, got, 0) != 0;
                    if (!ok) break;
                }
                if (++stage == kStages) stage = 0;
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue (both)
        const int q = warp & 3;  // warps 2..5: TMEM lane quarters 2, 3, 0, 1
        const uint32_t empty_leader0 = map_to_cta(smem_u32(&bk.tmem_empty[0]), 0);
        const uint32_t empty_leader1 = map_to_cta(smem_u32(&bk.tmem_empty[1]), 0);
        const int c2 = 2 * (lane & 3), r4 = lane >> 2;  // this thread's columns / rows
        int acc = 0;
        uint32_t acc_phase = 0;
        // output row m of the tile: dW2 rows, or dW1 rows (m < split) then dW3 rows
        auto out_row = [&](int e, int m) -> float* {
            return m < args.split
                       ? args.out0 + (static_cast<size_t>(e) * args.split + m) * args.N
                       : args.out1 + (static_cast<size_t>(e) * (args.M - args.split) +
                                      (m - args.split)) * args.N;
        };
        for (int tile = pair; tile < total; tile += npairs) {
            int e, mp, nt, r0, n_rows;
            tile_of(tile, e, mp, nt, r0, n_rows);
            const int m0 = mp * 2 * kRows + static_cast<int>(rank) * kRows;  // this CTA's rows
            const int col0 = nt * kN;
            if (n_rows == 0) {
                const int m = m0 + q * 32 + lane;
                if (m < args.M) {
                    float* out = out_row(e, m);
                    for (int col = col0; col < col0 + kN && col < args.N; col += 4)
                        *reinterpret_cast<float4*>(out + col) = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                continue;
            }
            if (!bar_all(mbar_wait_bounded(&bk.tmem_full[acc], acc_phase, abort_flag,
                                           args.status),
                         kVoteBarrier, kEpiThreads))
                break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(acc * kN);
            // rows past M (the peer's half of a last, partial pair tile) store nothing
            if (m0 + q * 32 < args.M) {
#pragma unroll 1
                for (int hf = 0; hf < 2; ++hf) {  // lanes 0..15 and 16..31 of this quarter
#pragma unroll 1
                    for (int cb = 0; cb < kN / 64; ++cb) {
                        uint32_t v[32];
                        tmem_ld_16x256b_x8(tbase + (static_cast<uint32_t>(hf * 16) << 16) + cb * 64, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int w = 0; w < 2; ++w) {
                            const int m = m0 + q * 32 + hf * 16 + r4 + 8 * w;
                            if (m >= args.M) continue;
                            float* out = out_row(e, m);
#pragma unroll
                            for (int rep = 0; rep < 8; ++rep) {
                                const int col = col0 + cb * 64 + rep * 8 + c2;
                                if (col < args.N)  // N is a multiple of 8: col + 1 < N too
                                    *reinterpret_cast<float2*>(out + col) =
                                        make_float2(bits_f32(v[4 * rep + 2 * w]),
                                                    bits_f32(v[4 * rep + 2 * w + 1]));
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
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the leader's MMAs into this CTA's TMEM and smem are done
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

}  // namespace

// Weight gradients on CTA pairs: A [rows, M] and B [rows, N] grouped bf16 operands
// (tensor maps with 64 x 64 boxes); fp32 outputs out0 [E, split, N] and out1
// [E, M - split, N].
cudaError_t launch_wgrad_pair(const CUtensorMap& A, const CUtensorMap& B, const int32_t* offsets,
                              int E, int rows,
                              int M, int N, int split, float* out0, float* out1, uint32_t* status,
                              int cap, cudaStream_t s, int pad_a, int pad_b) {
    static PerDeviceOnce smem_once;
    if (const cudaError_t err = opt_in_smem(smem_once, bwd_wgrad_pair_kernel, kSmemBytes);
        err != cudaSuccess)
        return err;
    PArgs p{offsets, E, rows, M, N, (M + 2 * kRows - 1) / (2 * kRows),
            (N + kN - 1) / kN, split, out0, out1, status, cap, pad_a, pad_b};
    const long long tiles = static_cast<long long>(E) * p.m_pairs * p.n_tiles;
    const int max_pairs = device_sm_count() / 2;
    const int npairs = static_cast<int>(tiles < max_pairs ? (tiles < 1 ? 1 : tiles) : max_pairs);
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
    cudaError_t err = cudaLaunchKernelEx(&cfg, bwd_wgrad_pair_kernel, A, B, p);
    return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
