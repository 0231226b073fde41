// backward_sm100.cu -- gradients of the layer for training.
//
// crackai "Mixtral of Experts", "Key Takeaways": routing is learned jointly with the
// model, so the backward pass reaches the router through the two gate weights.  The
// pages print no backward formulas; this is the exact derivative of the forward
// layer with the top-2 choice held fixed (it is piecewise constant in the inputs).
// For grouped row r = (token t, slot j) of expert e, with a = x W1^T, b = x W3^T:
//
//   dY[r]   = w[t,j] dy[t]                       (bf16, prep kernel)
//   dw[t,j] = <dy[t], Y[r]>                      (prep kernel; Y saved by the forward)
//   dH      = dY W2_e                            (GEMM, K = d; W2_e read MN-major)
//   du      = dH * b * silu'(a),  dv = dH * silu(a)
//                                                (GEMM recomputing a and b, K = d, with
//                                                 the elementwise step as its epilogue)
//   dX      = [du dv] [W1_e ; W3_e]              (GEMM, K = 2h; weights read MN-major)
//   dx[t]   = dX[r(t,0)] + dX[r(t,1)] + dlogits[t] Wg^T
//   dW2_e   = dY_e^T H_e,  [dW1_e ; dW3_e] = [du dv]_e^T x_e
//                                                (GEMMs whose reduction runs over the
//                                                 expert's own rows; both operands
//                                                 MN-major)
//   dlogits: the gap l_i1 - l_i2 gets (dw1 - dw2) w1 w2, logit i1 that, i2 minus that;
//   dWg     = x^T dlogits                        (CUDA cores, fixed-order reduction)
//
// The GEMMs use the same engine layout as the forward (persistent, warp-specialised:
// TMA producer, single-thread tcgen05.mma issuer, four epilogue warps; 128x256 fp32
// accumulators double-buffered in TMEM).  An operand stored with its M/N dimension
// contiguous is loaded as 64-column x 64-row boxes with 128-byte swizzle and handed to
// the tensor core as an MN-major operand (transpose bit in the instruction
// descriptor), so no weight or activation is ever transposed in memory.  In the
// weight-gradient GEMMs the reduction runs over an expert's rows, which start and
// end anywhere: the rows of a last, partial K block that belong to the next expert
// are zeroed in shared memory before the MMA reads them.  Every wait is bounded.
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
// Defined in grouped_gemm_pair_sm100.cu.
cudaError_t launch_bwd_rows_pair(int mode, const CUtensorMap& a, const CUtensorMap& b0,
                                 const CUtensorMap& b1, const int32_t* offsets, int E, int rows,
                                 int d, int h, void* out, const float* dH, uint32_t* status,
                                 int cap, cudaStream_t s, const uint8_t* skip_flag = nullptr);
// Defined in backward_pair_sm100.cu.
cudaError_t launch_wgrad_pair(const CUtensorMap& A, const CUtensorMap& B, const int32_t* offsets,
                              int E, int rows,
                              int M, int N, int split, float* out0, float* out1, uint32_t* status,
                              int cap, cudaStream_t s, int pad_a = 0, int pad_b = 0);

namespace {

constexpr int kBM = 128;                   // accumulator rows (TMEM lanes)
constexpr int kBK = 64;                    // K per stage
constexpr int kN = 256;                    // accumulator columns
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;     // 16 KiB
constexpr int kBBytes = kN * kBK * 2;      // 32 KiB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr uint32_t kTmemCols = 2 * kN;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 1024 /*bookkeeping*/;
// Weight-gradient epilogue: each epilogue warp stages 32-row x 32-column fp32 chunks
// (4 KiB) of its own accumulator rows for TMA stores, OUTBUFS buffers per warp.
constexpr int kStageOutBytes = 32 * 32 * 4;  // 4 KiB
template <int STAGES, int OUTBUFS>
constexpr int wgrad_smem_bytes() {
    return STAGES * kStageBytes + 4 * OUTBUFS * kStageOutBytes + 1024 /*align*/ + 1024 /*book*/;
}
constexpr int kVoteBarrier = 2;  // epilogue vote after a bounded wait
constexpr int kBox = kMnBoxBytes;          // one 64-column x 64-row box: 8 KiB

enum RowMode { kModeDH = 0, kModeDUV = 1, kModeDX = 2 };
enum WMode { kModeW2 = 0, kModeW13 = 1 };

struct Book {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int off[kMaxExperts + 1];
    int end[kMaxExperts];
    int tile_start[kMaxExperts + 1];
};
static_assert(sizeof(Book) <= 1024, "bookkeeping reserve");

// Group offsets (clamped, monotone) and kept ends; thread 0 only.
__device__ __forceinline__ void load_groups(Book& bk, const int32_t* offsets, int E, int rows,
                                            int cap) {
    int prev = 0;
    for (int g = 0; g <= E; ++g) {
        int v = offsets[g];
        v = v < prev ? prev : (v > rows ? rows : v);
        bk.off[g] = v;
        prev = v;
    }
    for (int g = 0; g < E; ++g) {
        const int n = bk.off[g + 1] - bk.off[g];
        bk.end[g] = bk.off[g] + (n < cap ? n : cap);
    }
}

__device__ __forceinline__ void init_barriers(Book& bk, int stages = kStages) {
    for (int s = 0; s < stages; ++s) {
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

// ================================================================ row-grouped GEMMs
// Tiles are (expert, 128-row block of its rows, 256-column block of the output), as in
// the forward; A is always the grouped activation [rows, K], K-major.
//   kModeDH : dH[r, :h]   = dY[r] . W2_e          B = W2_e [d, h] rows = k  (MN-major)
//   kModeDUV: du, dv      from a = x W1_e^T, b = x W3_e^T and dH (epilogue)
//             B = 128 rows of W1_e over the same 128 rows of W3_e (K-major, as GEMM1)
//   kModeDX : dX[r, :d]   = [du dv][r] . [W1_e ; W3_e]   B rows = k (MN-major),
//             k < h from W1, k >= h from W3
struct RowArgs {
    const int32_t* offsets;
    int E;
    int rows;
    int K;         // reduction length (d, d, 2h)
    int N;         // output columns (h, h, d)
    int n_tiles;
    int h;
    int d;
    void* out;         // dH fp32 [rows, h] | DUV bf16 [rows, 2h] | dX fp32 [rows, d]
    const float* dH;   // kModeDUV: dH fp32 [rows, h]
    uint32_t* status;
    int cap;
    // optional: the launch does nothing when bit 7 of this device byte is set (kModeDUV
    // after a forward that kept the pre-activations)
    const uint8_t* skip_flag;
};

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_rows_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, const RowArgs args) {
    constexpr bool kBmn = MODE != kModeDUV;
    constexpr uint32_t kIdesc = idesc_bf16_f32_major(kBM, kN, false, kBmn);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages * kABytes;
    Book& bk = *reinterpret_cast<Book*>(smem + kStages * kStageBytes);
    volatile int* abort_flag = &bk.abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = args.E;
    if (args.skip_flag != nullptr && (*args.skip_flag & kLayoutSavedAB) != 0) return;  // uniform

    if (threadIdx.x == 0) init_barriers(bk);
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB0);
        tma_prefetch_desc(&tmB1);
    }
    if (warp == 1) tmem_alloc(&bk.tmem_base, kTmemCols);
    if (threadIdx.x == 0) {
        load_groups(bk, args.offsets, E, args.rows, args.cap);
        bk.tile_start[0] = 0;
        for (int g = 0; g < E; ++g)
            bk.tile_start[g + 1] =
                bk.tile_start[g] + (bk.end[g] - bk.off[g] + kBM - 1) / kBM * args.n_tiles;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bk.tmem_base;
    const int total = bk.tile_start[E];
    const int num_kb = (args.K + kBK - 1) / kBK;

    auto tile_of = [&](int tile, int& e, int& row0, int& row_end, int& nt) {
        int g = 0;
        while (g + 1 < E && tile >= bk.tile_start[g + 1]) ++g;
        const int local = tile - bk.tile_start[g];
        const int m_tiles = (bk.end[g] - bk.off[g] + kBM - 1) / kBM;
        e = g;
        row0 = bk.off[g] + (local % m_tiles) * kBM;
        nt = local / m_tiles;
        row_end = bk.end[g];
    };

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, pending = 0, pending_phase = 0;
            bool ok = true;
            const uint64_t w_policy = l2_policy_evict_first();
            for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
                int e, row0, row_end, nt;
                tile_of(tile, e, row0, row_end, nt);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait_bounded(&bk.empty[stage], phase ^ 1u, abort_flag,
                                           args.status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bk.full[stage], kStageBytes);
                    const int kc = kb * kBK;
                    uint8_t* a = sA + stage * kABytes;
                    uint8_t* b = sB + stage * kBBytes;
                    tma_load_2d(&tmA, &bk.full[stage], a, kc, row0);
                    if (MODE == kModeDUV) {
                        const int brow = e * args.h + nt * 128;
                        tma_load_2d(&tmB0, &bk.full[stage], b, kc, brow);
                        tma_load_2d(&tmB1, &bk.full[stage], b + kBBytes / 2, kc, brow);
                    } else {
                        const CUtensorMap* map = &tmB0;
                        int krow;
                        if (MODE == kModeDH) {
                            krow = e * args.d + kc;
                        } else {
                            const bool second = kc >= args.h;
                            map = second ? &tmB1 : &tmB0;
                            krow = e * args.h + (second ? kc - args.h : kc);
                        }
                        // dH streams W2 once: first out of L2 (4-5% faster); dX keeps the
                        // default policy (slower with the hint)
#pragma unroll
                        for (int i = 0; i < kN / 64; ++i) {
                            if (MODE == kModeDH)
                                tma_load_2d_hint(map, &bk.full[stage], b + i * kBox,
                                                 nt * kN + 64 * i, krow, w_policy);
                            else
                                tma_load_2d(map, &bk.full[stage], b + i * kBox, nt * kN + 64 * i,
                                            krow);
                        }
                    }
                    pending |= 1u << stage;
                    pending_phase = (pending_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok)
                for (int s = 0; s < kStages; ++s)
                    if (pending & (1u << s)) drain_wait(&bk.full[s], (pending_phase >> s) & 1u);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true, issued = false;
            for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
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
                    const uint64_t bd = kBmn ? sw128_mn_desc(bs) : sw128_kmajor_desc(bs);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        umma_bf16(d_tmem, ad + kKDescStep * k, bd + (kBmn ? kMnDescStep : kKDescStep) * k,
                                  kIdesc, (kb | k) != 0);
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
                umma_commit(&bk.drain);
                drain_wait(&bk.drain, 0);
            }
        }
        __syncwarp();
    } else {
        const int q = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            int e, row0, row_end, nt;
            tile_of(tile, e, row0, row_end, nt);
            if (!bar_all(mbar_wait_bounded(&bk.tmem_full[acc], acc_phase, abort_flag,
                                           args.status),
                         kVoteBarrier, kEpiThreads))
                break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(acc * kN);
            const int row = row0 + q * 32 + lane;
            const bool valid = row < row_end;
            if (MODE == kModeDUV) {
                const int h = args.h;
                const float* g = args.dH + static_cast<size_t>(row) * h;
                __nv_bfloat16* du = static_cast<__nv_bfloat16*>(args.out) + static_cast<size_t>(row) * 2 * h;
                const int col0 = nt * 128;
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    uint32_t a[32], b[32];
                    tmem_ld_32cols(tbase + ch * 32, a);
                    tmem_ld_32cols(tbase + 128 + ch * 32, b);
                    tmem_ld_wait();
                    const int c0 = col0 + ch * 32;
                    if (valid && c0 < h) {
                        // h % 64 == 0, so a 32-column chunk is either whole or absent
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
                            float ru[2], rv[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const float av = bits_f32(a[2 * i + u]);
                                const float bv = bits_f32(b[2 * i + u]);
                                const float s = __frcp_rn(1.0f + __expf(-av));
                                ru[u] = gv[2 * i + u] * bv * (s * (1.0f + av * (1.0f - s)));
                                rv[u] = gv[2 * i + u] * (av * s);
                            }
                            pu[i] = pack_bf16x2(ru[0], ru[1]);
                            pv[i] = pack_bf16x2(rv[0], rv[1]);
                        }
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            *reinterpret_cast<uint4*>(du + c0 + 8 * v) =
                                make_uint4(pu[4 * v], pu[4 * v + 1], pu[4 * v + 2], pu[4 * v + 3]);
                            *reinterpret_cast<uint4*>(du + h + c0 + 8 * v) =
                                make_uint4(pv[4 * v], pv[4 * v + 1], pv[4 * v + 2], pv[4 * v + 3]);
                        }
                    }
                }
            } else {
                float* out = static_cast<float*>(args.out) + static_cast<size_t>(row) * args.N;
                const int col0 = nt * kN;
#pragma unroll 1
                for (int ch = 0; ch < 8; ++ch) {
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

// ================================================================ weight gradients
// out[e][m][n] = sum over the rows r of expert e of A[r, m] * B[r, n]: both operands
// are grouped activations, row-major with m / n contiguous (MN-major).  Tiles are
// (expert, 256-column block, 128-row block), row blocks inner so that consecutive
// tiles share B.  An expert with no rows gets a zero tile.
// The output is written by TMA (with an L2 evict-first hint), each epilogue warp on
// its own: a 32-column chunk of the warp's 32 accumulator rows goes to one of its
// staging buffers in the 128-byte-swizzled layout (row r at r * 128 bytes, 16-byte
// chunk j at position j ^ (r % 8), so the warp's stores hit distinct banks), and lane
// 0 stores it with a 3-D tensor store ([E, rows, cols]: rows past an expert's last
// are outside the tensor and not written).  A buffer is reused once its previous
// store has read it; no block-wide barrier is involved.  A tile that straddles the dW1 / dW3 boundary
// (h not a multiple of 128) is stored row by row instead.
// STAGES input stages and the staging buffers share the shared memory: a short
// reduction (few rows per expert) leaves the kernel bound by its output stores (more
// buffers); a long one wants deeper input stages.
// Tiles run column blocks innermost, so the CTAs running at one time write
// neighbouring parts of the same output rows.
//   kModeW2 : A = dY [rows, d], B = H [rows, h]         -> dW2 [E, d, h]
//   kModeW13: A = [du dv] [rows, 2h], B = x [rows, d]   -> dW1 [E, h, d] (m < h),
//                                                          dW3 [E, h, d] (m >= h)
struct WArgs {
    const int32_t* offsets;
    int E;
    int rows;
    int M;
    int N;
    int m_tiles;
    int n_tiles;
    int split;       // output rows m < split go to out0, the rest to out1
    float* out0;
    float* out1;
    uint32_t* status;
    int cap;
};

template <int MODE, int STAGES, int OUTBUFS>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_wgrad_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmO0,
                     const __grid_constant__ CUtensorMap tmO1, const WArgs args) {
    constexpr uint32_t kIdesc = idesc_bf16_f32_major(kBM, kN, true, true);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    static_assert(STAGES >= 2 && STAGES <= kStages && OUTBUFS >= 2, "pipeline shape");
    static_assert(wgrad_smem_bytes<STAGES, OUTBUFS>() <= 232448, "shared memory");
    uint8_t* sB = smem + STAGES * kABytes;
    uint8_t* sOut = smem + STAGES * kStageBytes;  // staging buffers, 1 KiB aligned
    Book& bk = *reinterpret_cast<Book*>(sOut + 4 * OUTBUFS * kStageOutBytes);
    volatile int* abort_flag = &bk.abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = args.E;

    if (threadIdx.x == 0) init_barriers(bk, STAGES);
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmO0);
        tma_prefetch_desc(&tmO1);
    }
    if (warp == 1) tmem_alloc(&bk.tmem_base, kTmemCols);
    if (threadIdx.x == 0) load_groups(bk, args.offsets, E, args.rows, args.cap);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bk.tmem_base;
    const int per_e = args.m_tiles * args.n_tiles;
    const int total = E * per_e;

    auto tile_of = [&](int tile, int& e, int& mt, int& nt, int& r0, int& n_rows) {
        e = tile / per_e;
        const int local = tile - e * per_e;
        nt = local % args.n_tiles;
        mt = local / args.n_tiles;
        r0 = bk.off[e];
        n_rows = bk.end[e] - bk.off[e];
    };

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, pending = 0, pending_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
                int e, mt, nt, r0, n_rows;
                tile_of(tile, e, mt, nt, r0, n_rows);
                const int nkb = (n_rows + kBK - 1) / kBK;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait_bounded(&bk.empty[stage], phase ^ 1u, abort_flag,
                                           args.status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bk.full[stage], kStageBytes);
                    const int r = r0 + kb * kBK;
                    uint8_t* a = sA + stage * kABytes;
                    uint8_t* b = sB + stage * kBBytes;
#pragma unroll
                    for (int i = 0; i < kBM / 64; ++i)
                        tma_load_2d(&tmA, &bk.full[stage], a + i * kBox, mt * kBM + 64 * i, r);
#pragma unroll
                    for (int i = 0; i < kN / 64; ++i)
                        tma_load_2d(&tmB, &bk.full[stage], b + i * kBox, nt * kN + 64 * i, r);
                    pending |= 1u << stage;
                    pending_phase = (pending_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok)
                for (int s = 0; s < STAGES; ++s)
                    if (pending & (1u << s)) drain_wait(&bk.full[s], (pending_phase >> s) & 1u);
        }
        __syncwarp();
    } else if (warp == 1) {
        // The whole warp runs this loop: lane 0 waits and issues, all lanes zero the
        // rows of a last partial K block that belong to the next expert.
        int stage = 0, acc = 0;
        uint32_t phase = 0, acc_phase = 0;
        bool ok = true, issued = false;
        for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
            int e, mt, nt, r0, n_rows;
            tile_of(tile, e, mt, nt, r0, n_rows);
            const int nkb = (n_rows + kBK - 1) / kBK;
            if (nkb == 0) continue;  // zero tile: written by the epilogue alone
            int got = 1;
            if (lane == 0)
                got = mbar_wait_bounded(&bk.tmem_empty[acc], acc_phase ^ 1u, abort_flag,
                                        args.status);
            ok = __shfl_sync(0xffffffffu, got, 0) != 0;
            if (!ok) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kN);
            for (int kb = 0; kb < nkb; ++kb) {
                if (lane == 0) got = mbar_wait_bounded(&bk.full[stage], phase, abort_flag, args.status);
                ok = __shfl_sync(0xffffffffu, got, 0) != 0;
                if (!ok) break;
                const int kv = n_rows - kb * kBK;  // rows of this block inside the group
                if (kv < kBK) {
                    // Rows kv..63 belong to the next group: clear them in A (its rows
                    // there may never have been written, e.g. dropped pairs' dY); with a
                    // capacity, B's dropped rows may hold garbage too, so clear B as well.
                    uint8_t* a = sA + stage * kABytes;
                    uint8_t* b = sB + stage * kBBytes;
                    const int nz = (kBK - kv) * 8;  // 16-byte chunks per box to clear
                    const int boxes = (args.cap != INT_MAX ? kBM + kN : kBM) / 64;
                    for (int i = lane; i < boxes * nz; i += 32) {
                        const int box = i / nz, c = i - box * nz;
                        uint8_t* base = box < kBM / 64 ? a + box * kBox : b + (box - kBM / 64) * kBox;
                        *reinterpret_cast<uint4*>(base + kv * 128 + c * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                if (lane == 0) {
                    tc_fence_after();
                    const uint64_t ad = sw128_mn_desc(smem_u32(sA + stage * kABytes));
                    const uint64_t bd = sw128_mn_desc(smem_u32(sB + stage * kBBytes));
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        umma_bf16(d_tmem, ad + kMnDescStep * k, bd + kMnDescStep * k, kIdesc,
                                  (kb | k) != 0);
                    umma_commit(&bk.empty[stage]);
                }
                issued = true;
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (lane == 0) umma_commit(&bk.tmem_full[acc]);
            __syncwarp();
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (!ok && issued && lane == 0) {
            umma_commit(&bk.drain);
            drain_wait(&bk.drain, 0);
        }
        __syncwarp();
    } else {
        const int q = warp & 3;
        const int r = q * 32 + lane;          // accumulator row of this thread
        uint8_t* wstage = sOut + q * OUTBUFS * kStageOutBytes;  // this warp's buffers
        // The gradients are written once and not read again here: first out of L2, so
        // that the stream of them does not evict the operand rows the next tiles reuse.
        const uint64_t out_policy = l2_policy_evict_first();
        int acc = 0, buf = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            int e, mt, nt, r0, n_rows;
            tile_of(tile, e, mt, nt, r0, n_rows);
            const int m0 = mt * kBM;
            const int m = m0 + r;
            const bool mvalid = m < args.M;
            float* out = m < args.split
                             ? args.out0 + (static_cast<size_t>(e) * args.split + m) * args.N
                             : args.out1 + (static_cast<size_t>(e) * (args.M - args.split) +
                                            (m - args.split)) * args.N;
            const int col0 = nt * kN;
            if (n_rows == 0) {
                if (mvalid)
                    for (int col = col0; col < col0 + kN && col < args.N; col += 4)
                        *reinterpret_cast<float4*>(out + col) = make_float4(0.f, 0.f, 0.f, 0.f);
                continue;
            }
            if (!bar_all(mbar_wait_bounded(&bk.tmem_full[acc], acc_phase, abort_flag,
                                           args.status),
                         kVoteBarrier, kEpiThreads))
                break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(acc * kN);
            const bool second = m0 >= args.split;
            const bool straddle = m0 < args.split && m0 + kBM > args.split;
#pragma unroll 1
            for (int ch = 0; ch < 8; ++ch) {
                uint32_t v[32];
                tmem_ld_32cols(tbase + ch * 32, v);
                tmem_ld_wait();
                if (!straddle) {
                    uint8_t* st = wstage + buf * kStageOutBytes;
                    if (lane == 0) bulk_wait_group_read<OUTBUFS - 1>();  // buffer free again
                    __syncwarp();
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<uint4*>(st + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                            make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_3d_hint(second ? &tmO1 : &tmO0, st, col0 + ch * 32,
                                          (second ? m0 - args.split : m0) + q * 32, e,
                                          out_policy);
                        bulk_commit_group();
                    }
                    if (++buf == OUTBUFS) buf = 0;
                } else if (mvalid) {
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
            tc_fence_before();
            mbar_arrive(&bk.tmem_empty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (lane == 0) bulk_wait_group<0>();  // every store complete before the block exits
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ================================================================ CUDA-core kernels
constexpr int kPrepThreads = 256;

// du, dv from dH and the pre-activations a, b that moe_layer_forward_train kept, element
// by element, with the formula of the recomputing GEMM's epilogue: the same a and b
// (the forward's GEMM1 accumulators) give the same du and dv.  Does nothing unless the
// forward's layout byte says that a and b were kept (then the recomputing GEMM does
// nothing instead).  du in columns [0, h) of each DUV row, dv in [h, 2h).
__global__ void __launch_bounds__(kPrepThreads)
    bwd_duv_saved_kernel(const uint8_t* __restrict__ y_layout, const float* __restrict__ dH,
                         const float* __restrict__ a_pre, const float* __restrict__ b_pre,
                         int P, int h, __nv_bfloat16* __restrict__ duv) {
    if ((*y_layout & kLayoutSavedAB) == 0) return;
    const int h4 = h / 4;
    const size_t n = static_cast<size_t>(P) * h4;
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const size_t r = i / h4;
        const size_t c = (i - r * h4) * 4;
        const float4 g = *reinterpret_cast<const float4*>(dH + r * h + c);
        const float4 a = *reinterpret_cast<const float4*>(a_pre + r * h + c);
        const float4 b = *reinterpret_cast<const float4*>(b_pre + r * h + c);
        const float gv[4] = {g.x, g.y, g.z, g.w}, av4[4] = {a.x, a.y, a.z, a.w},
                    bv4[4] = {b.x, b.y, b.z, b.w};
        float ru[4], rv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float av = av4[u];
            const float bv = bv4[u];
            const float s = __frcp_rn(1.0f + __expf(-av));
            ru[u] = gv[u] * bv * (s * (1.0f + av * (1.0f - s)));
            rv[u] = gv[u] * (av * s);
        }
        __nv_bfloat16* row = duv + r * 2 * h;
        *reinterpret_cast<uint2*>(row + c) = make_uint2(pack_bf16x2(ru[0], ru[1]), pack_bf16x2(ru[2], ru[3]));
        *reinterpret_cast<uint2*>(row + h + c) =
            make_uint2(pack_bf16x2(rv[0], rv[1]), pack_bf16x2(rv[2], rv[3]));
    }
}

// Is pair (t, j) kept?  (expert id valid, grouped row in range, within capacity)
__device__ __forceinline__ bool pair_kept(const int32_t* idx, const int32_t* offsets,
                                          const int32_t* inv, int f, int E, int P, int cap) {
    const unsigned e = static_cast<unsigned>(idx[f]);
    const unsigned r = static_cast<unsigned>(inv[f]);
    if (e >= static_cast<unsigned>(E) || r >= static_cast<unsigned>(P)) return false;
    return cap == INT_MAX || static_cast<int>(r) - offsets[e] < cap;
}

// One block per token: dY rows of its two pairs, dw, and the token's logit gradients.
// Small batches (kSplit) may have left their expert outputs as split-K partials in
// Ypart (split_stride floats apart, summed in order) and the byte at y_layout says
// whether they did; larger batches always leave them in Y, and their form keeps its
// register count low for streaming.
template <bool kSplit>
__global__ void __launch_bounds__(kPrepThreads)
    bwd_prep_kernel(const __nv_bfloat16* __restrict__ dy, const int32_t* __restrict__ idx,
                    const float* __restrict__ w, const int32_t* __restrict__ inv,
                    const int32_t* __restrict__ offsets, int T, int d, int E, int cap,
                    const float* __restrict__ Y1, const float* __restrict__ Ypart,
                    const uint8_t* __restrict__ y_layout, size_t split_stride,
                    __nv_bfloat16* __restrict__ dY, float* __restrict__ dw,
                    float* __restrict__ dlogits) {
    __shared__ float red[2][kPrepThreads / 32];
    const int P = 2 * T;
    int nsplit = kSplit ? (*y_layout & kLayoutSplitMask) : 1;
    nsplit = nsplit < 1 ? 1 : (nsplit > kDecodeSplitK ? kDecodeSplitK : nsplit);
    const float* __restrict__ Y = nsplit > 1 ? Ypart : Y1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int d4 = d >> 2;  // d % 8 == 0: rows of Y, dy and dY hold whole 4-column groups
    const size_t stride4 = split_stride >> 2;
    const float4* __restrict__ Y4 = reinterpret_cast<const float4*>(Y);
    // Expert output row r, columns 4c..4c+3: the partials summed in order.  Every
    // partial is loaded before the first add, so the loads overlap instead of forming
    // a chain of dependent misses.
    auto y_row = [&](int r, int c) {
        const size_t at = static_cast<size_t>(r) * d4 + c;
        if constexpr (!kSplit) {
            return Y4[at];
        } else {
            float4 p[kDecodeSplitK];
#pragma unroll
            for (int s = 0; s < kDecodeSplitK; ++s)
                if (s < nsplit) p[s] = Y4[s * stride4 + at];
            float4 y = p[0];
#pragma unroll
            for (int s = 1; s < kDecodeSplitK; ++s)
                if (s < nsplit) {
                    y.x += p[s].x;
                    y.y += p[s].y;
                    y.z += p[s].z;
                    y.w += p[s].w;
                }
            return y;
        }
    };
    auto store_dy = [&](int r, int c, float wt, const float (&g)[4]) {
        uint2 v;
        v.x = pack_bf16x2(wt * g[0], wt * g[1]);
        v.y = pack_bf16x2(wt * g[2], wt * g[3]);
        *reinterpret_cast<uint2*>(dY + static_cast<size_t>(r) * d + 4 * c) = v;
    };
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        const bool keep0 = pair_kept(idx, offsets, inv, 2 * t, E, P, cap);
        const bool keep1 = pair_kept(idx, offsets, inv, 2 * t + 1, E, P, cap);
        const int r0 = inv[2 * t], r1 = inv[2 * t + 1];
        const float w0 = keep0 ? w[2 * t] : 0.f, w1 = keep1 ? w[2 * t + 1] : 0.f;
        float s0 = 0.f, s1 = 0.f;
        for (int c = threadIdx.x; c < d4; c += blockDim.x) {
            const uint2 graw =
                *reinterpret_cast<const uint2*>(dy + static_cast<size_t>(t) * d + 4 * c);
            const float g[4] = {bf16_lo(graw.x), bf16_hi(graw.x), bf16_lo(graw.y),
                                bf16_hi(graw.y)};
            if (keep0) {
                const float4 y = y_row(r0, c);
                s0 = fmaf(g[0], y.x, s0);
                s0 = fmaf(g[1], y.y, s0);
                s0 = fmaf(g[2], y.z, s0);
                s0 = fmaf(g[3], y.w, s0);
                store_dy(r0, c, w0, g);
            }
            if (keep1) {
                const float4 y = y_row(r1, c);
                s1 = fmaf(g[0], y.x, s1);
                s1 = fmaf(g[1], y.y, s1);
                s1 = fmaf(g[2], y.z, s1);
                s1 = fmaf(g[3], y.w, s1);
                store_dy(r1, c, w1, g);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            s0 += __shfl_xor_sync(0xffffffffu, s0, o);
            s1 += __shfl_xor_sync(0xffffffffu, s1, o);
        }
        if (lane == 0) {
            red[0][warp] = s0;
            red[1][warp] = s1;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            float a = 0.f, b = 0.f;
            for (int i = 0; i < kPrepThreads / 32; ++i) {
                a += red[0][i];
                b += red[1][i];
            }
            dw[2 * t] = a;
            dw[2 * t + 1] = b;
            // w1 = sigma(l_i1 - l_i2), w2 = 1 - w1 (the stored weights, even if dropped)
            const float gap = (a - b) * w[2 * t] * w[2 * t + 1];
            for (int e = 0; e < E; ++e) dlogits[static_cast<size_t>(t) * E + e] = 0.f;
            const unsigned e0 = static_cast<unsigned>(idx[2 * t]);
            const unsigned e1 = static_cast<unsigned>(idx[2 * t + 1]);
            if (e0 < static_cast<unsigned>(E)) dlogits[static_cast<size_t>(t) * E + e0] += gap;
            if (e1 < static_cast<unsigned>(E)) dlogits[static_cast<size_t>(t) * E + e1] -= gap;
        }
        __syncthreads();
    }
}

// dx[t, c] = dX[r0, c] + dX[r1, c] (kept pairs) + sum_e dlogits[t, e] Wg[c, e], one
// rounding.  Four columns per thread (d % 8 == 0), 16-byte loads of dX.
__global__ void __launch_bounds__(kPrepThreads)
    bwd_dx_kernel(const float* __restrict__ dX, const int32_t* __restrict__ idx,
                  const int32_t* __restrict__ inv, const int32_t* __restrict__ offsets, int T,
                  int d, int E, int cap, const float* __restrict__ dlogits,
                  const __nv_bfloat16* __restrict__ Wg, __nv_bfloat16* __restrict__ dx) {
    const int P = 2 * T;
    const int d4 = d / 4;
    // One token per block iteration: its routing (which pairs were kept, their rows,
    // its logit gradients) is read once, then the columns run with independent loads.
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        const bool keep0 = pair_kept(idx, offsets, inv, 2 * t, E, P, cap);
        const bool keep1 = pair_kept(idx, offsets, inv, 2 * t + 1, E, P, cap);
        const float4* __restrict__ row0 =
            reinterpret_cast<const float4*>(dX + static_cast<size_t>(inv[2 * t]) * d);
        const float4* __restrict__ row1 =
            reinterpret_cast<const float4*>(dX + static_cast<size_t>(inv[2 * t + 1]) * d);
        const float* dl = dlogits + static_cast<size_t>(t) * E;
        float g8[8];
        if (E == 8) {
#pragma unroll
            for (int e = 0; e < 8; ++e) g8[e] = dl[e];
        }
#pragma unroll 2
        for (int c4 = threadIdx.x; c4 < d4; c4 += blockDim.x) {
            const int c = 4 * c4;
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            if (keep0) {
                const float4 a = row0[c4];
                v[0] += a.x;
                v[1] += a.y;
                v[2] += a.z;
                v[3] += a.w;
            }
            if (keep1) {
                const float4 a = row1[c4];
                v[0] += a.x;
                v[1] += a.y;
                v[2] += a.z;
                v[3] += a.w;
            }
            if (E == 8) {
                // W_g rows of the four columns: one 16-byte load each
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint4 q =
                        *reinterpret_cast<const uint4*>(Wg + static_cast<size_t>(c + u) * 8);
                    const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int p2 = 0; p2 < 4; ++p2) {
                        v[u] = fmaf(g8[2 * p2], bf16_lo(w4[p2]), v[u]);
                        v[u] = fmaf(g8[2 * p2 + 1], bf16_hi(w4[p2]), v[u]);
                    }
                }
            } else {
                for (int e = 0; e < E; ++e) {
                    const float g = dl[e];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        v[u] = fmaf(g, __bfloat162float(Wg[static_cast<size_t>(c + u) * E + e]),
                                    v[u]);
                }
            }
            uint2 o;
            o.x = pack_bf16x2(v[0], v[1]);
            o.y = pack_bf16x2(v[2], v[3]);
            *reinterpret_cast<uint2*>(dx + static_cast<size_t>(t) * d + c) = o;
        }
    }
}

// Padded copies of two grouped bf16 arrays [rows, d]: expert e's n_e rows move to
// row poff[e] = sum over g < e of round_up(n_g, 64) and are followed by zero rows up to
// the next multiple of 64.  A weight-gradient GEMM that reads one operand this way finds
// zeros in the rows past each expert's end, so every 64-row K block is a whole one.
constexpr int kPadRowAlign = 64;

__global__ void __launch_bounds__(kPrepThreads)
    bwd_pad_kernel(const int32_t* __restrict__ offsets, int E, int rows, int d8,
                   const uint4* __restrict__ src0, const uint4* __restrict__ src1,
                   uint4* __restrict__ dst0, uint4* __restrict__ dst1) {
    __shared__ int off[kMaxExperts + 1], poff[kMaxExperts + 1];
    if (threadIdx.x == 0) {
        int prev = 0;
        poff[0] = 0;
        for (int g = 0; g <= E; ++g) {
            int v = offsets[g];
            v = v < prev ? prev : (v > rows ? rows : v);
            off[g] = v;
            if (g > 0) {
                const int n = v - prev;
                poff[g] = poff[g - 1] + (n + kPadRowAlign - 1) / kPadRowAlign * kPadRowAlign;
            }
            prev = v;
        }
    }
    __syncthreads();
    for (int pr = blockIdx.x; pr < poff[E]; pr += gridDim.x) {
        int e = 0;
        while (e + 1 < E && pr >= poff[e + 1]) ++e;
        const int i = pr - poff[e];
        const bool data = i < off[e + 1] - off[e];
        const size_t src = static_cast<size_t>(off[e] + i) * d8;
        const size_t dst = static_cast<size_t>(pr) * d8;
        for (int c = threadIdx.x; c < d8; c += blockDim.x) {
            const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
            const uint4 v0 = data ? src0[src + c] : zero;
            const uint4 v1 = data ? src1[src + c] : zero;
            dst0[dst + c] = v0;
            dst1[dst + c] = v1;
        }
    }
}

// dWg = x^T dlogits in two deterministic passes: per chunk of kWgChunk tokens a
// partial [d, E], then the partials summed in chunk order.
constexpr int kWgChunk = 64;

// EMAX: the accumulator count (8 when E <= 8, else kMaxExperts); each thread owns two
// adjacent columns and runs the chunk's tokens in order, so the sums do not depend on
// the launch shape.
template <int EMAX>
__global__ void __launch_bounds__(kPrepThreads)
    bwd_dwg_partial_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ dlogits,
                           int T, int d, int E, float* __restrict__ part) {
    __shared__ __align__(16) float dl[kWgChunk * EMAX];
    const int chunk = blockIdx.y;
    const int t0 = chunk * kWgChunk;
    const int nt = min(kWgChunk, T - t0);
    // the chunk's logit gradients, E per token, zero-padded to EMAX
    for (int i = threadIdx.x; i < nt * EMAX; i += blockDim.x) {
        const int t = i / EMAX, e = i - t * EMAX;
        dl[i] = e < E ? dlogits[static_cast<size_t>(t0 + t) * E + e] : 0.f;
    }
    __syncthreads();
    const int c = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (c >= d) return;
    float acc0[EMAX], acc1[EMAX];
#pragma unroll
    for (int e = 0; e < EMAX; ++e) acc0[e] = acc1[e] = 0.f;
    const uint32_t* __restrict__ xc =
        reinterpret_cast<const uint32_t*>(x + static_cast<size_t>(t0) * d + c);
    const int d2 = d / 2;
#pragma unroll 4
    for (int t = 0; t < nt; ++t) {
        const uint32_t xv = xc[static_cast<size_t>(t) * d2];
        const float x0 = bf16_lo(xv), x1 = bf16_hi(xv);
#pragma unroll
        for (int e = 0; e < EMAX; ++e) {
            const float g = dl[t * EMAX + e];
            acc0[e] = fmaf(x0, g, acc0[e]);
            acc1[e] = fmaf(x1, g, acc1[e]);
        }
    }
    float* out = part + (static_cast<size_t>(chunk) * d + c) * E;
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
        if (e < E) {
            out[e] = acc0[e];
            out[E + e] = acc1[e];
        }
}

__global__ void __launch_bounds__(kPrepThreads)
    bwd_dwg_reduce_kernel(const float* __restrict__ part, int nchunk, int d, int E,
                          float* __restrict__ dWg) {
    const size_t n = static_cast<size_t>(d) * E;
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        float s = part[i];
        for (int c = 1; c < nchunk; ++c) s += part[static_cast<size_t>(c) * n + i];
        dWg[i] = s;
    }
}

// Opt each GEMM kernel into its dynamic shared memory once per device.  `slot` names
// the kernel: the instantiations share one function type, so it cannot be the key.
enum KernelSlot { kSlotDH, kSlotDUV, kSlotDX, kSlotW2, kSlotW13, kSlotW2s, kSlotW13s, kSlots };
template <typename Kern>
cudaError_t configure(Kern kern, KernelSlot slot, int smem_bytes) {
    static PerDeviceOnce once[kSlots];
    return opt_in_smem(once[slot], kern, smem_bytes);
}

// Grouped rows at or below which the weight-gradient GEMMs use the store-bound shape.
constexpr int kWgradShortRows = 1024;
constexpr int kWgradLong[2] = {4, 2};   // input stages, staging buffers per epilogue warp
constexpr int kWgradShort[2] = {2, 8};

template <int MODE>
cudaError_t launch_wgrad(bool short_k, int grid, cudaStream_t s, const CUtensorMap& A,
                         const CUtensorMap& B, const CUtensorMap& O0, const CUtensorMap& O1,
                         const WArgs& w) {
    if (short_k) {
        constexpr int st = kWgradShort[0], ob = kWgradShort[1];
        auto kern = bwd_wgrad_kernel<MODE, st, ob>;
        const cudaError_t err =
            configure(kern, MODE == kModeW2 ? kSlotW2s : kSlotW13s, wgrad_smem_bytes<st, ob>());
        if (err != cudaSuccess) return err;
        return launch_k(kern, grid, kThreads, wgrad_smem_bytes<st, ob>(), s, A, B, O0, O1, w);
    }
    constexpr int st = kWgradLong[0], ob = kWgradLong[1];
    auto kern = bwd_wgrad_kernel<MODE, st, ob>;
    const cudaError_t err =
        configure(kern, MODE == kModeW2 ? kSlotW2 : kSlotW13, wgrad_smem_bytes<st, ob>());
    if (err != cudaSuccess) return err;
    return launch_k(kern, grid, kThreads, wgrad_smem_bytes<st, ob>(), s, A, B, O0, O1, w);
}

int grid_for(long long work, int cap) {
    return static_cast<int>(work < 1 ? 1 : (work < cap ? work : cap));
}

}  // namespace

size_t bwd_dwg_chunks(int T) { return static_cast<size_t>((T + kWgChunk - 1) / kWgChunk); }

cudaError_t launch_layer_backward(const BwdArgs& a, cudaStream_t s) {
    const int T = a.T, d = a.d, h = a.h, E = a.E, P = 2 * T;
    const int sms = device_sm_count();
    cudaError_t err;
    auto mark = [&](int i) -> cudaError_t {  // optional events between the launches
        return (i < a.n_ev && a.ev[i]) ? cudaEventRecord(a.ev[i], s) : cudaSuccess;
    };
    if ((err = mark(0)) != cudaSuccess) return err;
    // 1. dY, dw, dlogits
    err = launch_k(P <= kFusedMaxRows ? bwd_prep_kernel<true> : bwd_prep_kernel<false>,
                   grid_for(T, 8 * sms), kPrepThreads, 0, s,
                   static_cast<const __nv_bfloat16*>(a.dy), a.idx, a.w, a.inv, a.offsets, T, d, E,
                   a.cap, a.Y, a.Ypart, a.y_layout, a.split_stride,
                   static_cast<__nv_bfloat16*>(a.dY), a.dw, a.dlogits);
    if (err != cudaSuccess || (err = mark(1)) != cudaSuccess) return err;

    CUtensorMap m_dY128, m_W2, m_x, m_W1r, m_W3r, m_duv128, m_W1mn, m_W3mn;
    if (!encode_bf16_2d(&m_dY128, a.dY, P, d, kBM) ||
        !encode_bf16_2d(&m_W2, a.W2, static_cast<uint64_t>(E) * d, h, 64) ||
        !encode_bf16_2d(&m_x, a.x_perm, P, d, kBM) ||
        !encode_bf16_2d(&m_W1r, a.W1, static_cast<uint64_t>(E) * h, d, 128) ||
        !encode_bf16_2d(&m_W3r, a.W3, static_cast<uint64_t>(E) * h, d, 128) ||
        !encode_bf16_2d(&m_duv128, a.DUV, P, 2 * h, kBM) ||
        !encode_bf16_2d(&m_W1mn, a.W1, static_cast<uint64_t>(E) * h, d, 64) ||
        !encode_bf16_2d(&m_W3mn, a.W3, static_cast<uint64_t>(E) * h, d, 64))
        return cudaErrorInvalidValue;
    const long long row_blocks = (static_cast<long long>(P) + 127LL * E) / kBM;
    // Many rows: the CTA-pair forms of the three row GEMMs (the forward's pair engine).
    const bool pairs = P >= kBwdPairMinRows && pair_gemm_enabled();

    // 2. dH = dY W2_e
    if (pairs) {
        err = launch_bwd_rows_pair(0, m_dY128, m_W2, m_W2, a.offsets, E, P, d, h, a.dH, nullptr,
                                   a.status, a.cap, s);
        if (err != cudaSuccess || (err = mark(2)) != cudaSuccess) return err;
    } else {
        RowArgs r{a.offsets, E, P, d, h, (h + kN - 1) / kN, h, d, a.dH, nullptr, a.status, a.cap};
        if ((err = configure(bwd_rows_kernel<kModeDH>, kSlotDH, kSmemBytes)) != cudaSuccess)
            return err;
        err = launch_k(bwd_rows_kernel<kModeDH>, grid_for(row_blocks * r.n_tiles, sms), kThreads,
                       kSmemBytes, s, m_dY128, m_W2, m_W2, r);
        if (err != cudaSuccess || (err = mark(2)) != cudaSuccess) return err;
    }
    // 3. du, dv: from the pre-activations the forward kept (moe_layer_forward_train), or
    // recomputing a and b; the forward's layout byte selects which of the two launches
    // does the work (the other returns at once), so the host never waits for it
    if (a.a_pre != nullptr) {
        const long long n4 = static_cast<long long>(P) * (h / 4);
        err = launch_k(bwd_duv_saved_kernel,
                       grid_for((n4 + kPrepThreads - 1) / kPrepThreads, 8 * sms), kPrepThreads, 0,
                       s, a.y_layout, static_cast<const float*>(a.dH), a.a_pre, a.b_pre, P, h,
                       static_cast<__nv_bfloat16*>(a.DUV));
        if (err != cudaSuccess) return err;
    }
    const uint8_t* duv_skip = a.a_pre != nullptr ? a.y_layout : nullptr;
    if (pairs) {
        err = launch_bwd_rows_pair(1, m_x, m_W1r, m_W3r, a.offsets, E, P, d, h, a.DUV, a.dH,
                                   a.status, a.cap, s, duv_skip);
        if (err != cudaSuccess || (err = mark(3)) != cudaSuccess) return err;
    } else {
        RowArgs r{a.offsets, E, P, d, h, (h + 127) / 128, h, d, a.DUV, a.dH, a.status, a.cap,
                  duv_skip};
        if ((err = configure(bwd_rows_kernel<kModeDUV>, kSlotDUV, kSmemBytes)) != cudaSuccess)
            return err;
        err = launch_k(bwd_rows_kernel<kModeDUV>, grid_for(row_blocks * r.n_tiles, sms),
                       kThreads, kSmemBytes, s, m_x, m_W1r, m_W3r, r);
        if (err != cudaSuccess || (err = mark(3)) != cudaSuccess) return err;
    }
    // 4. dX = [du dv] [W1_e ; W3_e]
    if (pairs) {
        err = launch_bwd_rows_pair(2, m_duv128, m_W1mn, m_W3mn, a.offsets, E, P, d, h, a.dX,
                                   nullptr, a.status, a.cap, s);
        if (err != cudaSuccess || (err = mark(4)) != cudaSuccess) return err;
    } else {
        RowArgs r{a.offsets, E, P, 2 * h, d, (d + kN - 1) / kN, h, d, a.dX, nullptr, a.status,
                  a.cap};
        if ((err = configure(bwd_rows_kernel<kModeDX>, kSlotDX, kSmemBytes)) != cudaSuccess)
            return err;
        err = launch_k(bwd_rows_kernel<kModeDX>, grid_for(row_blocks * r.n_tiles, sms), kThreads,
                       kSmemBytes, s, m_duv128, m_W1mn, m_W3mn, r);
        if (err != cudaSuccess || (err = mark(4)) != cudaSuccess) return err;
    }
    // 5. dx
    {
        err = launch_k(bwd_dx_kernel, grid_for(T, 8 * sms),
                       kPrepThreads, 0, s, static_cast<const float*>(a.dX), a.idx, a.inv,
                       a.offsets, T, d, E, a.cap, static_cast<const float*>(a.dlogits),
                       static_cast<const __nv_bfloat16*>(a.Wg), static_cast<__nv_bfloat16*>(a.dx));
        if (err != cudaSuccess || (err = mark(5)) != cudaSuccess) return err;
    }
    // 6. weight gradients
    CUtensorMap m_dY64, m_H64, m_duv64, m_x64, m_dW2, m_dW1, m_dW3;
    if (!encode_bf16_2d(&m_dY64, a.dY, P, d, 64) || !encode_bf16_2d(&m_H64, a.H, P, h, 64) ||
        !encode_bf16_2d(&m_duv64, a.DUV, P, 2 * h, 64) ||
        !encode_bf16_2d(&m_x64, a.x_perm, P, d, 64) ||
        !encode_f32_3d(&m_dW2, a.dW2, E, d, h, 32, 32) ||
        !encode_f32_3d(&m_dW1, a.dW1, E, h, d, 32, 32) ||
        !encode_f32_3d(&m_dW3, a.dW3, E, h, d, 32, 32))
        return cudaErrorInvalidValue;
    // Few rows per expert: the output stores bound the kernel (single-SM kernel with
    // deep staging); many: the reduction does (CTA pairs, deep input pipeline).
    if (P <= kWgradShortRows) {
        WArgs w{a.offsets, E, P, d, h, (d + kBM - 1) / kBM, (h + kN - 1) / kN, d, a.dW2, a.dW2,
                a.status, a.cap};
        err = launch_wgrad<kModeW2>(true, grid_for(static_cast<long long>(E) * w.m_tiles * w.n_tiles, sms),
                                    s, m_dY64, m_H64, m_dW2, m_dW2, w);
        if (err != cudaSuccess || (err = mark(6)) != cudaSuccess) return err;
        WArgs w13{a.offsets, E, P, 2 * h, d, (2 * h + kBM - 1) / kBM, (d + kN - 1) / kN, h,
                  a.dW1, a.dW3, a.status, a.cap};
        err = launch_wgrad<kModeW13>(true, grid_for(static_cast<long long>(E) * w13.m_tiles * w13.n_tiles, sms),
                                     s, m_duv64, m_x64, m_dW1, m_dW3, w13);
        if (err != cudaSuccess || (err = mark(7)) != cudaSuccess) return err;
    } else {
        // CTA pairs.  Without a capacity, one operand of each GEMM is read from a copy
        // whose experts are padded with zero rows (dY for dW2, x_perm for dW1/dW3), so
        // every K block is whole; the other operand's rows past an expert's end are the
        // next expert's (finite) rows or outside the array (zero-filled by TMA).  With a
        // capacity the dropped rows were never written, so the kernel clears the rows
        // of partial blocks in shared memory instead.
        const bool padded = a.cap == INT_MAX;
        CUtensorMap m_dYp64, m_xp64;
        if (padded) {
            const unsigned pad_rows = static_cast<unsigned>(bwd_pad_rows(T, E));
            if (!encode_bf16_2d(&m_dYp64, a.dY_pad, pad_rows, d, 64) ||
                !encode_bf16_2d(&m_xp64, a.x_pad, pad_rows, d, 64))
                return cudaErrorInvalidValue;
            err = launch_k(bwd_pad_kernel, grid_for(static_cast<long long>(pad_rows), 8 * sms),
                           kPrepThreads, 0, s, a.offsets, E, P, d / 8,
                           static_cast<const uint4*>(a.dY), static_cast<const uint4*>(a.x_perm),
                           static_cast<uint4*>(a.dY_pad), static_cast<uint4*>(a.x_pad));
            if (err != cudaSuccess) return err;
        }
        // A device that cannot co-schedule a CTA pair takes the single-SM kernel.
        err = padded ? launch_wgrad_pair(m_dYp64, m_H64, a.offsets, E, P, d, h, d, a.dW2, a.dW2,
                                         a.status, a.cap, s, 1, 0)
                     : launch_wgrad_pair(m_dY64, m_H64, a.offsets, E, P, d, h, d, a.dW2, a.dW2,
                                         a.status, a.cap, s);
        if (err != cudaSuccess) {
            cudaGetLastError();
            WArgs w{a.offsets, E, P, d, h, (d + kBM - 1) / kBM, (h + kN - 1) / kN, d, a.dW2,
                    a.dW2, a.status, a.cap};
            err = launch_wgrad<kModeW2>(false, grid_for(static_cast<long long>(E) * w.m_tiles * w.n_tiles, sms),
                                        s, m_dY64, m_H64, m_dW2, m_dW2, w);
        }
        if (err != cudaSuccess || (err = mark(6)) != cudaSuccess) return err;
        err = padded ? launch_wgrad_pair(m_duv64, m_xp64, a.offsets, E, P, 2 * h, d, h, a.dW1,
                                         a.dW3, a.status, a.cap, s, 0, 1)
                     : launch_wgrad_pair(m_duv64, m_x64, a.offsets, E, P, 2 * h, d, h, a.dW1,
                                         a.dW3, a.status, a.cap, s);
        if (err != cudaSuccess) {
            cudaGetLastError();
            WArgs w{a.offsets, E, P, 2 * h, d, (2 * h + kBM - 1) / kBM, (d + kN - 1) / kN, h,
                    a.dW1, a.dW3, a.status, a.cap};
            err = launch_wgrad<kModeW13>(false, grid_for(static_cast<long long>(E) * w.m_tiles * w.n_tiles, sms),
                                         s, m_duv64, m_x64, m_dW1, m_dW3, w);
        }
        if (err != cudaSuccess || (err = mark(7)) != cudaSuccess) return err;
    }
    // 7. dWg
    {
        const int nchunk = static_cast<int>(bwd_dwg_chunks(T));
        const dim3 grid((d / 2 + kPrepThreads - 1) / kPrepThreads, nchunk);
        err = launch_k(E <= 8 ? bwd_dwg_partial_kernel<8> : bwd_dwg_partial_kernel<kMaxExperts>,
                       grid, kPrepThreads, 0, s, static_cast<const __nv_bfloat16*>(a.x),
                       static_cast<const float*>(a.dlogits), T, d, E, a.dwg_part);
        if (err != cudaSuccess) return err;
        const long long n = static_cast<long long>(d) * E;
        err = launch_k(bwd_dwg_reduce_kernel, grid_for((n + kPrepThreads - 1) / kPrepThreads, 4 * sms),
                       kPrepThreads, 0, s, static_cast<const float*>(a.dwg_part), nchunk, d, E,
                       a.dWg);
        if (err != cudaSuccess) return err;
    }
    return mark(8);
}

}  // namespace moe
