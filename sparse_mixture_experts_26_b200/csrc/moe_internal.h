// moe_internal.h -- host-side pieces shared by the libmoe translation units:
// the workspace layout and the launchers of each kernel family.
#pragma once

#include <initializer_list>
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cstddef>
#include <cstdint>
#include <utility>

#include "../../include/moe.h"

namespace moe {

constexpr int kMaxExperts = 32;

// One-time host setup per device, such as a kernel's opt-in to more than 48 KiB of
// dynamic shared memory.  Thread-safe: threads that race may each run `fn` (it must be
// idempotent); a call skips it only once some call of it has succeeded on that device.
class PerDeviceOnce {
  public:
    template <typename Fn>
    cudaError_t operator()(Fn&& fn) {
        int dev = 0;
        cudaError_t err = cudaGetDevice(&dev);
        if (err != cudaSuccess) return err;
        const bool tracked = dev >= 0 && dev < kDevices;
        if (tracked && done_[dev].load(std::memory_order_acquire)) return cudaSuccess;
        err = fn();
        if (err == cudaSuccess && tracked) done_[dev].store(1, std::memory_order_release);
        return err;
    }

  private:
    static constexpr int kDevices = 64;
    std::atomic<int> done_[kDevices] = {};
};

// Opt `kern` into `bytes` of dynamic shared memory on the current device, once.
template <typename Kern>
cudaError_t opt_in_smem(PerDeviceOnce& once, Kern kern, int bytes) {
    return once([&] {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    });
}
// Tokens handled by one block of the permutation count / rank kernels.
constexpr int kPermChunk = 256;

// Grouped rows at or below which the weight-streaming (swap-AB) expert FFN is used
// (two launches, or one fused cooperative launch), the larger limit of the fused launch
// alone (token tiles of up to 128 rows), and how many K ranges its down projection is
// split into at most.
constexpr int kDecodeMaxRows = 128;
constexpr int kFusedMaxRows = 256;
constexpr int kDecodeSplitK = 8;

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline size_t dtype_bytes(moe_dtype dt) { return dt == MOE_BF16 ? 2 : 4; }

// Byte offsets of every workspace region (1 KiB aligned).  The status word sits at
// offset 0 so that every entry point sharing a workspace reports into one place.
struct WsLayout {
    size_t status, y_layout, sync, topk_idx, topk_w, offsets, blk_counts, blk_base, perm_token,
        inv_perm, x_perm, H, Ypart, Y, total;
    // Bytes needed by moe_permute (status + count/base scratch) and by moe_expert_ffn
    // (status + H); moe_layer_forward needs `total`.
    size_t permute_need, ffn_need;
};

inline int perm_blocks(int T) { return (T + kPermChunk - 1) / kPermChunk; }

inline WsLayout ws_layout(int T, int d, int h, int E, int k, moe_dtype dt) {
    WsLayout L{};
    const size_t P = static_cast<size_t>(T) * k;
    const size_t nb = static_cast<size_t>(perm_blocks(T));
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o = align_up(o + bytes, 1024);
        return at;
    };
    L.status = take(256);
    // one byte in the status region: how many split-K partials (in Ypart) hold the
    // expert outputs of the last layer call, or 1 for the single array Y (written by
    // the combine kernel, read by the backward pass)
    L.y_layout = L.status + 64;
    // dependency counters of the fused small-batch FFN (zero between calls)
    L.sync = take(2 * kMaxExperts * kDecodeSplitK * 4);
    L.blk_counts = take(nb * E * 4);
    L.blk_base = take(nb * E * 4);
    L.permute_need = o;
    L.H = take(P * h * (dt == MOE_BF16 ? 2 : 4));
    // fp32 partial sums of the split-K down projection (small batches, bf16 only)
    L.Ypart = take(dt == MOE_BF16 && P <= kFusedMaxRows ? kDecodeSplitK * P * d * 4 : 0);
    L.ffn_need = o;
    L.topk_idx = take(P * 4);
    L.topk_w = take(P * 4);
    L.offsets = take((E + 1) * 4);
    L.perm_token = take(P * 4);
    L.inv_perm = take(P * 4);
    L.x_perm = take(P * d * dtype_bytes(dt));
    L.Y = take(P * d * 4);
    L.total = o;
    return L;
}

int device_sm_count();
bool debug_sync_enabled();

// Argument checks shared by every entry point.  routed = false: the expert FFN alone,
// which also takes a single expert.
moe_status check_shape(int T, int d, int h, int E, int k, moe_dtype dt, bool need_h,
                       bool routed = true);
bool aligned16(const void* p);
bool ptrs_ok(std::initializer_list<const void*> ps);
// Programmatic dependent launch: used for the launches made inside a PdlScope(true)
// (the entry points open one for small batches, where launch gaps matter and every
// kernel is short), never when MOE_NO_PDL=1.  Measured: on T=16 it saves ~2% of the
// layer; on T=4096 early-resident dependents cost ~3%, so large batches do not use it.
bool pdl_enabled();
struct PdlScope {
    explicit PdlScope(bool on);
    ~PdlScope();
    bool prev;
};

// Launch `kern` on `s` with programmatic stream serialisation: the kernel may be
// scheduled while the previous kernel on the stream is finishing, and every libmoe
// kernel calls griddepcontrol.wait before it reads anything a previous kernel wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    cudaError_t err = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    return err != cudaSuccess ? err : cudaGetLastError();
}

// ---- launchers (each returns cudaGetLastError() of its launch) ----
// With `blk_counts` (zero on entry) the router also counts the pairs of every
// kPermChunk-token chunk per expert (only where dmma_route_applies(); otherwise
// cudaErrorInvalidValue).
cudaError_t launch_route(const void* x, const void* Wg, int T, int d, int E, moe_dtype dt,
                         int32_t* idx, float* w, cudaStream_t s, int32_t* blk_counts = nullptr);
bool dmma_route_applies(int T, int d, int E, moe_dtype dt);
// Batches of up to kPermSmallTokens tokens are grouped in one launch; larger ones in
// four (count, scan, rank, gather).  counts_ready: blk_counts already hold the
// router's per-chunk counts, so the count pass is skipped (larger batches only).  The
// scan leaves blk_counts at zero.
constexpr int kPermSmallTokens = 512;
cudaError_t launch_permute(const int32_t* idx, const void* x, int T, int d, int E, moe_dtype dt,
                           int32_t* offsets, int32_t* perm_token, int32_t* inv_perm,
                           void* x_perm, int32_t* blk_counts, int32_t* blk_base,
                           uint32_t* status, cudaStream_t s, bool counts_ready = false);
// `cap` (all FFN launchers): rows kept per expert group -- the first `cap` rows of
// each group are computed, the rest are neither computed nor written.
cudaError_t launch_ffn_f32(const float* x_perm, const int32_t* offsets, const float* W1,
                           const float* W3, const float* W2, int rows, int d, int h, int E,
                           float* H, float* Y, cudaStream_t s, cudaEvent_t between = nullptr,
                           int cap = INT_MAX);
// bf16 expert FFN.  The result is the sum of `out->nsplit` fp32 arrays [rows, d]
// starting at `out->Y`, `rows * d` floats apart: Y itself (nsplit = 1), or -- when
// the small-batch kernels run and `partials` has room for `partial_cap` of them --
// the split-K partial sums in `partials`.  With reduce = true the partials are
// summed (in order) into Y before returning, so Y always holds the result.
// `between` (optional) is recorded on `s` after the first FFN kernel (GEMM1 +
// SwiGLU) and before the second.  Returns cudaErrorInvalidValue if a tensor map
// cannot be encoded.
struct FfnOut {
    const float* Y;
    int nsplit;
    bool saved_ab = false;  // the pre-activations a and b were written (a_save / b_save)
};
cudaError_t launch_ffn_bf16(const void* x_perm, const int32_t* offsets, const void* W1,
                            const void* W3, const void* W2, int rows, int d, int h, int E,
                            void* H, float* Y, float* partials, int partial_cap, bool reduce,
                            FfnOut* out, uint32_t* status, cudaStream_t s,
                            cudaEvent_t between = nullptr, uint32_t* counters = nullptr,
                            int cap = INT_MAX, float* a_save = nullptr, float* b_save = nullptr);
// With `counters` (2 * kMaxExperts * kDecodeSplitK zeroed words, left zeroed) small
// batches run the fused single-launch FFN; `between` is then recorded after it.
// Large-batch expert FFN on CTA pairs (tcgen05 cta_group::2).
cudaError_t launch_ffn_bf16_pair(const void* x_perm, const int32_t* offsets, const void* W1,
                                 const void* W3, const void* W2, int rows, int d, int h, int E,
                                 void* H, float* Y, uint32_t* status, cudaStream_t s,
                                 cudaEvent_t between, int cap, float* a_out = nullptr,
                                 float* b_out = nullptr);
// Grouped rows from which the CTA-pair kernels are used (MOE_GEMM_PAIR=0 disables them):
// the forward's expert FFN, and the backward's row-grouped GEMMs.
constexpr int kPairMinRows = 1024;
constexpr int kBwdPairMinRows = 1024;
bool pair_gemm_enabled();
// Small-batch expert FFN as one cooperative launch (gate/up and split-K down units
// with per-(expert, K range) dependency counters, 2*E*ksplit zeroed words).
cudaError_t launch_ffn_bf16_decode_fused(const void* x_perm, const int32_t* offsets,
                                         const void* W1, const void* W3, const void* W2, int rows,
                                         int d, int h, int E, void* H, float* Ypart, int ksplit,
                                         uint32_t* counters, uint32_t* status, cudaStream_t s,
                                         int cap, float* a_out = nullptr, float* b_out = nullptr);
// Small-batch expert FFN; the down projection writes `ksplit` partial arrays.
cudaError_t launch_ffn_bf16_decode(const void* x_perm, const int32_t* offsets, const void* W1,
                                   const void* W3, const void* W2, int rows, int d, int h, int E,
                                   void* H, float* Yout, int ksplit, uint32_t* status,
                                   cudaStream_t s, cudaEvent_t between, int cap);
// y[t] = w0 * S(inv[t,0]) + w1 * S(inv[t,1]) with S(r) the in-order sum of the
// nsplit arrays Y + i * split_stride at row r.  With cap < INT_MAX (and idx,
// offsets, E given) a pair whose row lies cap or more rows into its expert's group
// was dropped and contributes nothing.
// With `layout_out`, one thread also stores nsplit there (the layer records where
// its expert outputs are, for the backward pass).
cudaError_t launch_combine(const float* Y, int nsplit, size_t split_stride,
                           const int32_t* inv_perm, const float* w, int T, int d, moe_dtype dt,
                           void* y, cudaStream_t s, const int32_t* idx = nullptr,
                           const int32_t* offsets = nullptr, int E = 0, int cap = INT_MAX,
                           uint8_t* layout_out = nullptr, uint8_t layout_flags = 0);
// The layout byte the combine records for the backward pass: the number of split-K
// partials holding the expert outputs (1: the single array Y) in bits 0..6, and bit 7
// set when the forward kept the pre-activations a and b (moe_layer_forward_train).
constexpr uint8_t kLayoutSavedAB = 0x80;
constexpr uint8_t kLayoutSplitMask = 0x7F;
// K ranges of the small-batch down projection: the largest split (at most
// partial_cap and kDecodeSplitK) that leaves no K range of 64-wide blocks empty.
inline int decode_ksplit(int h, int partial_cap) {
    const int num_kb = (h + 63) / 64;
    int ksplit = partial_cap < kDecodeSplitK ? partial_cap : kDecodeSplitK;
    while (ksplit > 1 && ((num_kb + ksplit - 1) / ksplit) * (ksplit - 1) >= num_kb) --ksplit;
    return ksplit < 1 ? 1 : ksplit;
}
// Everything the backward pass reads and writes (bf16 layer; see backward_sm100.cu).
struct BwdArgs {
    int T, d, h, E, cap;
    // upstream gradient and the forward's saved state
    const void* dy;            // bf16 [T, d]
    const int32_t* idx;        // [T, 2]
    const float* w;            // [T, 2]
    const int32_t* inv;        // [T, 2]
    const int32_t* offsets;    // [E + 1]
    const float* Y;            // expert outputs as one array [2T, d] ...
    const float* Ypart;        // ... or as split-K partials, split_stride floats apart
    const uint8_t* y_layout;   // device byte: number of partials (or 1 for Y), bit 7: a, b kept
    size_t split_stride;
    const void* x_perm;        // bf16 [2T, d]
    const void* H;             // bf16 [2T, h]
    const void *x, *Wg, *W1, *W3, *W2;
    // outputs
    void* dx;                  // bf16 [T, d]
    float *dWg, *dW1, *dW3, *dW2;
    // scratch (backward workspace)
    void* dY;                  // bf16 [2T, d]
    float* dw;                 // [T, 2]
    float* dlogits;            // [T, E]
    float* dH;                 // [2T, h]
    void* DUV;                 // bf16 [2T, 2h]: du then dv
    float* dX;                 // [2T, d]
    float* dwg_part;           // [bwd_dwg_chunks(T), d, E]
    // bf16 [bwd_pad_rows(T, E), d]: dY and x_perm with each expert's rows padded by
    // zero rows to a multiple of 64 (the weight-gradient GEMMs on CTA pairs)
    void* dY_pad;
    void* x_pad;
    // fp32 [2T, h] each: the pre-activations a and b moe_layer_forward_train kept (the
    // CTA-pair range); nullptr below that range
    const float* a_pre;
    const float* b_pre;
    uint32_t* status;
    // optional events recorded before the first launch and after each stage:
    // prep, dH, du/dv, dX, dx, dW2, dW1/dW3, dWg (null handles skipped)
    cudaEvent_t* ev;
    int n_ev;
};
size_t bwd_dwg_chunks(int T);
// Rows of a grouped [2T, d] array once every expert's rows are padded to a multiple of 64.
inline size_t bwd_pad_rows(int T, int E) { return 2 * static_cast<size_t>(T) + 64 * E; }
cudaError_t launch_layer_backward(const BwdArgs& a, cudaStream_t s);
// Bounded-wait self-test (see moe_selftest_wait_timeout).
cudaError_t launch_selftest_wait(uint32_t* status, uint32_t* scratch, unsigned long long limit_ns,
                                 cudaStream_t s);
// Y[i] = sum over j < nsplit of parts[j * n + i] (in order), for i < n.
cudaError_t launch_sum_splits(const float* parts, int nsplit, size_t n, float* Y,
                              cudaStream_t s);

}  // namespace moe
