// moe_api.cu -- the extern "C" entry points of libmoe (declared in include/moe.h).
//
// Each entry point validates its arguments on the host, then queues its kernels on
// the caller's stream.  Nothing here allocates, frees or synchronises (except the
// diagnostic moe_device_status and the opt-in MOE_DEBUG_SYNC=1 mode, which
// synchronises after every launch and reports device-side flags).
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "moe_internal.h"

namespace moe {

int device_sm_count() {
    static std::atomic<int> cache[64] = {};  // 0 = not yet read
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    const bool tracked = dev >= 0 && dev < 64;
    if (tracked) {
        const int n = cache[dev].load(std::memory_order_relaxed);
        if (n > 0) return n;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (tracked) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

namespace {
thread_local bool t_pdl_scope = false;
// Environment switches, read once (thread-safe static initialisation).
bool env_is(const char* name, char c) {
    const char* e = std::getenv(name);
    return e && e[0] == c;
}
bool pdl_allowed() {
    static const bool v = !env_is("MOE_NO_PDL", '1');
    return v;
}
// Small batches (the weight-streaming FFN's range): every kernel but the FFN is short,
// so overlapping launches pays off.
bool small_batch(int T) { return T <= kFusedMaxRows / 2; }
}  // namespace

bool pdl_enabled() { return t_pdl_scope && pdl_allowed(); }

bool pair_gemm_enabled() {
    static const bool v = !env_is("MOE_GEMM_PAIR", '0');
    return v;
}
PdlScope::PdlScope(bool on) : prev(t_pdl_scope) { t_pdl_scope = on; }
PdlScope::~PdlScope() { t_pdl_scope = prev; }

bool debug_sync_enabled() {
    static const bool v = env_is("MOE_DEBUG_SYNC", '1');
    return v;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// routed = false: the expert FFN alone, which also takes a single expert.
moe_status check_shape(int T, int d, int h, int E, int k, moe_dtype dt, bool need_h,
                       bool routed) {
    if (T < 0 || d <= 0 || (need_h && h <= 0) || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    if (dt != MOE_F32 && dt != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (k != 2 || E < (routed ? 2 : 1) || E > kMaxExperts) return MOE_ERR_UNSUPPORTED;
    if (d % 8 != 0 || (need_h && h % 8 != 0)) return MOE_ERR_UNSUPPORTED;
    // 32-bit row indices inside one grouped buffer (element offsets are 64-bit), and
    // 32-bit row coordinates in the flattened weight views [E*h, d] and [E*d, h].
    const long long P = 2LL * T;
    if (P * d >= (1LL << 40) || (need_h && P * h >= (1LL << 40)) || T > (1 << 29))
        return MOE_ERR_UNSUPPORTED;
    if (static_cast<long long>(E) * d >= (1LL << 31) ||
        (need_h && static_cast<long long>(E) * h >= (1LL << 31)))
        return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

bool ptrs_ok(std::initializer_list<const void*> ps) {
    for (const void* p : ps)
        if (p == nullptr || !aligned16(p)) return false;
    return true;
}

namespace {

// NVTX range around the host-side work of one stage (shows up in nsys / ncu timelines;
// free when no tool is attached).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

moe_status finish(cudaError_t err, cudaStream_t s, uint32_t* status) {
    if (err != cudaSuccess) return MOE_ERR_CUDA;
    if (debug_sync_enabled()) {
        if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
        if (status) {
            uint32_t flags = 0;
            if (cudaMemcpy(&flags, status, 4, cudaMemcpyDeviceToHost) != cudaSuccess)
                return MOE_ERR_CUDA;
            if (flags & MOE_DEV_FLAG_TIMEOUT) return MOE_ERR_TIMEOUT;
        }
    }
    return MOE_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

// Backward workspace regions (1 KiB aligned); the status word at offset 0.
struct BwdLayout {
    size_t status, dY, dw, dlogits, dH, DUV, dX, dwg_part, dY_pad, x_pad, a_pre, b_pre, total;
};

// Batches whose training forward can keep the pre-activations for the backward pass:
// every size (the fused small-batch FFN, the grouped GEMM1 and the CTA-pair GEMM1 all
// write them; the two-launch small-batch form, used only where the fused launch cannot
// be co-scheduled, does not, and the backward then recomputes).
bool keeps_pre_activations(int T) { return T > 0; }

BwdLayout bwd_layout(int T, int d, int h, int E) {
    BwdLayout B{};
    const size_t P = 2 * static_cast<size_t>(T);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at_ = o;
        o = align_up(o + bytes, 1024);
        return at_;
    };
    B.status = take(256);
    B.dY = take(P * d * 2);
    B.dw = take(P * 4);
    B.dlogits = take(static_cast<size_t>(T) * E * 4);
    B.dH = take(P * h * 4);
    B.DUV = take(P * 2 * h * 2);
    B.dX = take(P * d * 4);
    B.dwg_part = take(bwd_dwg_chunks(T) * d * E * 4);
    B.dY_pad = take(bwd_pad_rows(T, E) * d * 2);
    B.x_pad = take(bwd_pad_rows(T, E) * d * 2);
    // a = x W1^T and b = x W3^T of every grouped row, fp32, as moe_layer_forward_train
    // keeps them
    const bool keep = keeps_pre_activations(T);
    B.a_pre = take(keep ? P * h * 4 : 0);
    B.b_pre = take(keep ? P * h * 4 : 0);
    B.total = o;
    return B;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_bytes(int T, int d, int h, int E, int k, moe_dtype dt) {
    if (check_shape(T, d, h, E, k, dt, true) != MOE_OK) return 0;
    // Small batches keep split-K partial sums that larger ones do not, so the layout's
    // size drops where the grouped GEMMs take over; report the largest size of any batch
    // up to T, so that one workspace serves every smaller batch too.
    const int t_small = T < kFusedMaxRows / 2 ? T : kFusedMaxRows / 2;
    const size_t small = ws_layout(t_small, d, h, E, k, dt).total;
    const size_t own = ws_layout(T, d, h, E, k, dt).total;
    return own > small ? own : small;
}

const char* moe_status_string(moe_status st) {
    switch (st) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument (null/misaligned pointer or bad size)";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape (need k == 2, 2 <= E <= 32, d and h multiples of 8)";
        case MOE_ERR_WORKSPACE: return "workspace too small";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_TIMEOUT: return "device pipeline wait timed out";
    }
    return "unknown status";
}

moe_status moe_route(const void* x, const void* Wg, int T, int d, int E, int k, moe_dtype dt,
                     int32_t* topk_idx, float* topk_w, cudaStream_t stream) {
    moe_status st = check_shape(T, d, 8, E, k, dt, false);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    if (!ptrs_ok({x, Wg, topk_idx, topk_w})) return MOE_ERR_INVALID_ARG;
    PdlScope pdl(small_batch(T));
    return finish(launch_route(x, Wg, T, d, E, dt, topk_idx, topk_w, stream), stream, nullptr);
}

moe_status moe_permute(const int32_t* topk_idx, const void* x, int T, int d, int E, int k,
                       moe_dtype dt, int32_t* offsets, int32_t* perm_token, int32_t* inv_perm,
                       void* x_perm, void* ws, size_t ws_bytes, cudaStream_t stream) {
    moe_status st = check_shape(T, d, 8, E, k, dt, false);
    if (st != MOE_OK) return st;
    if (!ptrs_ok({offsets, ws})) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, d, 8, E, k, dt);
    if (ws_bytes < L.permute_need) return MOE_ERR_WORKSPACE;
    if (T == 0) {
        // Empty batch: every group is empty.
        if (cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), stream) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (!ptrs_ok({topk_idx, x, perm_token, inv_perm, x_perm})) return MOE_ERR_INVALID_ARG;
    uint32_t* status = at<uint32_t>(ws, L.status);
    PdlScope pdl(small_batch(T));
    return finish(launch_permute(topk_idx, x, T, d, E, dt, offsets, perm_token, inv_perm, x_perm,
                                 at<int32_t>(ws, L.blk_counts), at<int32_t>(ws, L.blk_base),
                                 status, stream),
                  stream, status);
}

moe_status moe_expert_ffn(const void* x_perm, const int32_t* offsets, const void* W1,
                          const void* W3, const void* W2, int rows, int d, int h, int E,
                          moe_dtype dt, float* y_perm, void* ws, size_t ws_bytes,
                          cudaStream_t stream) {
    if (rows < 0 || rows % 2 != 0) return MOE_ERR_INVALID_ARG;
    const int T = rows / 2;
    moe_status st = check_shape(T, d, h, E, 2, dt, true, /*routed=*/false);
    if (st != MOE_OK) return st;
    if (rows == 0) return MOE_OK;
    if (!ptrs_ok({x_perm, offsets, W1, W3, W2, y_perm, ws})) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, d, h, E, 2, dt);
    if (ws_bytes < L.ffn_need) return MOE_ERR_WORKSPACE;
    uint32_t* status = at<uint32_t>(ws, L.status);
    PdlScope pdl(small_batch(T));
    cudaError_t err;
    if (dt == MOE_BF16) {
        err = launch_ffn_bf16(x_perm, offsets, W1, W3, W2, rows, d, h, E, at<void>(ws, L.H), y_perm,
                              at<float>(ws, L.Ypart), kDecodeSplitK, /*reduce=*/true, nullptr,
                              status, stream, nullptr, at<uint32_t>(ws, L.sync));
        if (err == cudaErrorInvalidValue) return MOE_ERR_INVALID_ARG;  // tensor map refused
    } else {
        err = launch_ffn_f32(static_cast<const float*>(x_perm), offsets,
                             static_cast<const float*>(W1), static_cast<const float*>(W3),
                             static_cast<const float*>(W2), rows, d, h, E, at<float>(ws, L.H),
                             y_perm, stream);
    }
    return finish(err, stream, status);
}

moe_status moe_combine(const float* y_perm, const int32_t* inv_perm, const float* topk_w, int T,
                       int d, int k, moe_dtype dt, void* y, cudaStream_t stream) {
    moe_status st = check_shape(T, d, 8, 2, k, dt, false);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    if (!ptrs_ok({y_perm, inv_perm, topk_w, y})) return MOE_ERR_INVALID_ARG;
    PdlScope pdl(small_batch(T));
    return finish(launch_combine(y_perm, 1, 0, inv_perm, topk_w, T, d, dt, y, stream), stream,
                  nullptr);
}

}  // extern "C"

namespace moe {
namespace {

// The layer, with optional events recorded between its stages (profiling).  Above 512
// tokens (the four-launch grouping) the fp64 tensor-core router also counts the pairs
// of every chunk per expert, so the grouping skips its count pass.
moe_status layer_forward_impl(const void* x, const void* Wg, const void* W1, const void* W3,
                              const void* W2, int T, int d, int h, int E, int k, moe_dtype dt,
                              void* y, void* ws, size_t ws_bytes, cudaEvent_t* ev, int n_ev,
                              cudaStream_t stream, int cap, float* a_save = nullptr,
                              float* b_save = nullptr) {
    moe_status st = check_shape(T, d, h, E, k, dt, true);
    if (st != MOE_OK) return st;
    if (n_ev < 0 || (n_ev > 0 && ev == nullptr)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!ptrs_ok({x, Wg, W1, W3, W2, y, ws})) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, d, h, E, k, dt);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    uint32_t* status = at<uint32_t>(ws, L.status);
    int32_t* idx = at<int32_t>(ws, L.topk_idx);
    float* w = at<float>(ws, L.topk_w);
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* perm_token = at<int32_t>(ws, L.perm_token);
    int32_t* inv_perm = at<int32_t>(ws, L.inv_perm);
    void* x_perm = at<void>(ws, L.x_perm);
    float* Y = at<float>(ws, L.Y);
    const int P = 2 * T;
    PdlScope pdl(small_batch(T));
    auto mark = [&](int i) -> bool {  // null handles are skipped
        return i >= n_ev || ev[i] == nullptr || cudaEventRecord(ev[i], stream) == cudaSuccess;
    };

    const bool counts_in_router = T > kPermSmallTokens && dmma_route_applies(T, d, E, dt);
    NvtxRange layer_range("moe_layer_forward");
    if (!mark(0)) return MOE_ERR_CUDA;
    cudaError_t err;
    {
        NvtxRange r("route");
        err = launch_route(x, Wg, T, d, E, dt, idx, w, stream,
                           counts_in_router ? at<int32_t>(ws, L.blk_counts) : nullptr);
    }
    if ((st = finish(err, stream, status)) != MOE_OK) return st;
    {
        NvtxRange r("permute");
        err = launch_permute(idx, x, T, d, E, dt, offsets, perm_token, inv_perm, x_perm,
                             at<int32_t>(ws, L.blk_counts), at<int32_t>(ws, L.blk_base), status,
                             stream, counts_in_router);
    }
    if ((st = finish(err, stream, status)) != MOE_OK) return st;
    if (!mark(1)) return MOE_ERR_CUDA;
    FfnOut fo{Y, 1};
    {
        NvtxRange r("expert_ffn");
        if (dt == MOE_BF16) {
            err = launch_ffn_bf16(x_perm, offsets, W1, W3, W2, P, d, h, E, at<void>(ws, L.H), Y,
                                  at<float>(ws, L.Ypart), kDecodeSplitK, /*reduce=*/false, &fo,
                                  status, stream, n_ev > 2 ? ev[2] : nullptr,
                                  at<uint32_t>(ws, L.sync), cap, a_save, b_save);
            if (err == cudaErrorInvalidValue) return MOE_ERR_INVALID_ARG;
        } else {
            err = launch_ffn_f32(static_cast<const float*>(x_perm), offsets,
                                 static_cast<const float*>(W1), static_cast<const float*>(W3),
                                 static_cast<const float*>(W2), P, d, h, E, at<float>(ws, L.H),
                                 Y, stream, n_ev > 2 ? ev[2] : nullptr, cap);
        }
    }
    if ((st = finish(err, stream, status)) != MOE_OK) return st;
    if (!mark(3)) return MOE_ERR_CUDA;
    {
        NvtxRange r("combine");
        err = launch_combine(fo.Y, fo.nsplit, static_cast<size_t>(P) * d, inv_perm, w, T, d, dt,
                             y, stream, idx, offsets, E, cap, at<uint8_t>(ws, L.y_layout),
                             fo.saved_ab ? kLayoutSavedAB : 0);
    }
    if ((st = finish(err, stream, status)) != MOE_OK) return st;
    if (!mark(4)) return MOE_ERR_CUDA;
    return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" {

moe_status moe_layer_forward(const void* x, const void* Wg, const void* W1, const void* W3,
                             const void* W2, int T, int d, int h, int E, int k, moe_dtype dt,
                             void* y, void* ws, size_t ws_bytes, cudaStream_t stream) {
    return layer_forward_impl(x, Wg, W1, W3, W2, T, d, h, E, k, dt, y, ws, ws_bytes, nullptr, 0,
                              stream, INT_MAX);
}

moe_status moe_layer_forward_capacity(const void* x, const void* Wg, const void* W1,
                                      const void* W3, const void* W2, int T, int d, int h, int E,
                                      int k, moe_dtype dt, int capacity, void* y, void* ws,
                                      size_t ws_bytes, cudaStream_t stream) {
    return layer_forward_impl(x, Wg, W1, W3, W2, T, d, h, E, k, dt, y, ws, ws_bytes, nullptr, 0,
                              stream, capacity < 0 ? INT_MAX : capacity);
}

moe_status moe_layer_forward_events(const void* x, const void* Wg, const void* W1,
                                    const void* W3, const void* W2, int T, int d, int h, int E,
                                    int k, moe_dtype dt, void* y, void* ws, size_t ws_bytes,
                                    cudaEvent_t* events, int n_events, cudaStream_t stream) {
    return layer_forward_impl(x, Wg, W1, W3, W2, T, d, h, E, k, dt, y, ws, ws_bytes, events,
                              n_events, stream, INT_MAX);
}

moe_status moe_layer_forward_train(const void* x, const void* Wg, const void* W1, const void* W3,
                                   const void* W2, int T, int d, int h, int E, int k,
                                   moe_dtype dt, void* y, void* ws, size_t ws_bytes,
                                   void* bwd_ws, size_t bwd_ws_bytes, cudaStream_t stream) {
    moe_status st = check_shape(T, d, h, E, k, dt, true);
    if (st != MOE_OK) return st;
    if (dt != MOE_BF16 || h % 64 != 0) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;  // empty batch: nothing to queue, as moe_layer_forward
    if (!ptrs_ok({bwd_ws})) return MOE_ERR_INVALID_ARG;
    const BwdLayout B = bwd_layout(T, d, h, E);
    if (bwd_ws_bytes < B.total) return MOE_ERR_WORKSPACE;
    const bool keep = keeps_pre_activations(T);
    return layer_forward_impl(x, Wg, W1, W3, W2, T, d, h, E, k, dt, y, ws, ws_bytes, nullptr, 0,
                              stream, INT_MAX, keep ? at<float>(bwd_ws, B.a_pre) : nullptr,
                              keep ? at<float>(bwd_ws, B.b_pre) : nullptr);
}

size_t moe_backward_workspace_bytes(int T, int d, int h, int E, int k, moe_dtype dt) {
    if (check_shape(T, d, h, E, k, dt, true) != MOE_OK) return 0;
    if (dt != MOE_BF16 || h % 64 != 0) return 0;
    return bwd_layout(T, d, h, E).total;
}

}  // extern "C"

namespace moe {
namespace {

moe_status layer_backward_impl(const void* x, const void* Wg, const void* W1, const void* W3,
                               const void* W2, const void* dy, int T, int d, int h, int E, int k,
                               moe_dtype dt, int capacity, void* dx, float* dWg, float* dW1,
                               float* dW3, float* dW2, const void* fwd_ws, size_t fwd_ws_bytes,
                               void* bwd_ws, size_t bwd_ws_bytes, cudaEvent_t* ev, int n_ev,
                               cudaStream_t stream) {
    moe_status st = check_shape(T, d, h, E, k, dt, true);
    if (st != MOE_OK) return st;
    if (n_ev < 0 || (n_ev > 0 && ev == nullptr)) return MOE_ERR_INVALID_ARG;
    if (dt != MOE_BF16 || h % 64 != 0) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!ptrs_ok({x, Wg, W1, W3, W2, dy, dx, dWg, dW1, dW3, dW2, fwd_ws, bwd_ws}))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, d, h, E, k, dt);
    const BwdLayout B = bwd_layout(T, d, h, E);
    if (fwd_ws_bytes < L.total || bwd_ws_bytes < B.total) return MOE_ERR_WORKSPACE;
    const int P = 2 * T;
    void* fws = const_cast<void*>(fwd_ws);
    BwdArgs a{};
    a.T = T;
    a.d = d;
    a.h = h;
    a.E = E;
    a.cap = capacity < 0 ? INT_MAX : capacity;
    a.dy = dy;
    a.idx = at<int32_t>(fws, L.topk_idx);
    a.w = at<float>(fws, L.topk_w);
    a.inv = at<int32_t>(fws, L.inv_perm);
    a.offsets = at<int32_t>(fws, L.offsets);
    // the forward's combine recorded whether Y or the split-K partials hold its outputs
    a.Y = at<float>(fws, L.Y);
    a.Ypart = at<float>(fws, L.Ypart);
    a.y_layout = at<uint8_t>(fws, L.y_layout);
    a.split_stride = static_cast<size_t>(P) * d;
    a.x_perm = at<void>(fws, L.x_perm);
    a.H = at<void>(fws, L.H);
    a.x = x;
    a.Wg = Wg;
    a.W1 = W1;
    a.W3 = W3;
    a.W2 = W2;
    a.dx = dx;
    a.dWg = dWg;
    a.dW1 = dW1;
    a.dW3 = dW3;
    a.dW2 = dW2;
    a.dY = at<void>(bwd_ws, B.dY);
    a.dw = at<float>(bwd_ws, B.dw);
    a.dlogits = at<float>(bwd_ws, B.dlogits);
    a.dH = at<float>(bwd_ws, B.dH);
    a.DUV = at<void>(bwd_ws, B.DUV);
    a.dX = at<float>(bwd_ws, B.dX);
    a.dwg_part = at<float>(bwd_ws, B.dwg_part);
    a.dY_pad = at<void>(bwd_ws, B.dY_pad);
    a.x_pad = at<void>(bwd_ws, B.x_pad);
    // where moe_layer_forward_train may have kept a and b (the forward's layout byte
    // says whether it did); a capacity layer always recomputes them
    const bool keep = keeps_pre_activations(T) && a.cap == INT_MAX;
    a.a_pre = keep ? at<float>(bwd_ws, B.a_pre) : nullptr;
    a.b_pre = keep ? at<float>(bwd_ws, B.b_pre) : nullptr;
    a.status = at<uint32_t>(bwd_ws, B.status);
    a.ev = ev;
    a.n_ev = n_ev;
    PdlScope pdl(false);  // the backward kernels do not wait on griddepcontrol
    NvtxRange range("moe_layer_backward");
    cudaError_t err = launch_layer_backward(a, stream);
    if (err == cudaErrorInvalidValue) return MOE_ERR_INVALID_ARG;  // tensor map refused
    return finish(err, stream, a.status);
}

}  // namespace
}  // namespace moe

extern "C" {

moe_status moe_layer_backward(const void* x, const void* Wg, const void* W1, const void* W3,
                              const void* W2, const void* dy, int T, int d, int h, int E, int k,
                              moe_dtype dt, int capacity, void* dx, float* dWg, float* dW1,
                              float* dW3, float* dW2, const void* fwd_ws, size_t fwd_ws_bytes,
                              void* bwd_ws, size_t bwd_ws_bytes, cudaStream_t stream) {
    return layer_backward_impl(x, Wg, W1, W3, W2, dy, T, d, h, E, k, dt, capacity, dx, dWg, dW1,
                               dW3, dW2, fwd_ws, fwd_ws_bytes, bwd_ws, bwd_ws_bytes, nullptr, 0,
                               stream);
}

moe_status moe_layer_backward_events(const void* x, const void* Wg, const void* W1,
                                     const void* W3, const void* W2, const void* dy, int T, int d,
                                     int h, int E, int k, moe_dtype dt, int capacity, void* dx,
                                     float* dWg, float* dW1, float* dW3, float* dW2,
                                     const void* fwd_ws, size_t fwd_ws_bytes, void* bwd_ws,
                                     size_t bwd_ws_bytes, cudaEvent_t* events, int n_events,
                                     cudaStream_t stream) {
    return layer_backward_impl(x, Wg, W1, W3, W2, dy, T, d, h, E, k, dt, capacity, dx, dWg, dW1,
                               dW3, dW2, fwd_ws, fwd_ws_bytes, bwd_ws, bwd_ws_bytes, events,
                               n_events, stream);
}

moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes, double limit_seconds,
                                     uint32_t* outcome, cudaStream_t stream) {
    if (!ws || !outcome || ws_bytes < 2048 || !(limit_seconds > 0.0) || limit_seconds > 10.0)
        return MOE_ERR_INVALID_ARG;
    // status word at offset 0; scratch words at offset 1024 (inside the first region
    // of every workspace layout, which is at least 2 KiB)
    uint32_t* status = static_cast<uint32_t*>(ws);
    uint32_t* scratch = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + 1024);
    const auto ns = static_cast<unsigned long long>(limit_seconds * 1e9);
    if (launch_selftest_wait(status, scratch, ns, stream) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
    uint32_t got[2] = {0, 0};
    if (cudaMemcpy(got, scratch + 1, sizeof(got), cudaMemcpyDeviceToHost) != cudaSuccess)
        return MOE_ERR_CUDA;
    outcome[0] = got[0];
    outcome[1] = got[1];
    // the scratch words must be zero again for the layer's own use of this region
    if (cudaMemset(scratch, 0, 3 * sizeof(uint32_t)) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status moe_device_status(void* ws, size_t ws_bytes, uint32_t* flags, cudaStream_t stream) {
    if (!ws || !flags || ws_bytes < 256) return MOE_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, ws, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemset(ws, 0, 4) != cudaSuccess) return MOE_ERR_CUDA;
    *flags = v;
    return (v & MOE_DEV_FLAG_TIMEOUT) ? MOE_ERR_TIMEOUT : MOE_OK;
}

}  // extern "C"
