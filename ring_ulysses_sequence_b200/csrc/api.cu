// C ABI: argument validation, status codes, and dispatch to the kernels.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "internal.h"

namespace rm {

// Device status word: bit 0 = a bounded wait ran out. One copy per device.
__device__ unsigned g_status_word;
// Work-item counters of the persistent kernels (one slot per launch in flight).
__device__ int g_work_counters[kWorkSlots];
static std::atomic<uint32_t> g_work_seq{0};

cudaError_t next_work_counter(const LaunchCtx& ctx, int n_items, WorkCounter* counter) {
    const uint32_t seq = g_work_seq.fetch_add(1);
    const int gen = static_cast<int>((seq / kWorkSlots) % 255u) + 1;  // 1..255, in every byte
    counter->ptr = ctx.work_counters + (seq % kWorkSlots);
    counter->base = gen * 0x01010101;
    counter->n_items = n_items;
    return cudaMemsetAsync(counter->ptr, gen, sizeof(int), ctx.stream);
}

static thread_local int t_last_cuda_error = 0;
static std::atomic<uint64_t> g_watchdog_ns{2000000000ull};
static std::atomic<int> g_bwd_deterministic{1};

static rm_status cuda_fail(cudaError_t e) {
    t_last_cuda_error = static_cast<int>(e);
    return RM_ERR_CUDA;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Status-word address and SM count of the current device, looked up once per
// device with that device current.
static rm_status get_ctx(cudaStream_t stream, LaunchCtx* ctx) {
    static std::mutex mu;
    static unsigned* word_addr[128] = {};
    static int* counters_addr[128] = {};
    static int sms[128] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= 128) return RM_ERR_UNSUPPORTED;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!word_addr[dev]) {
            void* p = nullptr;
            e = cudaGetSymbolAddress(&p, g_status_word);
            if (e != cudaSuccess) return cuda_fail(e);
            void* pc = nullptr;
            e = cudaGetSymbolAddress(&pc, g_work_counters);
            if (e != cudaSuccess) return cuda_fail(e);
            counters_addr[dev] = static_cast<int*>(pc);
            int n = 0;
            e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return cuda_fail(e);
            sms[dev] = n;
            word_addr[dev] = static_cast<unsigned*>(p);
        }
        ctx->status_word = word_addr[dev];
        ctx->work_counters = counters_addr[dev];
        ctx->num_sms = sms[dev];
    }
    ctx->watchdog_ns = g_watchdog_ns.load();
    ctx->stream = stream;
    return RM_OK;
}

// Scratch of rm_ring_attn_bwd_noalloc: the Delta rows (B * H * S fp32 values)
// of the backward, at most kNoAllocMaxRows of them (8 MiB). It is a static
// device array, so every GPU that loads this library holds it until the
// process exits; all calls on a device share it.
constexpr size_t kNoAllocMaxRows = static_cast<size_t>(1) << 21;
static __device__ __align__(256) float g_noalloc_delta[kNoAllocMaxRows];

// Device address of g_noalloc_delta on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device, with that device current, and cached.
static rm_status noalloc_scratch(float** out) {
    static std::mutex mu;
    static float* addr[128] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= 128) return RM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_delta);
        if (e != cudaSuccess) return cuda_fail(e);
        addr[dev] = static_cast<float*>(p);
    }
    *out = addr[dev];
    return RM_OK;
}

static bool valid_order(rm_order o) { return o == RM_ORDER_CONTIGUOUS || o == RM_ORDER_ZIGZAG; }

// Shared shape rules of the forward and backward.
static rm_status check_attn(const void* q, const void* k, const void* v, int B, int H, int Hkv,
                            int S, int D, int P, rm_order order, rm_dtype dtype, float scale,
                            int tile_q) {
    if (B < 0 || H <= 0 || Hkv <= 0 || S < 0 || D <= 0 || P <= 0) return RM_ERR_INVALID_ARG;
    const bool empty = B == 0 || S == 0;  // pointers of empty tensors may be null
    if (!empty && (!q || !k || !v)) return RM_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return RM_ERR_INVALID_ARG;
    if (!valid_order(order)) return RM_ERR_INVALID_ARG;
    if (dtype != RM_DTYPE_BF16 && dtype != RM_DTYPE_FP32) return RM_ERR_INVALID_ARG;
    if (!(scale > 0.0f) || !std::isfinite(scale)) return RM_ERR_INVALID_ARG;
    if (H % Hkv != 0) return RM_ERR_INVALID_ARG;
    if (order == RM_ORDER_ZIGZAG ? (S % (2 * P) != 0) : (S % P != 0)) return RM_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return RM_ERR_UNSUPPORTED;
    // Tiles never straddle a chunk: the chunk must be a multiple of the tile,
    // and (tensor-core path) a rank's block a multiple of two tiles.
    const int64_t chunk = order == RM_ORDER_ZIGZAG ? S / (2 * P) : S / P;
    if (chunk % tile_q != 0) return RM_ERR_UNSUPPORTED;
    if (dtype == RM_DTYPE_BF16 && (S / P) % (2 * tile_q) != 0) return RM_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(B) * H * S >= (1ll << 31)) return RM_ERR_UNSUPPORTED;
    return RM_OK;
}

// Window argument of the *_window entry points -> AttnShape::window: a window
// that covers the whole sequence is plain causal attention (0).
static rm_status window_arg(int window, int S, int* out) {
    if (window < 1) return RM_ERR_INVALID_ARG;
    *out = window >= S ? 0 : window;
    // the tile iterators add window and position in int arithmetic
    if (*out && S >= (1 << 30)) return RM_ERR_UNSUPPORTED;
    return RM_OK;
}

static rm_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int Hkv, int S, int D, int P, int causal, int window,
                          const void* bounds, rm_order order, rm_dtype dtype, float scale,
                          cudaStream_t stream, int mode = 0, int rank = 0, int owner = 0,
                          int merge = 0) {
    const int tile_q = dtype == RM_DTYPE_BF16 ? 128 : 64;
    rm_status st = check_attn(q, k, v, B, H, Hkv, S, D, P, order, dtype, scale, tile_q);
    if (st != RM_OK) return st;
    if (B == 0 || S == 0) return RM_OK;  // empty batch or sequence: nothing to do
    if (!o || !lse || !aligned16(o) || !aligned16(lse)) return RM_ERR_INVALID_ARG;
    LaunchCtx ctx;
    if ((st = get_ctx(stream, &ctx)) != RM_OK) return st;
    AttnShape sh{B, H, Hkv, S, D, P, causal ? 1 : 0, order == RM_ORDER_ZIGZAG ? 1 : 0, scale,
                 window, bounds, mode, rank, owner, merge};
    cudaError_t e = dtype == RM_DTYPE_BF16
                        ? launch_fwd_tc(sh, q, k, v, o, lse, ctx)
                        : launch_fwd_fp32(sh, static_cast<const float*>(q),
                                          static_cast<const float*>(k),
                                          static_cast<const float*>(v), static_cast<float*>(o),
                                          lse, ctx);
    return e == cudaSuccess ? RM_OK : cuda_fail(e);
}

static rm_status bwd_impl(const void* q, const void* k, const void* v, const void* o,
                          const float* lse, const void* dout, float* dq, float* dk, float* dv,
                          void* workspace, size_t workspace_bytes, int B, int H, int Hkv, int S,
                          int D, int P, int causal, int window, const void* bounds,
                          rm_order order, rm_dtype dtype, float scale, cudaStream_t stream);

// Layout of a varlen bounds buffer: S int4 entries, then (256-byte aligned) a
// device copy of the n_docs + 1 boundaries the entries were built from.
static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
static size_t varlen_table_bytes(int S) { return align256(static_cast<size_t>(S) * 16); }

}  // namespace rm

using namespace rm;

extern "C" {

const char* rm_status_string(rm_status s) {
    switch (s) {
        case RM_OK: return "ok";
        case RM_ERR_INVALID_ARG: return "invalid argument";
        case RM_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case RM_ERR_CUDA: return "CUDA error";
        case RM_ERR_TIMEOUT: return "in-kernel wait timed out";
        case RM_ERR_SLOT_REUSE: return "more launches in flight than work-counter slots";
        case RM_ERR_SMEM_LAYOUT: return "shared-memory layout did not fit the block";
    }
    return "unknown status";
}

int rm_last_cuda_error(void) { return t_last_cuda_error; }

void rm_set_watchdog_ns(uint64_t ns) { g_watchdog_ns.store(ns < 1000 ? 1000 : ns); }

void rm_set_bwd_deterministic(int on) { g_bwd_deterministic.store(on ? 1 : 0); }

int rm_get_bwd_deterministic(void) { return g_bwd_deterministic.load(); }

rm_status rm_check_device_status(cudaStream_t stream) {
    LaunchCtx ctx;
    rm_status st = get_ctx(stream, &ctx);
    if (st != RM_OK) return st;
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned word = 0;
    e = cudaMemcpyFromSymbol(&word, g_status_word, sizeof(word));
    if (e != cudaSuccess) return cuda_fail(e);
    if (word) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e);
        if (word & kErrSlotReuse) return RM_ERR_SLOT_REUSE;
        return (word & kErrSmemLayout) ? RM_ERR_SMEM_LAYOUT : RM_ERR_TIMEOUT;
    }
    return RM_OK;
}

rm_status rm_watchdog_selftest(uint64_t timeout_ns, cudaStream_t stream) {
    LaunchCtx ctx;
    rm_status st = get_ctx(stream, &ctx);
    if (st != RM_OK) return st;
    ctx.watchdog_ns = timeout_ns < 1000 ? 1000 : timeout_ns;
    cudaError_t e = launch_watchdog_selftest(ctx);
    return e == cudaSuccess ? RM_OK : cuda_fail(e);
}

rm_status rm_ring_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int H, int Hkv, int S, int D, int P, int causal,
                           rm_order order, rm_dtype dtype, float scale, cudaStream_t stream) {
    return fwd_impl(q, k, v, o, lse, B, H, Hkv, S, D, P, causal, 0, nullptr, order, dtype, scale,
                    stream);
}

rm_status rm_allgather_attn_fwd(const void* q, const void* k_all, const void* v_all, void* o,
                                float* lse, int B, int H, int Hkv, int S, int D, int P, int causal,
                                rm_order order, rm_dtype dtype, float scale, cudaStream_t stream) {
    if (dtype == RM_DTYPE_FP32) return RM_ERR_UNSUPPORTED;
    return fwd_impl(q, k_all, v_all, o, lse, B, H, Hkv, S, D, P, causal, 0, nullptr, order, dtype,
                    scale, stream, 1);
}

rm_status rm_ring_attn_fwd_step(const void* q_local, const void* k_block, const void* v_block,
                                float* o_part, float* lse_part, int B, int H, int Hkv, int S,
                                int D, int P, int rank, int owner, int causal, rm_order order,
                                rm_dtype dtype, float scale, cudaStream_t stream) {
    if (P <= 0 || rank < 0 || rank >= P || owner < 0 || owner >= P) return RM_ERR_INVALID_ARG;
    if (dtype == RM_DTYPE_FP32) return RM_ERR_UNSUPPORTED;
    return fwd_impl(q_local, k_block, v_block, o_part, lse_part, B, H, Hkv, S, D, P, causal, 0,
                    nullptr, order, dtype, scale, stream, 2, rank, owner);
}

rm_status rm_ring_attn_fwd_step_merge(const void* q_local, const void* k_block,
                                      const void* v_block, float* o_acc, float* lse_acc, int B,
                                      int H, int Hkv, int S, int D, int P, int rank, int owner,
                                      int causal, rm_order order, rm_dtype dtype, float scale,
                                      cudaStream_t stream) {
    if (P <= 0 || rank < 0 || rank >= P || owner < 0 || owner >= P) return RM_ERR_INVALID_ARG;
    if (dtype == RM_DTYPE_FP32) return RM_ERR_UNSUPPORTED;
    return fwd_impl(q_local, k_block, v_block, o_acc, lse_acc, B, H, Hkv, S, D, P, causal, 0,
                    nullptr, order, dtype, scale, stream, 2, rank, owner, 1);
}

rm_status rm_ring_attn_fwd_window(const void* q, const void* k, const void* v, void* o,
                                  float* lse, int B, int H, int Hkv, int S, int D, int P,
                                  int window, rm_order order, rm_dtype dtype, float scale,
                                  cudaStream_t stream) {
    int w = 0;
    rm_status st = window_arg(window, S, &w);
    if (st != RM_OK) return st;
    return fwd_impl(q, k, v, o, lse, B, H, Hkv, S, D, P, 1, w, nullptr, order, dtype, scale, stream);
}

size_t rm_varlen_bounds_size(int S, int n_docs) {
    if (S <= 0 || n_docs <= 0) return 0;
    return varlen_table_bytes(S) + align256(static_cast<size_t>(n_docs + 1) * 4);
}

rm_status rm_varlen_bounds(const int* cu_seqlens, int n_docs, int S, int causal, int window,
                           void* bounds, size_t bounds_bytes, cudaStream_t stream) {
    if (n_docs <= 0 || S < 0 || window < 0 || !cu_seqlens) return RM_ERR_INVALID_ARG;
    if (window > 0 && !causal) return RM_ERR_INVALID_ARG;
    if (cu_seqlens[0] != 0 || cu_seqlens[n_docs] != S) return RM_ERR_INVALID_ARG;
    for (int d = 0; d < n_docs; ++d)
        if (cu_seqlens[d] > cu_seqlens[d + 1]) return RM_ERR_INVALID_ARG;
    if (S == 0) return RM_OK;
    if (!bounds || (reinterpret_cast<uintptr_t>(bounds) & 255u) != 0) return RM_ERR_INVALID_ARG;
    if (bounds_bytes < rm_varlen_bounds_size(S, n_docs)) return RM_ERR_INVALID_ARG;
    if (window >= S) window = 0;
    LaunchCtx ctx;
    rm_status st = get_ctx(stream, &ctx);
    if (st != RM_OK) return st;
    int* cu_dev = reinterpret_cast<int*>(static_cast<char*>(bounds) + varlen_table_bytes(S));
    // from pageable host memory: the host array may be reused once this returns
    cudaError_t e = cudaMemcpyAsync(cu_dev, cu_seqlens, static_cast<size_t>(n_docs + 1) * 4,
                                    cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    e = launch_varlen_bounds(cu_dev, n_docs, S, causal ? 1 : 0, window, bounds, ctx);
    return e == cudaSuccess ? RM_OK : cuda_fail(e);
}

rm_status rm_ring_attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                                  const void* bounds, int B, int H, int Hkv, int S, int D, int P,
                                  rm_order order, rm_dtype dtype, float scale,
                                  cudaStream_t stream) {
    if (S > 0 && B > 0 && (!bounds || (reinterpret_cast<uintptr_t>(bounds) & 255u) != 0))
        return RM_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, o, lse, B, H, Hkv, S, D, P, 1, 0, bounds, order, dtype, scale,
                    stream);
}

size_t rm_ring_attn_bwd_workspace_size(int B, int H, int S) {
    if (B <= 0 || H <= 0 || S <= 0) return 0;  // empty problems need no scratch
    const size_t delta = static_cast<size_t>(B) * H * S * sizeof(float);
    return (delta + 255) & ~static_cast<size_t>(255);
}

rm_status rm_ring_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                           const float* lse, const void* dout, float* dq, float* dk, float* dv,
                           void* workspace, size_t workspace_bytes, int B, int H, int Hkv,
                           int S, int D, int P, int causal, rm_order order, rm_dtype dtype,
                           float scale, cudaStream_t stream) {
    return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv, S, D,
                    P, causal, 0, nullptr, order, dtype, scale, stream);
}

rm_status rm_ring_attn_bwd_window(const void* q, const void* k, const void* v, const void* o,
                                  const float* lse, const void* dout, float* dq, float* dk,
                                  float* dv, void* workspace, size_t workspace_bytes, int B,
                                  int H, int Hkv, int S, int D, int P, int window, rm_order order,
                                  rm_dtype dtype, float scale, cudaStream_t stream) {
    int w = 0;
    rm_status st = window_arg(window, S, &w);
    if (st != RM_OK) return st;
    return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv, S, D,
                    P, 1, w, nullptr, order, dtype, scale, stream);
}

rm_status rm_ring_attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                                  const float* lse, const void* dout, float* dq, float* dk,
                                  float* dv, const void* bounds, void* workspace,
                                  size_t workspace_bytes, int B, int H, int Hkv, int S, int D,
                                  int P, rm_order order, rm_dtype dtype, float scale,
                                  cudaStream_t stream) {
    if (S > 0 && B > 0 && (!bounds || (reinterpret_cast<uintptr_t>(bounds) & 255u) != 0))
        return RM_ERR_INVALID_ARG;
    return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv, S, D,
                    P, 1, 0, bounds, order, dtype, scale, stream);
}

}  // extern "C"

namespace rm {

static rm_status bwd_impl(const void* q, const void* k, const void* v, const void* o,
                          const float* lse, const void* dout, float* dq, float* dk, float* dv,
                          void* workspace, size_t workspace_bytes, int B, int H, int Hkv, int S,
                          int D, int P, int causal, int window, const void* bounds,
                          rm_order order, rm_dtype dtype, float scale, cudaStream_t stream) {
    rm_status st = check_attn(q, k, v, B, H, Hkv, S, D, P, order, dtype, scale, 128);
    if (st != RM_OK) return st;
    if (dtype != RM_DTYPE_BF16) return RM_ERR_UNSUPPORTED;
    if (B == 0 || S == 0) return RM_OK;
    const void* ptrs[] = {o, lse, dout, dq, dk, dv, workspace};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return RM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return RM_ERR_INVALID_ARG;
    if (workspace_bytes < rm_ring_attn_bwd_workspace_size(B, H, S)) return RM_ERR_INVALID_ARG;
    LaunchCtx ctx;
    if ((st = get_ctx(stream, &ctx)) != RM_OK) return st;
    AttnShape sh{B, H, Hkv, S, D, P, causal ? 1 : 0, order == RM_ORDER_ZIGZAG ? 1 : 0, scale,
                 window, bounds};
    sh.deterministic = g_bwd_deterministic.load();
    cudaError_t e = launch_bwd(sh, q, k, v, o, lse, dout, dq, dk, dv,
                               static_cast<float*>(workspace), ctx);
    return e == cudaSuccess ? RM_OK : cuda_fail(e);
}

}  // namespace rm

extern "C" {

rm_status rm_ring_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                   const float* lse, const void* dout, float* dq, float* dk,
                                   float* dv, int B, int H, int Hkv, int S, int D, int P, int causal,
                                   rm_order order, rm_dtype dtype, float scale, cudaStream_t stream) {
    rm_status st = check_attn(q, k, v, B, H, Hkv, S, D, P, order, dtype, scale, 128);
    if (st != RM_OK) return st;
    if (dtype != RM_DTYPE_BF16) return RM_ERR_UNSUPPORTED;
    if (B == 0 || S == 0) return RM_OK;
    const void* ptrs[] = {o, lse, dout, dq, dk, dv};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return RM_ERR_INVALID_ARG;
    if (static_cast<size_t>(B) * H * S > kNoAllocMaxRows) return RM_ERR_UNSUPPORTED;
    LaunchCtx ctx;
    if ((st = get_ctx(stream, &ctx)) != RM_OK) return st;
    float* scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != RM_OK) return st;
    AttnShape sh{B, H, Hkv, S, D, P, causal ? 1 : 0, order == RM_ORDER_ZIGZAG ? 1 : 0, scale};
    sh.deterministic = g_bwd_deterministic.load();
    // Delta is rewritten in full by the backward's first kernel, so the
    // previous call's contents need no clearing.
    cudaError_t e = launch_bwd(sh, q, k, v, o, lse, dout, dq, dk, dv, scratch, ctx);
    return e == cudaSuccess ? RM_OK : cuda_fail(e);
}

rm_status rm_ring_attn_bwd_delta(const void* o, const void* dout, float* delta, int64_t rows,
                                 int D, rm_dtype o_dtype, cudaStream_t stream) {
    if (rows < 0 || D <= 0) return RM_ERR_INVALID_ARG;
    if (o_dtype != RM_DTYPE_BF16 && o_dtype != RM_DTYPE_FP32) return RM_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return RM_ERR_UNSUPPORTED;
    if (rows == 0) return RM_OK;
    if (!o || !dout || !delta || !aligned16(o) || !aligned16(dout) || !aligned16(delta))
        return RM_ERR_INVALID_ARG;
    LaunchCtx ctx;
    rm_status st = get_ctx(stream, &ctx);
    if (st != RM_OK) return st;
    cudaError_t e = launch_bwd_delta(o, o_dtype == RM_DTYPE_FP32, dout, delta, rows, D, ctx);
    return e == cudaSuccess ? RM_OK : cuda_fail(e);
}

rm_status rm_ring_attn_bwd_step(const void* q_local, const void* k_block, const void* v_block,
                                const float* lse_local, const float* delta_local,
                                const void* dout_local, float* dq_local, float* dk_block,
                                float* dv_block, int B, int H, int Hkv, int S, int D, int P,
                                int rank, int owner, int causal, rm_order order, rm_dtype dtype,
                                float scale, cudaStream_t stream) {
    if (P <= 0 || rank < 0 || rank >= P || owner < 0 || owner >= P) return RM_ERR_INVALID_ARG;
    rm_status st = check_attn(q_local, k_block, v_block, B, H, Hkv, S, D, P, order, dtype, scale,
                              128);
    if (st != RM_OK) return st;
    if (dtype != RM_DTYPE_BF16) return RM_ERR_UNSUPPORTED;
    if (B == 0 || S == 0) return RM_OK;
    const void* ptrs[] = {lse_local, delta_local, dout_local, dq_local, dk_block, dv_block};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return RM_ERR_INVALID_ARG;
    LaunchCtx ctx;
    if ((st = get_ctx(stream, &ctx)) != RM_OK) return st;
    AttnShape sh{B, H, Hkv, S, D, P, causal ? 1 : 0, order == RM_ORDER_ZIGZAG ? 1 : 0, scale, 0,
                 nullptr, 2, rank, owner, 0};
    sh.deterministic = g_bwd_deterministic.load();
    cudaError_t e = launch_bwd(sh, q_local, k_block, v_block, nullptr, lse_local, dout_local,
                               dq_local, dk_block, dv_block, const_cast<float*>(delta_local), ctx);
    return e == cudaSuccess ? RM_OK : cuda_fail(e);
}

rm_status rm_lse_merge(float* o_acc, float* lse_acc, const float* o_part, const float* lse_part,
                       int64_t rows, int D, cudaStream_t stream) {
    if (rows < 0 || D <= 0) return RM_ERR_INVALID_ARG;
    if (rows == 0) return RM_OK;
    if (!o_acc || !lse_acc || !o_part || !lse_part) return RM_ERR_INVALID_ARG;
    if (!aligned16(o_acc) || !aligned16(o_part) || !aligned16(lse_acc) || !aligned16(lse_part))
        return RM_ERR_INVALID_ARG;
    LaunchCtx ctx;
    rm_status st = get_ctx(stream, &ctx);
    if (st != RM_OK) return st;
    cudaError_t e = launch_lse_merge(o_acc, lse_acc, o_part, lse_part, rows, D, ctx);
    return e == cudaSuccess ? RM_OK : cuda_fail(e);
}

static rm_status check_permute(int B, int S, int D, int U, int R, int elem_bytes,
                               rm_permute_dir dir) {
    if (B < 0 || S < 0 || D <= 0 || U <= 0 || R <= 0) return RM_ERR_INVALID_ARG;
    if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)
        return RM_ERR_INVALID_ARG;
    if (dir != RM_SEQ_TO_HEAD && dir != RM_HEAD_TO_SEQ) return RM_ERR_INVALID_ARG;
    if (S % (U * R) != 0) return RM_ERR_INVALID_ARG;
    return RM_OK;
}

rm_status rm_ulysses_permute(const void* src, void* dst, int B, int S, int Hx, int D, int U,
                             int R, int elem_bytes, rm_permute_dir dir, cudaStream_t stream) {
    rm_status st = check_permute(B, S, D, U, R, elem_bytes, dir);
    if (st != RM_OK) return st;
    if (Hx <= 0 || Hx % U != 0) return RM_ERR_INVALID_ARG;
    if (B == 0 || S == 0) return RM_OK;
    if (!src || !dst || !aligned16(src) || !aligned16(dst) || src == dst) return RM_ERR_INVALID_ARG;
    LaunchCtx ctx;
    if ((st = get_ctx(stream, &ctx)) != RM_OK) return st;
    PermuteTensor t{src, dst, Hx};
    cudaError_t e = launch_ulysses_permute(&t, 1, B, S, D, elem_bytes, dir == RM_HEAD_TO_SEQ, ctx);
    return e == cudaSuccess ? RM_OK : cuda_fail(e);
}

rm_status rm_ulysses_permute_qkv(const void* q_src, const void* k_src, const void* v_src,
                                 void* q_dst, void* k_dst, void* v_dst, int B, int S, int H,
                                 int Hkv, int D, int U, int R, int elem_bytes,
                                 rm_permute_dir dir, cudaStream_t stream) {
    rm_status st = check_permute(B, S, D, U, R, elem_bytes, dir);
    if (st != RM_OK) return st;
    if (H <= 0 || Hkv <= 0 || H % U != 0 || Hkv % U != 0) return RM_ERR_INVALID_ARG;
    if (B == 0 || S == 0) return RM_OK;
    const void* ptrs[] = {q_src, k_src, v_src, q_dst, k_dst, v_dst};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return RM_ERR_INVALID_ARG;
    LaunchCtx ctx;
    if ((st = get_ctx(stream, &ctx)) != RM_OK) return st;
    PermuteTensor t[3] = {{q_src, q_dst, H}, {k_src, k_dst, Hkv}, {v_src, v_dst, Hkv}};
    cudaError_t e = launch_ulysses_permute(t, 3, B, S, D, elem_bytes, dir == RM_HEAD_TO_SEQ, ctx);
    return e == cudaSuccess ? RM_OK : cuda_fail(e);
}

static rm_status ulysses_exchange(const void* const* tensors, const int* heads, int ntensors,
                                  void* buf, int B, int s, int D, int U, int elem_bytes,
                                  rm_permute_dir dir, int pack, cudaStream_t stream) {
    if (B < 0 || s < 0 || D <= 0 || U <= 0) return RM_ERR_INVALID_ARG;
    if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)
        return RM_ERR_INVALID_ARG;
    if (dir != RM_SEQ_TO_HEAD && dir != RM_HEAD_TO_SEQ) return RM_ERR_INVALID_ARG;
    if (ntensors < 1 || ntensors > 3 || !tensors || !heads) return RM_ERR_INVALID_ARG;
    UlyTensor t[3];
    for (int i = 0; i < ntensors; ++i) {
        if (heads[i] <= 0 || heads[i] % U != 0) return RM_ERR_INVALID_ARG;
        t[i] = UlyTensor{tensors[i], heads[i]};
    }
    if (static_cast<int64_t>(U) * s >= (1ll << 31)) return RM_ERR_UNSUPPORTED;
    if (B == 0 || s == 0) return RM_OK;
    if (!buf || !aligned16(buf)) return RM_ERR_INVALID_ARG;
    for (int i = 0; i < ntensors; ++i)
        if (!t[i].tensor || !aligned16(t[i].tensor) || t[i].tensor == buf) return RM_ERR_INVALID_ARG;
    LaunchCtx ctx;
    rm_status st = get_ctx(stream, &ctx);
    if (st != RM_OK) return st;
    const int head_side = pack ? dir == RM_HEAD_TO_SEQ : dir == RM_SEQ_TO_HEAD;
    cudaError_t e = launch_ulysses_exchange(t, ntensors, buf, B, s, D, U, elem_bytes, pack,
                                            head_side, ctx);
    return e == cudaSuccess ? RM_OK : cuda_fail(e);
}

size_t rm_ulysses_buffer_size(const int* heads, int ntensors, int B, int s, int D,
                              int elem_bytes) {
    if (!heads || ntensors < 1 || ntensors > 3 || B <= 0 || s <= 0 || D <= 0 || elem_bytes <= 0)
        return 0;
    size_t n = 0;
    for (int i = 0; i < ntensors; ++i) n += static_cast<size_t>(heads[i] > 0 ? heads[i] : 0);
    return n * static_cast<size_t>(B) * s * D * elem_bytes;
}

rm_status rm_ulysses_pack(const void* const* tensors, const int* heads, int ntensors,
                          void* send_buf, int B, int s, int D, int U, int elem_bytes,
                          rm_permute_dir dir, cudaStream_t stream) {
    return ulysses_exchange(tensors, heads, ntensors, send_buf, B, s, D, U, elem_bytes, dir, 1,
                            stream);
}

rm_status rm_ulysses_unpack(const void* recv_buf, void* const* tensors, const int* heads,
                            int ntensors, int B, int s, int D, int U, int elem_bytes,
                            rm_permute_dir dir, cudaStream_t stream) {
    return ulysses_exchange(const_cast<const void* const*>(tensors), heads, ntensors,
                            const_cast<void*>(recv_buf), B, s, D, U, elem_bytes, dir, 0, stream);
}

rm_status rm_seq_reorder(const void* src, void* dst, int B, int H, int S, int D, int P,
                         rm_order order, rm_reorder_dir dir, int elem_bytes,
                         cudaStream_t stream) {
    if (B < 0 || H <= 0 || S < 0 || D <= 0 || P <= 0) return RM_ERR_INVALID_ARG;
    if (!valid_order(order)) return RM_ERR_INVALID_ARG;
    if (dir != RM_NATURAL_TO_RANK_MAJOR && dir != RM_RANK_MAJOR_TO_NATURAL)
        return RM_ERR_INVALID_ARG;
    if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)
        return RM_ERR_INVALID_ARG;
    if (order == RM_ORDER_ZIGZAG ? (S % (2 * P) != 0) : (S % P != 0)) return RM_ERR_INVALID_ARG;
    if (static_cast<int64_t>(B) * H >= (1ll << 31)) return RM_ERR_UNSUPPORTED;
    if (B == 0 || S == 0) return RM_OK;
    if (!src || !dst || src == dst) return RM_ERR_INVALID_ARG;
    LaunchCtx ctx;
    rm_status st = get_ctx(stream, &ctx);
    if (st != RM_OK) return st;
    cudaError_t e = launch_seq_reorder(src, dst, B * H, S, D, P, order == RM_ORDER_ZIGZAG,
                                       dir == RM_RANK_MAJOR_TO_NATURAL, elem_bytes, ctx);
    return e == cudaSuccess ? RM_OK : cuda_fail(e);
}

}  // extern "C"
