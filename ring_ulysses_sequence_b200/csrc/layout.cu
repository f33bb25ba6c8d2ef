// HBM-bound layout kernels: the Ulysses seq<->head permute (one tensor or fused
// Q/K/V), the natural <-> rank-major token reorder, the standalone LSE merge,
// and the watchdog self-test.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace rm {

namespace {

template <int V> struct VecT;
template <> struct VecT<16> { using T = uint4; };
template <> struct VecT<8> { using T = uint2; };
template <> struct VecT<4> { using T = uint32_t; };
template <> struct VecT<2> { using T = uint16_t; };
template <> struct VecT<1> { using T = uint8_t; };

// Streaming (evict-first) accesses: every byte is touched exactly once.
template <typename T> __device__ __forceinline__ T ld_stream(const T* p) { return __ldcs(p); }
template <typename T> __device__ __forceinline__ void st_stream(T* p, T v) { __stcs(p, v); }
template <> __device__ __forceinline__ uint16_t ld_stream(const uint16_t* p) { return *p; }
template <> __device__ __forceinline__ void st_stream(uint16_t* p, uint16_t v) { *p = v; }
template <> __device__ __forceinline__ uint8_t ld_stream(const uint8_t* p) { return *p; }
template <> __device__ __forceinline__ void st_stream(uint8_t* p, uint8_t v) { *p = v; }

constexpr int kThreads = 256;
constexpr int kUnroll = 4;
constexpr int kTileVecs = 4096;  // vectors moved per block (64 KB at 16 B)

struct PermuteTensorArgs {
    const char* src;
    char* dst;
    int H;
    int tok_per_tile;      // tokens per block tile
    int tiles_per_b;
    int64_t block_start;   // first block of this tensor
    FastDiv div_vpr;       // by vectors per row
    FastDiv div_h;         // by heads
};

struct PermuteArgs {
    PermuteTensorArgs t[3];
    int64_t block_end;
    int ntensors;
    int S, vec_per_row;
    int head_to_seq;
};

// Element (b, s, h, :) sits at row (b*S + s)*H + h in the sequence-sharded
// layout [B, S, H, D] and at row (b*H + h)*S + s in the head-sharded layout
// [B, H, S, D]. A block moves tok_per_tile whole tokens (all heads) of one b:
// its sequence-side range is one contiguous run, its head-side accesses whole
// D-element rows.
template <int V>
__global__ void __launch_bounds__(kThreads) ulysses_permute_kernel(const __grid_constant__ PermuteArgs a) {
    using T = typename VecT<V>::T;
    int ti = 0;
    while (ti + 1 < a.ntensors && static_cast<int64_t>(blockIdx.x) >= a.t[ti + 1].block_start) ++ti;
    const PermuteTensorArgs& pt = a.t[ti];
    const int64_t blk = static_cast<int64_t>(blockIdx.x) - pt.block_start;
    const int64_t b = blk / pt.tiles_per_b;
    const int s0 = static_cast<int>(blk - b * pt.tiles_per_b) * pt.tok_per_tile;
    const int ns = min(pt.tok_per_tile, a.S - s0);
    const int H = pt.H, vpr = a.vec_per_row;
    const uint32_t n = static_cast<uint32_t>(ns) * H * vpr;
    const int64_t seq_base = ((b * a.S + s0) * H) * vpr;
    const int64_t head_base = (b * H * static_cast<int64_t>(a.S) + s0) * vpr;
    const int64_t head_stride = static_cast<int64_t>(a.S) * vpr;  // between heads
    const T* src = reinterpret_cast<const T*>(pt.src);
    T* dst = reinterpret_cast<T*>(pt.dst);
    for (uint32_t i0 = threadIdx.x; i0 < n; i0 += kThreads * kUnroll) {
        T val[kUnroll];
        int64_t hoff[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t i = i0 + u * kThreads;
            hoff[u] = -1;
            if (i < n) {
                const uint32_t row = pt.div_vpr.div(i);
                const uint32_t vin = i - row * vpr;
                const uint32_t sl = pt.div_h.div(row);
                const uint32_t h = row - sl * H;
                hoff[u] = head_base + h * head_stride + static_cast<int64_t>(sl) * vpr + vin;
                val[u] = ld_stream(a.head_to_seq ? src + hoff[u] : src + seq_base + i);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t i = i0 + u * kThreads;
            if (hoff[u] >= 0) st_stream(a.head_to_seq ? dst + seq_base + i : dst + hoff[u], val[u]);
        }
    }
}

// Ulysses exchange buffers of one device (U devices per Ulysses group, each
// holding s tokens of all heads before the all-to-all). The buffer is U
// chunks, chunk u for (or from) device u; in a chunk the tensors follow one
// another, tensor x as [B, s, heads_x / U, D] (the s tokens of the sending
// device for the heads of the receiving one). The device's own tensor x is
//   sequence side [B, s, heads_x, D]          (heads u*hU + hh of token t), or
//   head side     [B, hU, U*s, D]             (token u*s + t of head hh),
// hU = heads_x / U. pack: tensor -> buffer; unpack: buffer -> tensor. A block
// moves tok_per_tile tokens x hU heads of one (x, u, b): a contiguous run of
// the buffer, whole D-element rows of the tensor.
struct UlyPart {
    const char* tensor;
    char* buf;           // the buffer's first byte (the same for every tensor)
    int hU;              // heads of the tensor per device
    int heads;           // all heads of the tensor (sequence side)
    int64_t chunk_off;   // vectors from a chunk's start to this tensor's part
    int tok_per_tile, tiles_per_ub;
    int64_t block_start;
    FastDiv div_row;     // by hU * vec_per_row
};

struct UlyArgs {
    UlyPart t[3];
    int ntensors;
    int B, s, U, vec_per_row;
    int64_t chunk_vecs;  // vectors per chunk
    int pack, head_side;
    FastDiv div_vpr;
};

template <int V>
__global__ void __launch_bounds__(kThreads) ulysses_exchange_kernel(const __grid_constant__ UlyArgs a) {
    using T = typename VecT<V>::T;
    int ti = 0;
    while (ti + 1 < a.ntensors && static_cast<int64_t>(blockIdx.x) >= a.t[ti + 1].block_start) ++ti;
    const UlyPart& pt = a.t[ti];
    int64_t blk = static_cast<int64_t>(blockIdx.x) - pt.block_start;
    const int tile = static_cast<int>(blk % pt.tiles_per_ub);
    blk /= pt.tiles_per_ub;
    const int b = static_cast<int>(blk % a.B);
    const int u = static_cast<int>(blk / a.B);
    const int t0 = tile * pt.tok_per_tile;
    const int nt = min(pt.tok_per_tile, a.s - t0);
    const int vpr = a.vec_per_row, hU = pt.hU;
    const uint32_t n = static_cast<uint32_t>(nt) * hU * vpr;
    const int64_t buf_base = u * a.chunk_vecs + pt.chunk_off +
                             (static_cast<int64_t>(b) * a.s + t0) * hU * vpr;
    T* buf = reinterpret_cast<T*>(pt.buf);
    T* ten = reinterpret_cast<T*>(const_cast<char*>(pt.tensor));
    for (uint32_t i0 = threadIdx.x; i0 < n; i0 += kThreads * kUnroll) {
        T val[kUnroll];
        int64_t toff[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const uint32_t i = i0 + k * kThreads;
            toff[k] = -1;
            if (i < n) {
                const uint32_t tl = pt.div_row.div(i);            // token within the tile
                const uint32_t rem = i - tl * hU * vpr;
                const uint32_t hh = a.div_vpr.div(rem);           // head within the device's share
                const uint32_t vin = rem - hh * vpr;
                const int64_t t = t0 + tl;
                toff[k] = a.head_side
                              ? ((static_cast<int64_t>(b) * hU + hh) * a.U * a.s + u * a.s + t) * vpr + vin
                              : ((b * a.s + t) * pt.heads + u * hU + hh) * vpr + vin;
                val[k] = ld_stream(a.pack ? ten + toff[k] : buf + buf_base + i);
            }
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const uint32_t i = i0 + k * kThreads;
            if (toff[k] >= 0) st_stream(a.pack ? buf + buf_base + i : ten + toff[k], val[k]);
        }
    }
}

struct ReorderArgs {
    const char* src;
    char* dst;
    int S, vec_per_row, rows_per_tile, tiles_per_bh;
    int to_natural;
    FastDiv div_vpr;
    RingLayout lay;
};

// A block fills rows_per_tile consecutive destination rows of one (b, h).
template <int V>
__global__ void __launch_bounds__(kThreads) seq_reorder_kernel(const __grid_constant__ ReorderArgs a) {
    using T = typename VecT<V>::T;
    const int64_t blk = blockIdx.x;
    const int64_t bh = blk / a.tiles_per_bh;
    const int s0 = static_cast<int>(blk - bh * a.tiles_per_bh) * a.rows_per_tile;
    const int ns = min(a.rows_per_tile, a.S - s0);
    const uint32_t n = static_cast<uint32_t>(ns) * a.vec_per_row;
    const T* src = reinterpret_cast<const T*>(a.src) + bh * a.S * static_cast<int64_t>(a.vec_per_row);
    T* dst = reinterpret_cast<T*>(a.dst) + (bh * a.S + s0) * static_cast<int64_t>(a.vec_per_row);
    for (uint32_t i = threadIdx.x; i < n; i += kThreads) {
        const uint32_t sl = a.div_vpr.div(i);
        const uint32_t vin = i - sl * a.vec_per_row;
        const int s = s0 + static_cast<int>(sl);
        // natural->rank-major: destination slot s takes natural position pos(s);
        // rank-major->natural: destination position s takes the slot holding it.
        const int from = a.to_natural ? a.lay.slot_of_pos(s) : a.lay.pos_of_slot(s);
        dst[i] = src[static_cast<int64_t>(from) * a.vec_per_row + vin];
    }
}

// One warp per row: every lane reads the row's two LSE values before lane 0
// overwrites lse_acc, so the in-place update needs no cross-warp ordering.
__global__ void __launch_bounds__(kThreads) lse_merge_kernel(float* __restrict__ o_acc,
                                                             float* __restrict__ lse_acc,
                                                             const float* __restrict__ o_part,
                                                             const float* __restrict__ lse_part,
                                                             int64_t rows, int D) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    for (int64_t r = warp; r < rows; r += nwarps) {
        const float a = lse_acc[r], b = lse_part[r];
        const float M = fmaxf(a, b);
        float* oa = o_acc + r * D;
        const float* ob = o_part + r * D;
        if (M == -INFINITY) {
            for (int d = lane; d < D; d += 32) oa[d] = 0.0f;
            __syncwarp();
            if (lane == 0) lse_acc[r] = -INFINITY;
            continue;
        }
        const float wa = expf(a - M), wb = expf(b - M);
        const float inv = 1.0f / (wa + wb);
        if ((D & 3) == 0) {
            float4* oa4 = reinterpret_cast<float4*>(oa);
            const float4* ob4 = reinterpret_cast<const float4*>(ob);
            for (int d = lane; d < D / 4; d += 32) {
                float4 x = oa4[d], y = ob4[d];
                x.x = (wa * x.x + wb * y.x) * inv;
                x.y = (wa * x.y + wb * y.y) * inv;
                x.z = (wa * x.z + wb * y.z) * inv;
                x.w = (wa * x.w + wb * y.w) * inv;
                oa4[d] = x;
            }
        } else {
            for (int d = lane; d < D; d += 32) oa[d] = (wa * oa[d] + wb * ob[d]) * inv;
        }
        __syncwarp();
        if (lane == 0) lse_acc[r] = M + logf(wa + wb);
    }
}

// A barrier that nothing completes: the bounded wait must give up and report.
__global__ void watchdog_selftest_kernel(unsigned* status_word, uint64_t limit_ns) {
    __shared__ alignas(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(smem_u32(&bar), 1);
        fence_barrier_init();
    }
    __syncthreads();
    Watchdog wd{status_word, &abort_flag, limit_ns};
    if (threadIdx.x == 0) (void)mbar_wait(smem_u32(&bar), 0, wd);
    __syncthreads();
}

int pick_vec(int64_t row_bytes, const void* a, const void* b) {
    const uintptr_t al = reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b);
    for (int v = 16; v > 1; v >>= 1)
        if (row_bytes % v == 0 && (al % v) == 0) return v;
    return 1;
}

// Per-token visibility bounds of packed documents (axolotl-ringmaster README,
// Status: packing / varlen). cu[0..n] rises from 0 to S (checked on the host);
// token i lies in document d with cu[d] <= i < cu[d+1] (the last such d when
// empty documents repeat a boundary). A query sees the keys of its own
// document, up to itself when causal and not before i - W + 1 with a window:
//   lo(i) = max(cu[d], i - W + 1),  hi(i) = causal ? i : cu[d+1] - 1;
// and a key j is seen by the queries
//   imin(j) = causal ? j : cu[d],  imax(j) = min(cu[d+1] - 1, j + W - 1).
__global__ void __launch_bounds__(256) varlen_bounds_kernel(const int* __restrict__ cu, int n_docs,
                                                            int S, int causal, int window,
                                                            int4* __restrict__ tab) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < S; i += gridDim.x * blockDim.x) {
        int a = 0, b = n_docs - 1;  // largest d in [0, n) with cu[d] <= i
        while (a < b) {
            const int mid = (a + b + 1) >> 1;
            if (cu[mid] <= i) a = mid;
            else b = mid - 1;
        }
        const int ds = cu[a], de = cu[a + 1];
        int lo = ds, imax = de - 1;
        if (causal && window) {
            lo = max(lo, i - window + 1);
            imax = min(imax, i + window - 1);
        }
        tab[i] = make_int4(lo, causal ? i : de - 1, causal ? i : ds, imax);
    }
}

}  // namespace

cudaError_t launch_varlen_bounds(const int* cu_dev, int n_docs, int S, int causal, int window,
                                 void* table, const LaunchCtx& ctx) {
    const int threads = 256;
    const int blocks = std::max(1, std::min((S + threads - 1) / threads, ctx.num_sms * 8));
    varlen_bounds_kernel<<<blocks, threads, 0, ctx.stream>>>(cu_dev, n_docs, S, causal, window,
                                                             static_cast<int4*>(table));
    return cudaGetLastError();
}

cudaError_t launch_ulysses_permute(const PermuteTensor* t, int ntensors, int B, int S, int D,
                                   int elem_bytes, int head_to_seq, const LaunchCtx& ctx) {
    const int64_t row_bytes = static_cast<int64_t>(D) * elem_bytes;
    int V = 16;
    for (int i = 0; i < ntensors; ++i) V = std::min(V, pick_vec(row_bytes, t[i].src, t[i].dst));
    PermuteArgs a{};
    a.ntensors = ntensors;
    a.S = S;
    a.vec_per_row = static_cast<int>(row_bytes / V);
    a.head_to_seq = head_to_seq;
    int64_t blocks = 0;
    for (int i = 0; i < ntensors; ++i) {
        PermuteTensorArgs& p = a.t[i];
        p.src = static_cast<const char*>(t[i].src);
        p.dst = static_cast<char*>(t[i].dst);
        p.H = t[i].heads;
        const int64_t per_tok = static_cast<int64_t>(p.H) * a.vec_per_row;
        if (per_tok >= (1ll << 30)) return cudaErrorInvalidValue;
        p.tok_per_tile = static_cast<int>(std::max<int64_t>(1, kTileVecs / per_tok));
        p.tok_per_tile = std::min(p.tok_per_tile, S);
        p.tiles_per_b = (S + p.tok_per_tile - 1) / p.tok_per_tile;
        p.block_start = blocks;
        p.div_vpr.init(static_cast<uint32_t>(a.vec_per_row));
        p.div_h.init(static_cast<uint32_t>(p.H));
        blocks += static_cast<int64_t>(B) * p.tiles_per_b;
    }
    a.block_end = blocks;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffll) return cudaErrorInvalidValue;
    dim3 grid(static_cast<unsigned>(blocks));
    switch (V) {
        case 16: ulysses_permute_kernel<16><<<grid, kThreads, 0, ctx.stream>>>(a); break;
        case 8: ulysses_permute_kernel<8><<<grid, kThreads, 0, ctx.stream>>>(a); break;
        case 4: ulysses_permute_kernel<4><<<grid, kThreads, 0, ctx.stream>>>(a); break;
        case 2: ulysses_permute_kernel<2><<<grid, kThreads, 0, ctx.stream>>>(a); break;
        default: ulysses_permute_kernel<1><<<grid, kThreads, 0, ctx.stream>>>(a); break;
    }
    return cudaGetLastError();
}

cudaError_t launch_ulysses_exchange(const UlyTensor* t, int ntensors, void* buf, int B, int s,
                                    int D, int U, int elem_bytes, int pack, int head_side,
                                    const LaunchCtx& ctx) {
    const int64_t row_bytes = static_cast<int64_t>(D) * elem_bytes;
    int V = 16;
    for (int i = 0; i < ntensors; ++i) V = std::min(V, pick_vec(row_bytes, t[i].tensor, buf));
    UlyArgs a{};
    a.ntensors = ntensors;
    a.B = B;
    a.s = s;
    a.U = U;
    a.vec_per_row = static_cast<int>(row_bytes / V);
    a.pack = pack;
    a.head_side = head_side;
    a.div_vpr.init(static_cast<uint32_t>(a.vec_per_row));
    int64_t off = 0, blocks = 0;
    for (int i = 0; i < ntensors; ++i) {
        UlyPart& p = a.t[i];
        p.tensor = static_cast<const char*>(t[i].tensor);
        p.buf = static_cast<char*>(buf);
        p.heads = t[i].heads;
        p.hU = t[i].heads / U;
        p.chunk_off = off;
        const int64_t per_tok = static_cast<int64_t>(p.hU) * a.vec_per_row;
        if (per_tok >= (1ll << 30)) return cudaErrorInvalidValue;
        off += static_cast<int64_t>(B) * s * per_tok;
        p.tok_per_tile = static_cast<int>(std::min<int64_t>(s, std::max<int64_t>(1, kTileVecs / per_tok)));
        p.tiles_per_ub = (s + p.tok_per_tile - 1) / p.tok_per_tile;
        p.block_start = blocks;
        p.div_row.init(static_cast<uint32_t>(per_tok));
        blocks += static_cast<int64_t>(U) * B * p.tiles_per_ub;
    }
    a.chunk_vecs = off;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffll) return cudaErrorInvalidValue;
    dim3 grid(static_cast<unsigned>(blocks));
    switch (V) {
        case 16: ulysses_exchange_kernel<16><<<grid, kThreads, 0, ctx.stream>>>(a); break;
        case 8: ulysses_exchange_kernel<8><<<grid, kThreads, 0, ctx.stream>>>(a); break;
        case 4: ulysses_exchange_kernel<4><<<grid, kThreads, 0, ctx.stream>>>(a); break;
        case 2: ulysses_exchange_kernel<2><<<grid, kThreads, 0, ctx.stream>>>(a); break;
        default: ulysses_exchange_kernel<1><<<grid, kThreads, 0, ctx.stream>>>(a); break;
    }
    return cudaGetLastError();
}

cudaError_t launch_seq_reorder(const void* src, void* dst, int BH, int S, int D, int P, int zigzag,
                               int to_natural, int elem_bytes, const LaunchCtx& ctx) {
    const int64_t row_bytes = static_cast<int64_t>(D) * elem_bytes;
    const int V = pick_vec(row_bytes, src, dst);
    if (row_bytes / V >= (1ll << 30)) return cudaErrorInvalidValue;
    ReorderArgs a{};
    a.src = static_cast<const char*>(src);
    a.dst = static_cast<char*>(dst);
    a.vec_per_row = static_cast<int>(row_bytes / V);
    a.S = S;
    a.rows_per_tile = std::min<int>(S, static_cast<int>(std::max<int64_t>(1, kTileVecs / a.vec_per_row)));
    a.tiles_per_bh = (S + a.rows_per_tile - 1) / a.rows_per_tile;
    a.to_natural = to_natural;
    a.div_vpr.init(static_cast<uint32_t>(a.vec_per_row));
    a.lay = RingLayout{S, P, S / P, zigzag ? S / (2 * P) : S / P, zigzag};
    const int64_t blocks = static_cast<int64_t>(BH) * a.tiles_per_bh;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffll) return cudaErrorInvalidValue;
    dim3 grid(static_cast<unsigned>(blocks));
    switch (V) {
        case 16: seq_reorder_kernel<16><<<grid, kThreads, 0, ctx.stream>>>(a); break;
        case 8: seq_reorder_kernel<8><<<grid, kThreads, 0, ctx.stream>>>(a); break;
        case 4: seq_reorder_kernel<4><<<grid, kThreads, 0, ctx.stream>>>(a); break;
        case 2: seq_reorder_kernel<2><<<grid, kThreads, 0, ctx.stream>>>(a); break;
        default: seq_reorder_kernel<1><<<grid, kThreads, 0, ctx.stream>>>(a); break;
    }
    return cudaGetLastError();
}

cudaError_t launch_lse_merge(float* o_acc, float* lse_acc, const float* o_part,
                             const float* lse_part, int64_t rows, int D, const LaunchCtx& ctx) {
    const int64_t warps_per_block = kThreads / 32;
    int64_t blocks = (rows + warps_per_block - 1) / warps_per_block;
    blocks = std::min<int64_t>(blocks, static_cast<int64_t>(ctx.num_sms) * 16);
    lse_merge_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, ctx.stream>>>(
        o_acc, lse_acc, o_part, lse_part, rows, D);
    return cudaGetLastError();
}

cudaError_t launch_watchdog_selftest(const LaunchCtx& ctx) {
    watchdog_selftest_kernel<<<1, 32, 0, ctx.stream>>>(ctx.status_word, ctx.watchdog_ns);
    return cudaGetLastError();
}

}  // namespace rm
