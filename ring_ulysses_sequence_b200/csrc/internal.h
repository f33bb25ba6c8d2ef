// Host-side interfaces between the C ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "rm.h"

namespace rm {

// Per-launch context: device status word, watchdog limit, device properties.
struct LaunchCtx {
    unsigned* status_word;   // device address of the status word
    int* work_counters;      // device address of kWorkSlots dynamic-schedule counters
    uint64_t watchdog_ns;
    int num_sms;
    cudaStream_t stream;
};

struct AttnShape {
    int B, H, Hkv, S, D, P, causal, zigzag;
    float scale;
    int window;            // causal left window in keys (query i sees i - window < j <= i); 0 = none
    const void* bounds;    // per-token int4 {lo, hi, imin, imax} of packed documents, or null
    // Forward only. mode 0: the whole ring (q, k, v rank-major, all S rows);
    // 1: k, v hold all S keys in natural order (all-gather); 2: one ring step of
    // rank `rank` (q, o, lse: its L = S / P rows; k, v: the L rows of `owner`'s
    // block; o is fp32).
    int mode;
    int rank, owner;
    int merge;             // mode 2: o, lse hold the running pair; fold the step into it
    // Backward only: 1 = the two-kernel path (every gradient element written
    // once: bitwise reproducible); 0 = the fused kernel (dQ by reductions).
    int deterministic;
};

// Dynamic work distribution: a persistent kernel's CTAs take work items from a
// counter in device memory. Each launch uses its own counter slot (rotating
// over kWorkSlots), set to a generation-tagged base on the launch's stream
// just before it; at most kWorkSlots launches may be in flight at once. A
// launch whose slot another launch re-arms while it runs detects it, stops
// and raises kErrSlotReuse in the status word (WorkCounter in common.cuh).
constexpr int kWorkSlots = 256;
// Arms a fresh counter slot on ctx.stream for a launch of n_items items.
cudaError_t next_work_counter(const LaunchCtx& ctx, int n_items, WorkCounter* counter);

// Forward, bf16, tcgen05 tensor cores (fwd_tc.cu). Modes: see AttnShape::mode.
cudaError_t launch_fwd_tc(const AttnShape& sh, const void* q, const void* k, const void* v,
                          void* o, float* lse, const LaunchCtx& ctx);
// Forward, fp32 FMA path (fwd_simt.cu).
cudaError_t launch_fwd_fp32(const AttnShape& sh, const float* q, const float* k, const float* v,
                            float* o, float* lse, const LaunchCtx& ctx);
// Backward, bf16 (bwd.cu). delta: Delta [B, H, S] fp32, computed here from o
// and dout; with mode 2 (one ring step of `rank` against `owner`'s block, the
// q-side arrays holding the rank's L rows and the k-side ones the block's) it
// is an input, o is not read, and dq, dk, dv are added to. sh.deterministic
// picks the kernels (see AttnShape).
cudaError_t launch_bwd(const AttnShape& sh, const void* q, const void* k, const void* v,
                       const void* o, const float* lse, const void* dout, float* dq, float* dk,
                       float* dv, float* delta, const LaunchCtx& ctx);
// Delta = rowsum(dO * O) over `rows` rows of D; o bf16 or (o_fp32) float32.
cudaError_t launch_bwd_delta(const void* o, int o_fp32, const void* dout, float* delta,
                             int64_t rows, int D, const LaunchCtx& ctx);

// Layout kernels (layout.cu).
struct PermuteTensor {
    const void* src;
    void* dst;
    int heads;
};
cudaError_t launch_ulysses_permute(const PermuteTensor* t, int ntensors, int B, int S, int D,
                                   int elem_bytes, int head_to_seq, const LaunchCtx& ctx);
// Ulysses exchange buffer <-> one device's tensors (layout.cu): buf holds U
// chunks, each the tensors' parts [B, s, heads / U, D] one after another.
// pack: tensors -> buf; else buf -> tensors. head_side: the tensors are the
// device's head shards [B, heads / U, U * s, D], else its sequence shards
// [B, s, heads, D].
struct UlyTensor {
    const void* tensor;
    int heads;
};
cudaError_t launch_ulysses_exchange(const UlyTensor* t, int ntensors, void* buf, int B, int s,
                                    int D, int U, int elem_bytes, int pack, int head_side,
                                    const LaunchCtx& ctx);
cudaError_t launch_seq_reorder(const void* src, void* dst, int BH, int S, int D, int P,
                               int zigzag, int to_natural, int elem_bytes, const LaunchCtx& ctx);
cudaError_t launch_lse_merge(float* o_acc, float* lse_acc, const float* o_part,
                             const float* lse_part, int64_t rows, int D, const LaunchCtx& ctx);
cudaError_t launch_watchdog_selftest(const LaunchCtx& ctx);
// Per-token bounds of packed documents into `table` (S int4); cu_dev holds
// n_docs + 1 checked boundaries in device memory.
cudaError_t launch_varlen_bounds(const int* cu_dev, int n_docs, int S, int causal, int window,
                                 void* table, const LaunchCtx& ctx);

}  // namespace rm
