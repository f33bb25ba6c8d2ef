/*
 * rm.h — C ABI of the B200 (sm_100a) blockwise ring attention library.
 *
 * What it computes. P virtual sequence-parallel ranks are simulated on one GPU.
 * Each rank keeps its query block fixed while the key/value blocks travel
 * around the ring ("Sequence Parallelism III: Ring Attention for Context That
 * Does Not Fit", duoan.github.io LLM tag index). Every step runs a flash-style
 * tile pass (QK^T, causal mask, online softmax, PV). Its partial output and
 * log-sum-exp fold into a running (O, LSE) pair by max-shifted exponential
 * weights ("DeDLOC Guide: Decentralized Long-Context Attention", section 3,
 * Online Softmax Rescaling Across Decentralized Ranks; Step 3, the local step
 * and the merge). The ring's block rotation is HBM block indexing: at step t
 * rank i reads the key/value block of owner (i - t) mod P.
 *
 * Conventions for every entry point:
 *   - All tensor arguments are DEVICE pointers owned by the caller; the library
 *     never allocates device memory and keeps no pointer after it returns.
 *   - Calls are asynchronous on `stream` (0 = legacy default stream). Inputs
 *     must stay valid, and outputs untouched, until the stream reaches the work.
 *   - Tensors are dense row-major. Attention tensors are [B, heads, S, D] with
 *     the S axis RANK-MAJOR: rank 0's L = S/P tokens, then rank 1's, and so
 *     on, each rank's tokens in its local chunk order (see rm_order).
 *   - Host-side validation runs before any launch; on RM_ERR_INVALID_ARG or
 *     RM_ERR_UNSUPPORTED nothing is launched and nothing is written.
 *   - Empty problems (B == 0 or S == 0, rows == 0) are valid and do nothing.
 *   - Pointers must be 16-byte aligned (TMA and vector access).
 *   - A launch failure returns RM_ERR_CUDA; rm_last_cuda_error() then gives the
 *     cudaError_t of the calling thread's last failure.
 *   - Every wait inside a kernel is bounded (see rm_set_watchdog_ns). A wait that
 *     runs out makes the kernel stop early, write nothing further and set a
 *     device status word that rm_check_device_status() reports as
 *     RM_ERR_TIMEOUT. Outputs of such a call are undefined.
 *   - Launches in flight. The attention kernels (forward, backward and their
 *     step variants) are persistent: their blocks take work items from a
 *     counter in device memory. The library keeps 256 such counters per
 *     device and gives each launch the next one in turn, re-armed on the
 *     launch's stream just before it. So at most 256 of these launches may be
 *     in flight at once on a device (on any streams). A CUDA graph that
 *     captured a launch keeps that launch's counter: replays of one graph must
 *     not overlap each other, and a replay must not overlap the 256th eager
 *     launch after the capture. A launch whose counter is re-armed by another
 *     one while it runs notices it, stops taking work and sets the status word,
 *     which rm_check_device_status() reports as RM_ERR_SLOT_REUSE; the outputs
 *     of both launches are then undefined. (Overlapping replays of one graph
 *     re-arm with the same value and cannot be told apart.)
 */
#ifndef RM_H
#define RM_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define RM_API __attribute__((visibility("default")))
#else
#define RM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum rm_status {
    RM_OK = 0,
    RM_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad enum, misalignment */
    RM_ERR_UNSUPPORTED = 2,  /* valid request outside the shapes/dtypes built */
    RM_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
    RM_ERR_TIMEOUT = 4,      /* a bounded in-kernel wait ran out */
    RM_ERR_SLOT_REUSE = 5,   /* more launches in flight than work-counter slots */
    RM_ERR_SMEM_LAYOUT = 6   /* a kernel's shared-memory layout did not fit its block */
} rm_status;

/* Token order of the ring ("context parallelism", Last Dictionary: causal
 * imbalance is handled by reordering chunks; axolotl-ringmaster README,
 * Layout: balancers.py head_tail/contiguous index generation).
 *   CONTIGUOUS: rank i holds natural tokens [i*L, (i+1)*L), L = S/P.
 *   ZIGZAG:     the sequence is cut into 2P chunks of c = S/(2P); rank i holds
 *               chunk i followed by chunk 2P-1-i (balances causal work). */
typedef enum rm_order { RM_ORDER_CONTIGUOUS = 0, RM_ORDER_ZIGZAG = 1 } rm_order;

typedef enum rm_dtype { RM_DTYPE_BF16 = 0, RM_DTYPE_FP32 = 1 } rm_dtype;

typedef enum rm_permute_dir { RM_SEQ_TO_HEAD = 0, RM_HEAD_TO_SEQ = 1 } rm_permute_dir;

typedef enum rm_reorder_dir {
    RM_NATURAL_TO_RANK_MAJOR = 0,
    RM_RANK_MAJOR_TO_NATURAL = 1
} rm_reorder_dir;

/*
 * rm_ring_attn_fwd — ring attention forward over P virtual ranks.
 *
 * Follows "DeDLOC Guide", Step 3 (scores = scale * Q K^T, LSE = logsumexp over
 * keys, O = softmax * V) run blockwise with the online-softmax merge of
 * section 3, and the Best Practices table's "Causal Mask Handling" (whole
 * masked blocks are skipped). Causal visibility uses GLOBAL token positions:
 * key j is visible to query i iff pos(j) <= pos(i) (diagonal included).
 *
 *   q    [B, H,   S, D]  dtype            (rank-major S)
 *   k, v [B, Hkv, S, D]  dtype; query head h reads KV head h / (H/Hkv)
 *   o    [B, H,   S, D]  dtype, written
 *   lse  [B, H,   S]     float32, written: natural log of sum_j exp(scale*q.k_j)
 *   scale > 0 (usually 1/sqrt(D)).
 *
 * Supported: dtype BF16 (tensor cores, fp32 accumulation) or FP32 (exact fp32
 * FMA path); D in {64, 128}; H % Hkv == 0; P >= 1; ZIGZAG needs S % (2P*128)
 * == 0, CONTIGUOUS needs S % (P*256) == 0 (for FP32: S % (2P*64) == 0 and
 * S % (P*64) == 0 respectively). Other shapes return RM_ERR_UNSUPPORTED.
 */
RM_API rm_status rm_ring_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int H, int Hkv, int S, int D, int P, int causal,
                           rm_order order, rm_dtype dtype, float scale, cudaStream_t stream);

/*
 * rm_allgather_attn_fwd — the all-gather alternative to the ring (forward).
 *
 * The axolotl-ringmaster README (Benchmark section) offers two ways to bring
 * every rank's keys to its queries: the p2p ring (O(S/P) keys resident per
 * rank) and an "allgather" rotater that collects all keys first (faster, more
 * memory). This is the second: each rank's queries attend, in one pass in
 * position order, to the keys of all ranks gathered into natural token order.
 * The result is the same attention as rm_ring_attn_fwd (up to fp32 rounding
 * order).
 *
 *   q            [B, H,   S, D]  BF16, rank-major S (each rank's shard, as for
 *                                the ring)
 *   k_all, v_all [B, Hkv, S, D]  BF16, NATURAL token order: the gathered keys
 *                                (rm_seq_reorder RANK_MAJOR_TO_NATURAL of the
 *                                rank-major k and v forms them on one device)
 *   o, lse       as rm_ring_attn_fwd (rank-major S)
 *   P, order     the layout of q, o and lse.
 *
 * Shapes and validation as rm_ring_attn_fwd. FP32 returns RM_ERR_UNSUPPORTED.
 */
RM_API rm_status rm_allgather_attn_fwd(const void* q, const void* k_all, const void* v_all,
                                       void* o, float* lse, int B, int H, int Hkv, int S, int D,
                                       int P, int causal, rm_order order, rm_dtype dtype,
                                       float scale, cudaStream_t stream);

/*
 * rm_ring_attn_fwd_step — one ring step of one rank, for a ring whose ranks
 * are separate devices.
 *
 * "DeDLOC Guide", Step 3 (the local step) and section 3 (the online-softmax
 * merge of step partials); "Sequence Parallelism III: Ring Attention"
 * (duoan.github.io): rank `rank` keeps its queries and at each step attends to
 * the K/V block it holds, which at step t belongs to owner (rank - t) mod P;
 * the block then moves on to rank + 1. This call computes that step's partial:
 * softmax attention of the rank's queries over the owner's keys only, with the
 * causal mask on GLOBAL positions (as rm_ring_attn_fwd). The caller folds the
 * partials of the P steps with rm_lse_merge, in any order.
 *
 *   q_local      [B, H,   L, D]  BF16: rank `rank`'s L = S / P query rows, in
 *                                its local chunk order (the rank's slice of the
 *                                rank-major layout)
 *   k_block,
 *   v_block      [B, Hkv, L, D]  BF16: owner `owner`'s L rows, local order
 *   o_part       [B, H,   L, D]  float32, written: the partial, normalised over
 *                                the visible keys of this block
 *   lse_part     [B, H,   L]     float32, written: natural log of the partial
 *                                sum; a row that sees no key of the block gets
 *                                O = 0, LSE = -inf (the identity of the merge)
 *   S, P, order  the global layout (S = P * L); 0 <= rank, owner < P.
 *
 * Shapes and validation as rm_ring_attn_fwd (S, P and order describe the whole
 * sequence). FP32 returns RM_ERR_UNSUPPORTED.
 */
RM_API rm_status rm_ring_attn_fwd_step(const void* q_local, const void* k_block,
                                       const void* v_block, float* o_part, float* lse_part, int B,
                                       int H, int Hkv, int S, int D, int P, int rank, int owner,
                                       int causal, rm_order order, rm_dtype dtype, float scale,
                                       cudaStream_t stream);

/*
 * rm_ring_attn_fwd_step_merge — rm_ring_attn_fwd_step folded straight into the
 * rank's running (O, LSE) pair, so that no partial is written.
 *
 * "DeDLOC Guide", section 3 (the alpha/beta rescaling of step partials) and
 * Step 3: with a = lse_acc and b the step's LSE, M = max(a, b),
 *   O_acc <- (e^(a-M) O_acc + e^(b-M) O_step) / (e^(a-M) + e^(b-M)),
 *   lse_acc <- M + ln(e^(a-M) + e^(b-M)).
 * The same result as rm_ring_attn_fwd_step followed by rm_lse_merge (up to
 * fp32 rounding order), in one launch and without the partial's round trip
 * through memory.
 *
 *   q_local, k_block, v_block, B..order, dtype, scale : as rm_ring_attn_fwd_step
 *   o_acc   [B, H, L, D] float32, read and written: the running output
 *   lse_acc [B, H, L]    float32, read and written: the running LSE
 * Start a ring with o_acc = 0 and lse_acc = -inf (the empty pair) and call this
 * once per step, in any order of owners. Rows that see no key of the block keep
 * their pair unchanged. After the P steps of a rank, (o_acc, lse_acc) is its
 * attention output and LSE. Shapes and validation as rm_ring_attn_fwd_step.
 */
RM_API rm_status rm_ring_attn_fwd_step_merge(const void* q_local, const void* k_block,
                                             const void* v_block, float* o_acc, float* lse_acc,
                                             int B, int H, int Hkv, int S, int D, int P, int rank,
                                             int owner, int causal, rm_order order,
                                             rm_dtype dtype, float scale, cudaStream_t stream);

/*
 * rm_ring_attn_fwd_window — rm_ring_attn_fwd with a causal sliding window.
 *
 * The axolotl-ringmaster README's Status table (phase 4) lists sliding-window
 * attention, passed to flash attention as its `window`. Here the window counts
 * keys: query at global position i sees keys j with i - window < j <= i, that
 * is itself and the window - 1 keys before it (flash's left window of
 * window - 1, right window 0). Positions are global, as for the causal mask,
 * so the result does not depend on P or the chunk order.
 *
 *   Arguments and layouts as rm_ring_attn_fwd, with the mask always causal.
 *   window >= 1; window >= S gives plain causal attention. window < 1 returns
 *   RM_ERR_INVALID_ARG; S >= 2^30 with a window below S returns
 *   RM_ERR_UNSUPPORTED.
 *   Key tiles outside every row's window are skipped, so the work grows with
 *   S * window instead of S^2 / 2.
 */
RM_API rm_status rm_ring_attn_fwd_window(const void* q, const void* k, const void* v, void* o,
                                         float* lse, int B, int H, int Hkv, int S, int D, int P,
                                         int window, rm_order order, rm_dtype dtype, float scale,
                                         cudaStream_t stream);

/*
 * rm_varlen_bounds_size / rm_varlen_bounds — the per-token visibility table of
 * packed variable-length documents (axolotl-ringmaster README, Status table:
 * packing / varlen).
 *
 * The S tokens (natural order) are the concatenation of n_docs documents with
 * boundaries cu_seqlens[0] = 0 <= cu_seqlens[1] <= ... <= cu_seqlens[n_docs] =
 * S (empty documents allowed). A query sees only keys of its own document,
 * and within it keys j <= i when causal, and j > i - window when window > 0
 * (causal only; window >= S means none). The ring layout (contiguous or
 * zigzag) shards the packed sequence as one sequence; masks use global
 * positions, so results do not depend on P or the order.
 *
 *   cu_seqlens : HOST int32 array of n_docs + 1 boundaries, checked on the host
 *                (RM_ERR_INVALID_ARG if it does not rise from 0 to S)
 *   bounds     : device buffer of at least rm_varlen_bounds_size(S, n_docs)
 *                bytes, 256-byte aligned, owned by the caller. It receives one
 *                int4 per token {lo, hi, imin, imax}: query i sees keys
 *                lo..hi, key j is seen by queries imin..imax (natural
 *                positions), followed by a copy of cu_seqlens.
 * The host array may be reused as soon as the call returns. Build the table
 * once per batch layout and pass it to every rm_ring_attn_*_varlen call with
 * the same S (each batch row uses the same documents).
 */
RM_API size_t rm_varlen_bounds_size(int S, int n_docs);

RM_API rm_status rm_varlen_bounds(const int* cu_seqlens, int n_docs, int S, int causal,
                                  int window, void* bounds, size_t bounds_bytes,
                                  cudaStream_t stream);

/*
 * rm_ring_attn_fwd_varlen — rm_ring_attn_fwd over packed documents.
 *
 * Arguments, layouts and shape rules as rm_ring_attn_fwd; the mask (causal or
 * not, window, documents) comes from `bounds`, a table made by
 * rm_varlen_bounds for this S. Key tiles no query row can see (other
 * documents, before a window) are skipped, so the work follows the documents'
 * lengths.
 */
RM_API rm_status rm_ring_attn_fwd_varlen(const void* q, const void* k, const void* v, void* o,
                                         float* lse, const void* bounds, int B, int H, int Hkv,
                                         int S, int D, int P, rm_order order, rm_dtype dtype,
                                         float scale, cudaStream_t stream);

/*
 * rm_ring_attn_bwd — gradients of L = sum(dO * O) through the ring forward
 * (axolotl-ringmaster README: flash-style reverse-ring backward; gradients
 * accumulate in fp32 across ring steps).
 *
 * With P_ij = exp(scale*q_i.k_j - LSE_i) over visible keys and
 * Delta_i = <dO_i, O_i>: dV_j = sum_i P_ij dO_i, dS_ij = P_ij (<dO_i, v_j> -
 * Delta_i), dQ_i = scale sum_j dS_ij k_j, dK_j = scale sum_i dS_ij q_i; a KV
 * head's dK/dV sum over the query heads that share it.
 *
 *   q, k, v, o, dout : as in the forward (dtype; o is the forward's output)
 *   lse              : [B, H, S] float32 from the forward
 *   dq [B,H,S,D], dk, dv [B,Hkv,S,D] : float32, every element overwritten
 *                      (no atomics: each is written exactly once)
 *   workspace        : device scratch of at least
 *                      rm_ring_attn_bwd_workspace_size(B, H, S) bytes, 256-byte
 *                      aligned, owned by the caller, contents need not be set
 *                      (it receives Delta = rowsum(dO * O), [B, H, S] fp32).
 * Supported: dtype BF16, D in {64, 128}, same shape rules as the forward.
 */
RM_API size_t rm_ring_attn_bwd_workspace_size(int B, int H, int S);

RM_API rm_status rm_ring_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                           const float* lse, const void* dout, float* dq, float* dk,
                           float* dv, void* workspace, size_t workspace_bytes, int B, int H,
                           int Hkv, int S, int D, int P, int causal, rm_order order,
                           rm_dtype dtype, float scale, cudaStream_t stream);

/*
 * rm_ring_attn_bwd_window — rm_ring_attn_bwd through rm_ring_attn_fwd_window:
 * the same gradients with P_ij = 0 outside the window (query i, keys
 * i - window < j <= i). Arguments, layouts, workspace, outputs and status codes
 * as rm_ring_attn_bwd; window rules as rm_ring_attn_fwd_window. o and lse must
 * come from the windowed forward with the same window.
 */
RM_API rm_status rm_ring_attn_bwd_window(const void* q, const void* k, const void* v,
                                         const void* o, const float* lse, const void* dout,
                                         float* dq, float* dk, float* dv, void* workspace,
                                         size_t workspace_bytes, int B, int H, int Hkv, int S,
                                         int D, int P, int window, rm_order order,
                                         rm_dtype dtype, float scale, cudaStream_t stream);

/*
 * rm_ring_attn_bwd_varlen — rm_ring_attn_bwd through rm_ring_attn_fwd_varlen:
 * the same gradients with P_ij = 0 for pairs the documents' mask hides.
 * Arguments, layouts, workspace, outputs and status codes as rm_ring_attn_bwd;
 * `bounds` as for the forward (the same table the forward used).
 */
RM_API rm_status rm_ring_attn_bwd_varlen(const void* q, const void* k, const void* v,
                                         const void* o, const float* lse, const void* dout,
                                         float* dq, float* dk, float* dv, const void* bounds,
                                         void* workspace, size_t workspace_bytes, int B, int H,
                                         int Hkv, int S, int D, int P, rm_order order,
                                         rm_dtype dtype, float scale, cudaStream_t stream);

/*
 * rm_ring_attn_bwd_noalloc — rm_ring_attn_bwd for callers that cannot allocate.
 *
 * The pages have no counterpart of this call; it serves library users. Some
 * callers of this code cannot call cudaMalloc: a plugin inside a host
 * framework that reserved all device memory up front and hands out only the
 * tensors themselves, or a latency-critical loop where an allocation (which
 * may synchronise the device or fail) is not allowed. This entry point takes
 * the same tensors as rm_ring_attn_bwd but no workspace: its scratch (the
 * Delta rows) lives in a static device array of the library that holds
 * 2,097,152 fp32 values (8 MiB). Every GPU that loads the library keeps that
 * array until the process exits.
 *
 *   Arguments, layouts, outputs and status codes as rm_ring_attn_bwd.
 *   Limit: B * H * S <= 2,097,152; larger problems return RM_ERR_UNSUPPORTED
 *   before anything is launched.
 *   The first call on a device looks up the array's device address (a CUDA
 *   runtime query, no allocation); make that first call before any stream
 *   capture begins on that device.
 *   All calls on a device share the one array, which keeps the last call's
 *   contents. The backward rewrites the whole scratch it reads, so nothing
 *   has to be cleared, but calls that overlap on the GPU (for example on two
 *   streams) race on it and give undefined results: serialise them.
 *   Nothing is allocated: no cudaMalloc, no cudaFree, no allocating library
 *   routine.
 */
RM_API rm_status rm_ring_attn_bwd_noalloc(const void* q, const void* k, const void* v,
                                          const void* o, const float* lse, const void* dout,
                                          float* dq, float* dk, float* dv, int B, int H, int Hkv,
                                          int S, int D, int P, int causal, rm_order order,
                                          rm_dtype dtype, float scale, cudaStream_t stream);

/*
 * rm_ring_attn_bwd_delta — Delta_i = <dO_i, O_i> (fp32) for rows of D values:
 * the per-row term of the backward's dS_ij = P_ij (<dO_i, v_j> - Delta_i)
 * (the gradient stated at rm_ring_attn_bwd). A rank of a ring across devices
 * computes it once for its own rows and passes it to every
 * rm_ring_attn_bwd_step of the backward.
 *
 *   o     [rows, D] o_dtype (BF16, or FP32 as rm_ring_attn_fwd_step_merge
 *                   accumulates it)
 *   dout  [rows, D] BF16
 *   delta [rows]    float32, written
 * D in {64, 128} (else RM_ERR_UNSUPPORTED); rows >= 0.
 */
RM_API rm_status rm_ring_attn_bwd_delta(const void* o, const void* dout, float* delta,
                                        int64_t rows, int D, rm_dtype o_dtype,
                                        cudaStream_t stream);

/*
 * rm_ring_attn_bwd_step — one step of the backward of a ring whose ranks are
 * separate devices (axolotl-ringmaster README, Benchmark section: the p2p
 * rotater's flash-style reverse-ring backward, gradients accumulated in fp32
 * across ring steps).
 *
 * The gradients of rm_ring_attn_bwd restricted to the pairs (query of rank
 * `rank`, key of owner `owner`'s block): rank `rank` holds its queries and the
 * block of `owner`, and this call ADDS
 *   dq_local += scale sum_{j in block} dS_ij k_j      (the rank's rows)
 *   dk_block += scale sum_{i of rank} dS_ij q_i       (the block's rows)
 *   dv_block +=       sum_{i of rank} P_ij dO_i
 * with P_ij = exp(scale q_i.k_j - LSE_i) over the pairs the causal mask (global
 * positions) leaves visible. Over the P steps a rank's dq_local collects every
 * owner's part, and a block's dk/dv, travelling with it, every rank's part.
 *
 *   q_local, dout_local [B, H, L, D]  BF16, the rank's rows (local order)
 *   lse_local           [B, H, L]     float32, the rank's final forward LSE
 *   delta_local         [B, H, L]     float32, rm_ring_attn_bwd_delta of the
 *                                     rank's O and dO
 *   k_block, v_block    [B, Hkv, L, D] BF16, owner `owner`'s rows
 *   dq_local            [B, H, L, D]  float32, read and written
 *   dk_block, dv_block  [B, Hkv, L, D] float32, read and written
 *   S, P, rank, owner, causal, order, scale : as rm_ring_attn_fwd_step
 * Zero the three gradient arrays before the first step. Tiles that see nothing
 * of the other side are not touched; every element is updated by one thread
 * per call, so the sums are deterministic. Shapes and validation as
 * rm_ring_attn_bwd (BF16, D in {64, 128}).
 */
RM_API rm_status rm_ring_attn_bwd_step(const void* q_local, const void* k_block,
                                       const void* v_block, const float* lse_local,
                                       const float* delta_local, const void* dout_local,
                                       float* dq_local, float* dk_block, float* dv_block, int B,
                                       int H, int Hkv, int S, int D, int P, int rank, int owner,
                                       int causal, rm_order order, rm_dtype dtype, float scale,
                                       cudaStream_t stream);

/*
 * rm_lse_merge — fold one partial (O, LSE) into a running pair, row by row,
 * in place ("DeDLOC Guide", section 3 alpha/beta rescaling, in the
 * normalised-output form of Step 3's merge):
 *   M = max(a, b); if M = -inf: O = 0, LSE = -inf (empty + empty);
 *   else wa = exp(a - M), wb = exp(b - M),
 *        O = (wa O_acc + wb O_part) / (wa + wb), LSE = M + ln(wa + wb).
 *   o_acc [rows, D] f32 (in/out), lse_acc [rows] f32 (in/out),
 *   o_part [rows, D] f32, lse_part [rows] f32. D >= 1, rows >= 0.
 */
RM_API rm_status rm_lse_merge(float* o_acc, float* lse_acc, const float* o_part, const float* lse_part,
                       int64_t rows, int D, cudaStream_t stream);

/*
 * rm_ulysses_permute — the DeepSpeed-Ulysses all-to-all as a layout transform
 * on one device ("Sequence Parallelism II: DeepSpeed Ulysses and All-to-All
 * Attention", duoan.github.io LLM tag index: before the exchange every rank
 * has all heads for a subset of tokens, after it all tokens for a subset of
 * heads; axolotl-ringmaster README: Ulysses is capped by the KV-head count).
 *
 * Mesh: U Ulysses ranks x R ring ranks; shard n = r*U + u holds tokens
 * [n*S/(U R), (n+1)*S/(U R)) of the rank-major sequence.
 *   SEQ_TO_HEAD: src [B, S, Hx, D] (= [B, U*R shards, S/(U R), Hx, D]) ->
 *                dst [B, Hx, S, D]; device (r, u)'s share afterwards is heads
 *                [u*Hx/U, (u+1)*Hx/U) x tokens [r*S/R, (r+1)*S/R).
 *   HEAD_TO_SEQ: the exact inverse.
 * Requires Hx % U == 0, S % (U*R) == 0, elem_bytes in {1, 2, 4, 8}.
 * Bit-exact data movement.
 */
RM_API rm_status rm_ulysses_permute(const void* src, void* dst, int B, int S, int Hx, int D, int U,
                             int R, int elem_bytes, rm_permute_dir dir, cudaStream_t stream);

/* As rm_ulysses_permute for Q (H heads) and K, V (Hkv heads) in ONE launch
 * (axolotl-ringmaster README: the Ulysses leg fuses K/V into one exchange).
 * Requires H % U == 0, Hkv % U == 0 (so U <= Hkv). */
RM_API rm_status rm_ulysses_permute_qkv(const void* q_src, const void* k_src, const void* v_src,
                                 void* q_dst, void* k_dst, void* v_dst, int B, int S, int H,
                                 int Hkv, int D, int U, int R, int elem_bytes,
                                 rm_permute_dir dir, cudaStream_t stream);

/*
 * rm_ulysses_buffer_size / rm_ulysses_pack / rm_ulysses_unpack — one device's
 * side of the DeepSpeed-Ulysses all-to-all when the U devices of a Ulysses
 * group are separate GPUs ("Sequence Parallelism II: DeepSpeed Ulysses and
 * All-to-All Attention": before the exchange a device has all heads of its
 * tokens, after it all tokens of its heads; axolotl-ringmaster README: the
 * Ulysses leg exchanges K and V together, and Ulysses is capped by the
 * KV-head count).
 *
 * Device u of the group holds s = S_group / U consecutive tokens (its
 * sequence shard). The exchange buffer is U equal chunks, chunk u' for
 * (pack) or from (unpack) device u'; a collective all-to-all with equal
 * splits (ncclSend/ncclRecv pairs, torch.distributed.all_to_all_single) moves
 * chunk u' of every device to device u'. Inside a chunk the tensors follow
 * one another, tensor x as [B, s, heads[x] / U, D]: the sender's s tokens of
 * the receiver's heads. Up to three tensors (Q, K, V; or O alone) share one
 * buffer, so one collective moves them all.
 *   sequence shard of tensor x: [B, s, heads[x], D]        (device's tokens)
 *   head shard of tensor x:     [B, heads[x]/U, U*s, D]    (device's heads,
 *       token u'*s + t = token t of device u', i.e. the group's tokens in order)
 * Device u's head shard holds heads [u*heads/U, (u+1)*heads/U).
 *
 *   rm_ulysses_pack   SEQ_TO_HEAD: tensors = sequence shards -> send_buf
 *                     HEAD_TO_SEQ: tensors = head shards     -> send_buf
 *   rm_ulysses_unpack SEQ_TO_HEAD: recv_buf -> tensors = head shards
 *                     HEAD_TO_SEQ: recv_buf -> tensors = sequence shards
 * So pack(SEQ_TO_HEAD), all-to-all, unpack(SEQ_TO_HEAD) turns every device's
 * sequence shard into its head shard, and the HEAD_TO_SEQ pair undoes it.
 *
 *   tensors, heads : HOST arrays of ntensors (1..3) device pointers and head
 *                    counts; heads[x] % U == 0
 *   send_buf / recv_buf : device buffer of rm_ulysses_buffer_size(heads,
 *                    ntensors, B, s, D, elem_bytes) bytes, not overlapping any
 *                    tensor, 16-byte aligned like every pointer here
 *   elem_bytes in {1, 2, 4, 8}. Bit-exact data movement (HBM-bound).
 * rm_ulysses_buffer_size returns 0 for invalid arguments.
 */
RM_API size_t rm_ulysses_buffer_size(const int* heads, int ntensors, int B, int s, int D,
                                     int elem_bytes);

RM_API rm_status rm_ulysses_pack(const void* const* tensors, const int* heads, int ntensors,
                                 void* send_buf, int B, int s, int D, int U, int elem_bytes,
                                 rm_permute_dir dir, cudaStream_t stream);

RM_API rm_status rm_ulysses_unpack(const void* recv_buf, void* const* tensors, const int* heads,
                                   int ntensors, int B, int s, int D, int U, int elem_bytes,
                                   rm_permute_dir dir, cudaStream_t stream);

/*
 * rm_seq_reorder — natural token order <-> rank-major ring order along S.
 *   src, dst [B, H, S, D] elements of elem_bytes each (D = 1 for LSE).
 *   NATURAL_TO_RANK_MAJOR: dst[.., s, :] = src[.., pos(s), :]
 *   RANK_MAJOR_TO_NATURAL: dst[.., pos(s), :] = src[.., s, :]
 * pos(s) as in rm_order. Requires S % P == 0 (contiguous) or S % (2P) == 0
 * (zigzag). src and dst must not overlap. Bit-exact.
 */
RM_API rm_status rm_seq_reorder(const void* src, void* dst, int B, int H, int S, int D, int P,
                         rm_order order, rm_reorder_dir dir, int elem_bytes,
                         cudaStream_t stream);

/* Synchronises `stream`, then reads and clears the device status word of the
 * current device. Returns RM_ERR_SLOT_REUSE if a launch found its work counter
 * re-armed by another launch since the last check, else RM_ERR_SMEM_LAYOUT if
 * a launch found its dynamic shared memory placed too far from a 1024-byte
 * boundary for its layout (it then returned at once, having written nothing;
 * only the fused backward checks this, and it has not been seen on sm_100a),
 * else RM_ERR_TIMEOUT if a bounded wait ran out, RM_ERR_CUDA if the
 * synchronisation failed, else RM_OK. */
RM_API rm_status rm_check_device_status(cudaStream_t stream);

/* Limit for every in-kernel wait, in nanoseconds (default 2e9). Applies to
 * launches made after the call; values below 1000 are raised to 1000. */
RM_API void rm_set_watchdog_ns(uint64_t ns);

/* Which kernels the backward entry points (rm_ring_attn_bwd*, including the
 * window, varlen, no-alloc and step variants) use, process-wide, for calls
 * made after this one. 1 (the default): two kernels (KV-stationary dK/dV,
 * Q-stationary dQ) that write every gradient element exactly once, so the
 * result is bitwise reproducible. 0: one fused kernel that computes S and dP
 * once per tile pair (five tensor-core products instead of seven) and adds dQ
 * into place with fp32 reductions at L2 (TMA reduce-add); the order of those
 * additions varies between runs, so dQ may differ in its last bits from run
 * to run (dK and dV do not). On B200 the fused kernel is the faster of the
 * two, by about 10% on a 64k-token causal backward with the whole ring in
 * one call. */
RM_API void rm_set_bwd_deterministic(int on);
RM_API int rm_get_bwd_deterministic(void);

/* Launches one kernel that waits on a barrier nothing will complete, bounded
 * by timeout_ns, so that callers can see the watchdog path end in
 * RM_ERR_TIMEOUT (reported by rm_check_device_status) without a hang. */
RM_API rm_status rm_watchdog_selftest(uint64_t timeout_ns, cudaStream_t stream);

RM_API const char* rm_status_string(rm_status status);
RM_API int rm_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* RM_H */
