// Ring attention forward, bf16 in / fp32 accumulate, on the sm_100a tensor
// cores (tcgen05.mma with TMEM accumulators, TMA-staged tiles).
//
// What it computes ("DeDLOC Guide: Decentralized Long-Context Attention",
// Step 3 local step and section 3 online-softmax merge; "Sequence Parallelism
// III: Ring Attention ...", duoan.github.io): every query tile of virtual rank
// i keeps its block fixed and visits the key/value block of owner
// r = (i - t) mod P at ring step t = 0..P-1. Each visit is a flash tile pass
// S = Q K^T, causal mask on global positions, online softmax, O += P V. The
// running (m, l, O) simply continues across step boundaries, which is exactly
// the alpha/beta merge of the steps' (O, LSE) partials, done in registers and
// TMEM. Tiles the causal mask hides completely are never computed ("DeDLOC
// Guide", Best Practices, Causal Mask Handling).
//
// Block structure (persistent, one CTA per SM, 320 threads):
//   warps 0-3  softmax warpgroup for query tile 0, warps 4-7 for tile 1
//              (thread = one query row = one TMEM lane); they also write O/LSE
//   warp 8     MMA issuer (one thread)
//   warp 9     TMA producer (one thread)
// The two query tiles share every K/V tile: they are two heads of one GQA
// group at the same slots, or (odd group size) two consecutive 128-slot tiles
// of one head within one rank.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [384,384+D).
// P (bf16) overwrites the first 64 columns of its S tile and is the TMEM
// A-operand of the PV product. Issue order per key tile j:
//   PV0_j, QK0_{j+1}, PV1_j, QK1_{j+1}
// so the tensor pipe runs one tile's products while the other tile's softmax
// runs. O is rescaled only when a row maximum grows by more than 2^8 (in exp2
// units); the sum l uses the same reference maximum, so the result is exact.
//
// Three instantiations (kMode):
//   kRing      all P ranks' queries and all P steps in one launch (K/V of every
//              rank resident, rank-major).
//   kGathered  the all-gather variant (the "allgather" rotater of the
//              axolotl-ringmaster README, Benchmark section: faster, more
//              memory): K/V gathered from every rank into natural token order;
//              each query tile makes one pass over its visible key tiles.
//   kStep      one ring step of one rank, as a rank of a real multi-device ring
//              runs it: that rank's L local queries against one owner's L-token
//              K/V block. O (fp32, normalised over this block's keys) and LSE
//              are the step's partial; a row that sees none of the block gets
//              (0, -inf), the identity of the (O, LSE) merge. With `merge` set,
//              o and lse are instead the rank's running pair, and the epilogue
//              folds the partial into it ("DeDLOC Guide", section 3: weights
//              exp(a - M) and exp(b - M), M the larger LSE); rows that see none
//              of the block are left as they are.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tmap.h"

namespace rm {

namespace {

constexpr int kBM = 128;        // query rows per tile (UMMA M)
constexpr int kBN = 128;        // keys per tile (UMMA N of QK^T, K of PV)
constexpr int kStages = 4;      // K/V ring in shared memory (one tile per stage)
constexpr int kThreads = 320;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 of the largest stale-max factor
enum Mode : int { kRing = 0, kGathered = 1, kStep = 2 };

template <int D>
struct Cfg {
    static constexpr int kTileBytes = kBM * D * 2;  // one Q, K or V tile
    static constexpr int kBoxes = D / 64;           // 128-byte swizzle boxes along D
    static constexpr int kBoxBytes = kBM * 128;     // 16 KB
    static constexpr int kQOff = 0;
    static constexpr int kKVOff = 2 * kTileBytes;
    static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
    static constexpr int kSmemBytes = kBarOff + 512 + 1024;  // + barriers + alignment slack
};

struct TcArgs {
    CUtensorMap tm_q, tm_k, tm_v;
    void* o;
    float* lse;
    unsigned* status;
    WorkCounter work;  // this launch's work-item counter
    unsigned long long timeout_ns;
    int H, Hkv, S, P, causal, G;
    MaskSpec mk;       // which keys each query sees
    int head_pair;     // 1: tiles are heads (h, h+1) at one slot; 0: one head, slots s, s+128
    int head_major;    // item order: grouped by KV head (see decode_item)
    int n_units;       // query units per head unit
    int n_head_units;  // B * (head_pair ? H / 2 : H)
    int n_items;
    float scale, scale_log2;
    RingLayout lay;
    int q_len;         // rows per head of q, o, lse: S, or L for one step
    int q_slot0;       // global slot of their first row: 0, or rank * L for one step
    int kv_len;        // rows per head of k, v: S, or L for one step
    int owner;         // one step: the rank whose block k, v hold
    int merge;         // one step: o, lse are the running pair to fold into
};

struct Item {
    int b, h0, h1, g, slot0, slot1, pos0, pos1, rank;
};

// Work item w -> two query tiles, ordered by the natural position of their
// queries, latest first when causal (the most key tiles first).
//   head_major: items grouped by KV head (the head units that read one KV
//     head), positions inside a group, the group's head units innermost; the
//     CTAs running at one time then sweep the K/V of one KV head, which stays
//     in L2 (plain causal or full masks, where a query tile sweeps up to all S
//     keys and the K/V of every head would not fit).
//   otherwise: positions outermost, every head of a position adjacent (windows
//     and packed documents, where a position's keys are few, and one step).
// One step covers only the launching rank's slots, in slot order.
template <int kMode>
__device__ __forceinline__ Item decode_item(const TcArgs& a, int w) {
    Item it;
    int unit_rank, hu;
    if (a.head_major) {
        const int gu = a.head_pair ? a.G / 2 : a.G;  // head units per KV head
        const int per_group = a.n_units * gu;
        const int grp = w / per_group;
        const int rem = w - grp * per_group;
        unit_rank = rem / gu;
        hu = grp * gu + (rem - unit_rank * gu);
    } else {
        unit_rank = w / a.n_head_units;
        hu = w - unit_rank * a.n_head_units;
    }
    const int heads_per_b = a.head_pair ? a.H / 2 : a.H;
    it.b = hu / heads_per_b;
    const int hh = hu - it.b * heads_per_b;
    it.h0 = a.head_pair ? 2 * hh : hh;
    it.h1 = a.head_pair ? it.h0 + 1 : it.h0;
    it.g = it.h0 / a.G;
    const int U = a.head_pair ? kBM : 2 * kBM;
    const int nu = a.causal ? a.n_units - 1 - unit_rank : unit_rank;
    int slot;
    if (kMode == kStep)
        slot = a.q_slot0 + nu * U;
    else if (!a.lay.zigzag || a.lay.c % U == 0)
        slot = a.lay.slot_of_pos(nu * U);  // the unit is contiguous in slots too
    else
        slot = nu * U;                     // chunk of one tile: take slot order
    it.slot0 = slot;
    it.slot1 = a.head_pair ? slot : slot + kBM;
    it.pos0 = a.lay.pos_of_slot(it.slot0);
    it.pos1 = a.lay.pos_of_slot(it.slot1);
    it.rank = slot / a.lay.L;
    return it;
}

// Key tiles of an item in ring order: step t visits owner (rank - t) mod P.
// An owner's block is one run (contiguous order) or two runs (zigzag: chunk r
// then chunk 2P-1-r) of consecutive natural positions. The keys that either
// query tile can see form one interval [lo, hi] (the bounds are monotone), so
// the tiles to visit in each run are an interval too: O(1) work per tile
// returned, no division. kpos holds the natural position of the tile last
// returned.
//
// Gathered variant: the keys are one run of all S positions in natural order
// (slot = position), visited once. One step: the runs of the owner's block
// only; kslot is then the row within the block.
template <int kMode>
struct KvIter {
    int rank, lo, hi, t, run, u, u_end, s0, p0, kpos;
    __device__ __forceinline__ KvIter(const TcArgs& a, const Item& it)
        : rank(it.rank), t(0), run(-1), u(0), u_end(0), s0(0), p0(0), kpos(0) {
        lo = min(row_bounds(a.mk, it.pos0).x, row_bounds(a.mk, it.pos1).x);
        hi = max(row_bounds(a.mk, it.pos0 + kBM - 1).y, row_bounds(a.mk, it.pos1 + kBM - 1).y);
    }
    // `a` is the kernel's parameter block itself
    __device__ __forceinline__ bool next(const TcArgs& a, int& kslot) {
        const RingLayout& lay = a.lay;
        if constexpr (kMode == kStep) {
            while (u >= u_end) {
                const int runs = lay.zigzag ? 2 : 1;
                if (run + 1 >= runs) {  // run starts at -1; stays at runs once done
                    run = runs;
                    return false;
                }
                ++run;
                const int r = a.owner;
                const int ctiles = (lay.zigzag ? lay.c : lay.L) / kBN;
                s0 = run * lay.c;
                p0 = lay.zigzag ? (run == 0 ? r * lay.c : (2 * lay.P - 1 - r) * lay.c) : r * lay.L;
                u = max(0, ceil_div128(lo - (kBN - 1) - p0));
                u_end = min(ctiles, max(((hi - p0) >> 7) + 1, 0));
            }
            kpos = p0 + u * kBN;
            kslot = s0 + u * kBN;
            ++u;
            return true;
        } else if constexpr (kMode == kGathered) {
            if (u >= u_end) {
                if (run >= 0) return false;  // run starts at -1: one run only
                run = 0;
                s0 = p0 = 0;
                u = max(0, ceil_div128(lo - (kBN - 1)));
                u_end = min(lay.S / kBN, max((hi >> 7) + 1, 0));
                if (u >= u_end) return false;
            }
            kpos = kslot = u * kBN;
            ++u;
            return true;
        } else {
            while (u >= u_end) {
                const int runs = lay.zigzag ? 2 : 1;
                if (++run == runs) {  // run starts at -1, so the first call opens run 0 of step 0
                    run = 0;
                    if (++t == lay.P) return false;
                }
                const int r = lay.owner(rank, t);
                const int ctiles = (lay.zigzag ? lay.c : lay.L) / kBN;
                s0 = r * lay.L + run * lay.c;
                p0 = lay.zigzag ? (run == 0 ? r * lay.c : (2 * lay.P - 1 - r) * lay.c) : r * lay.L;
                // tiles whose keys meet [lo, hi]: p0 + 128 u <= hi and p0 + 128 u + 127 >= lo
                u = max(0, ceil_div128(lo - (kBN - 1) - p0));
                u_end = min(ctiles, max(((hi - p0) >> 7) + 1, 0));
            }
            kpos = p0 + u * kBN;
            kslot = s0 + u * kBN;
            ++u;
            return true;
        }
    }
};

constexpr int kItemReaders = 9;  // the MMA thread and one lane of each softmax warp

struct Bars {
    ItemRing items;  // work items claimed by the producer (dynamic distribution)
    uint64_t q_full, q_empty, drain;
    uint64_t kv_full[kStages], kv_empty[kStages];
    uint64_t s_full[2], p_full[2], o_full[2];
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block");

template <int D>
__device__ __forceinline__ void issue_qk(uint32_t tmem_s, uint32_t q_smem, uint32_t k_smem) {
    constexpr uint32_t idesc = umma_idesc_bf16(kBM, kBN, 0, 0);
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * Cfg<D>::kBoxBytes + (k & 3) * 32;
        umma_ss(tmem_s, umma_desc_sw128(q_smem + off, 16, 1024),
                umma_desc_sw128(k_smem + off, 16, 1024), idesc, k > 0 ? 1u : 0u);
    }
}

template <int D>
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint32_t v_smem,
                                         bool accumulate) {
    constexpr uint32_t idesc = umma_idesc_bf16(kBM, D, 0, 1);
#pragma unroll
    for (int k = 0; k < kBN / 16; ++k)
        umma_ts(tmem_o, tmem_p + 8 * k,
                umma_desc_sw128(v_smem + k * 2048, Cfg<D>::kBoxBytes, 1024), idesc,
                (accumulate || k > 0) ? 1u : 0u);
}

template <int D, int kMode>
__global__ void __launch_bounds__(kThreads, 1) ring_fwd_tc_kernel(const __grid_constant__ TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    Bars& bars = *reinterpret_cast<Bars*>(smem + Cfg<D>::kBarOff);
    const uint32_t q_smem = smem_u32(smem + Cfg<D>::kQOff);
    const uint32_t kv_smem = smem_u32(smem + Cfg<D>::kKVOff);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        bars.abort_flag = 0;
        item_ring_init(bars.items, kItemReaders);
        mbar_init(smem_u32(&bars.q_full), 1);
        mbar_init(smem_u32(&bars.q_empty), 1);
        mbar_init(smem_u32(&bars.drain), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&bars.kv_full[s]), 1);
            mbar_init(smem_u32(&bars.kv_empty[s]), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(smem_u32(&bars.s_full[x]), 1);
            mbar_init(smem_u32(&bars.p_full[x]), 128);
            mbar_init(smem_u32(&bars.o_full[x]), 1);
        }
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&bars.tmem_base), 512);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;
    const Watchdog wd{a.status, &bars.abort_flag, a.timeout_ns};

    if (warp == kLoadWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&a.tm_q);
            prefetch_tmap(&a.tm_k);
            prefetch_tmap(&a.tm_v);
            uint32_t q_iter = 0, kv_iter = 0;
            bool ok = true;
            for (uint32_t k = 0; ok; ++k) {
                int w;
                ok = item_claim(bars.items, a.work, k, w, wd);
                if (!ok || w >= a.n_items) break;
                const Item it = decode_item<kMode>(a, w);
                KvIter<kMode> kv(a, it);
                int kslot;
                bool more = kv.next(a, kslot);
                if (kMode == kStep && !more) continue;  // nothing of this block is visible
                if (q_iter > 0) ok = mbar_wait(smem_u32(&bars.q_empty), (q_iter - 1) & 1, wd);
                if (!ok) break;
                ++q_iter;
                mbar_arrive_expect_tx(smem_u32(&bars.q_full), 2 * Cfg<D>::kTileBytes);
                for (int x = 0; x < 2; ++x) {
                    const int row = ((it.b * a.H) + (x ? it.h1 : it.h0)) * a.q_len +
                                    (x ? it.slot1 : it.slot0) - a.q_slot0;
                    for (int bx = 0; bx < Cfg<D>::kBoxes; ++bx)
                        tma_load_2d(q_smem + x * Cfg<D>::kTileBytes + bx * Cfg<D>::kBoxBytes, &a.tm_q,
                                    bx * 64, row, smem_u32(&bars.q_full));
                }
                for (; ok && more; more = kv.next(a, kslot)) {
                    const int row = (it.b * a.Hkv + it.g) * a.kv_len + kslot;
                    for (int which = 0; which < 2 && ok; ++which) {  // K then V
                        const int st = kv_iter % kStages;
                        const uint32_t use = kv_iter / kStages;
                        if (use > 0) ok = mbar_wait(smem_u32(&bars.kv_empty[st]), (use - 1) & 1, wd);
                        if (!ok) break;
                        mbar_arrive_expect_tx(smem_u32(&bars.kv_full[st]), Cfg<D>::kTileBytes);
                        for (int bx = 0; bx < Cfg<D>::kBoxes; ++bx)
                            tma_load_2d(kv_smem + st * Cfg<D>::kTileBytes + bx * Cfg<D>::kBoxBytes,
                                        which ? &a.tm_v : &a.tm_k, bx * 64, row,
                                        smem_u32(&bars.kv_full[st]));
                        ++kv_iter;
                    }
                }
            }
            if (!ok) {
                // Let the copies already issued land before the CTA exits; the
                // abort flag is up, so these waits use a watchdog of their own.
                volatile int no_abort = 0;
                const Watchdog w2{a.status, &no_abort, a.timeout_ns};
                for (uint32_t i = kv_iter > kStages ? kv_iter - kStages : 0; i < kv_iter; ++i)
                    (void)mbar_wait(smem_u32(&bars.kv_full[i % kStages]), (i / kStages) & 1, w2);
                if (q_iter > 0) (void)mbar_wait(smem_u32(&bars.q_full), (q_iter - 1) & 1, w2);
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t tS[2] = {tmem, tmem + 128};
            const uint32_t tO[2] = {tmem + 256, tmem + 384};
            uint32_t q_iter = 0, kv_iter = 0, p_cnt[2] = {0, 0};
            bool ok = true;
            for (uint32_t k = 0; ok; ++k) {
                int w;
                ok = item_read(bars.items, k, w, false, wd);
                if (!ok || w >= a.n_items) break;
                const Item it = decode_item<kMode>(a, w);
                KvIter<kMode> kv(a, it);
                int ks;
                bool have_cur = kv.next(a, ks);   // tile 0 (every item has one, but
                if (kMode == kStep && !have_cur)  // in one step it may see none)
                    continue;
                bool have_next = kv.next(a, ks);  // tile 1
                ok = mbar_wait(smem_u32(&bars.q_full), q_iter & 1, wd);
                if (!ok) break;
                ++q_iter;
                // prologue: S_x = Q_x K_0^T
                uint32_t stK = kv_iter % kStages;
                ok = mbar_wait(smem_u32(&bars.kv_full[stK]), (kv_iter / kStages) & 1, wd);
                if (!ok) break;
                ++kv_iter;
                tc_fence_after();
                issue_qk<D>(tS[0], q_smem, kv_smem + stK * Cfg<D>::kTileBytes);
                umma_commit(smem_u32(&bars.s_full[0]));
                issue_qk<D>(tS[1], q_smem + Cfg<D>::kTileBytes, kv_smem + stK * Cfg<D>::kTileBytes);
                umma_commit(smem_u32(&bars.s_full[1]));
                umma_commit(smem_u32(&bars.kv_empty[stK]));
                if (!have_next) umma_commit(smem_u32(&bars.q_empty));
                for (int j = 0; have_cur && ok; ++j) {
                    const bool have_next2 = have_next && kv.next(a, ks);  // tile j + 2
                    const uint32_t stV = kv_iter % kStages;
                    ok = mbar_wait(smem_u32(&bars.kv_full[stV]), (kv_iter / kStages) & 1, wd);
                    if (!ok) break;
                    ++kv_iter;
                    const uint32_t v_addr = kv_smem + stV * Cfg<D>::kTileBytes;
                    ok = mbar_wait(smem_u32(&bars.p_full[0]), (p_cnt[0]++) & 1, wd);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv<D>(tO[0], tS[0], v_addr, j > 0);
                    if (!have_next) umma_commit(smem_u32(&bars.o_full[0]));
                    if (have_next) {
                        stK = kv_iter % kStages;
                        ok = mbar_wait(smem_u32(&bars.kv_full[stK]), (kv_iter / kStages) & 1, wd);
                        if (!ok) break;
                        ++kv_iter;
                        tc_fence_after();
                        issue_qk<D>(tS[0], q_smem, kv_smem + stK * Cfg<D>::kTileBytes);
                        umma_commit(smem_u32(&bars.s_full[0]));
                    }
                    ok = mbar_wait(smem_u32(&bars.p_full[1]), (p_cnt[1]++) & 1, wd);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv<D>(tO[1], tS[1], v_addr, j > 0);
                    umma_commit(smem_u32(&bars.kv_empty[stV]));
                    if (!have_next) umma_commit(smem_u32(&bars.o_full[1]));
                    if (have_next) {
                        issue_qk<D>(tS[1], q_smem + Cfg<D>::kTileBytes,
                                    kv_smem + stK * Cfg<D>::kTileBytes);
                        umma_commit(smem_u32(&bars.s_full[1]));
                        umma_commit(smem_u32(&bars.kv_empty[stK]));
                        if (!have_next2) umma_commit(smem_u32(&bars.q_empty));
                    }
                    have_cur = have_next;
                    have_next = have_next2;
                }
            }
            // Every product issued must finish before TMEM is released.
            umma_commit(smem_u32(&bars.drain));
            volatile int no_abort = 0;
            const Watchdog w2{a.status, &no_abort, a.timeout_ns};
            (void)mbar_wait(smem_u32(&bars.drain), 0, w2);
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int x = warp >> 2;                    // query tile of this warpgroup
        const int quarter = warp & 3;               // TMEM lane quarter
        const int r = quarter * 32 + lane;          // query row in the tile
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_off + x * 128;
        const uint32_t tO = tmem + lane_off + 256 + x * 128;
        const float sl2 = a.scale_log2;
        uint32_t s_cnt = 0, o_cnt = 0;
        bool ok = true;
        for (uint32_t k = 0; ok; ++k) {
            int w;
            ok = item_read(bars.items, k, w, true, wd);
            if (!ok || w >= a.n_items) break;
            const Item it = decode_item<kMode>(a, w);
            float m = -INFINITY, l = 0.f;
            KvIter<kMode> kv(a, it);
            const int qpos = x ? it.pos1 : it.pos0;
            const int2 bf = row_bounds(a.mk, qpos), bl = row_bounds(a.mk, qpos + kBM - 1);
            int kslot, j = 0;
            while (ok && kv.next(a, kslot)) {
                const int cls = class_from_rows(bf, bl, kv.kpos);
                ok = mbar_wait(smem_u32(&bars.s_full[x]), (s_cnt++) & 1, wd);
                if (!ok) break;
                tc_fence_after();
                if (cls == kSkip) {
                    uint32_t z[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) z[c] = 0u;
                    tmem_st32(tS, z);
                    tmem_st32(tS + 32, z);
                } else {
                    uint32_t raw[64];
                    float s[128];
                    tmem_ld64(tS, raw);
#pragma unroll
                    for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(raw[c]);
                    tmem_ld64(tS + 64, raw);
#pragma unroll
                    for (int c = 0; c < 64; ++c) s[64 + c] = __uint_as_float(raw[c]);
                    if (cls == kMask) {
                        // key column c is visible iff lo(i) <= kpos + c <= hi(i)
                        const int2 rb = row_bounds(a.mk, qpos + r);
                        const int lo = rb.x - kv.kpos;
                        const unsigned w = static_cast<unsigned>(rb.y - rb.x);
#pragma unroll
                        for (int c = 0; c < 128; ++c)
                            if (static_cast<unsigned>(c - lo) > w) s[c] = -INFINITY;
                    }
                    float mx = s[0];
#pragma unroll
                    for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
                    const float m_new = fmaxf(m, mx);
                    float alpha = 1.f;
                    bool rescale_o = false;
                    if ((m_new - m) * sl2 > kRescaleThreshold) {
                        alpha = ex2_approx((m - m_new) * sl2);  // 0 when m = -inf
                        l *= alpha;
                        m = m_new;
                        rescale_o = j > 0;
                    }
                    // m stays -inf while a row has seen no key of its band: p = 0 then
                    const float neg = m == -INFINITY ? 0.f : -m * sl2;
                    float rs = 0.f;
                    uint32_t pk[32];
#pragma unroll
                    for (int c = 0; c < 64; c += 2) {
                        const float p0 = ex2_approx(fmaf(s[c], sl2, neg));
                        const float p1 = ex2_approx(fmaf(s[c + 1], sl2, neg));
                        rs += p0 + p1;
                        pk[c >> 1] = pack_bf16x2(p0, p1);
                    }
                    tmem_st32(tS, pk);
#pragma unroll
                    for (int c = 64; c < 128; c += 2) {
                        const float p0 = ex2_approx(fmaf(s[c], sl2, neg));
                        const float p1 = ex2_approx(fmaf(s[c + 1], sl2, neg));
                        rs += p0 + p1;
                        pk[(c - 64) >> 1] = pack_bf16x2(p0, p1);
                    }
                    tmem_st32(tS + 32, pk);
                    l += rs;
                    if (__any_sync(0xffffffffu, rescale_o)) {
                        const float f = rescale_o ? alpha : 1.f;
#pragma unroll 1
                        for (int cc = 0; cc < D; cc += 32) {
                            uint32_t ov[32];
                            tmem_ld32(tO + cc, ov);
#pragma unroll
                            for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * f);
                            tmem_st32(tO + cc, ov);
                        }
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(smem_u32(&bars.p_full[x]));
                ++j;
            }
            if (!ok) break;
            const int h = x ? it.h1 : it.h0;
            const int64_t orow = (static_cast<int64_t>(it.b) * a.H + h) * a.q_len +
                                 (x ? it.slot1 : it.slot0) - a.q_slot0 + r;
            if constexpr (kMode == kStep) {
                if (j == 0) {  // the item saw nothing of this block: the merge identity
                    if (a.merge) continue;  // folding the identity changes nothing
                    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.o) + orow * D);
#pragma unroll 1
                    for (int c = 0; c < D / 4; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
                    a.lse[orow] = -INFINITY;
                    continue;
                }
            }
            // epilogue: O / l -> bf16 (fp32 for one step), LSE = m * scale + ln l
            ok = mbar_wait(smem_u32(&bars.o_full[x]), (o_cnt++) & 1, wd);
            if (!ok) break;
            tc_fence_after();
            const float inv = l > 0.f ? 1.0f / l : 0.f;
            if constexpr (kMode == kStep) {
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.o) + orow * D);
                if (a.merge) {
                    // (acc, partial) -> acc with the partial's LSE b = m*scale + ln l:
                    // O = ca * O_acc + cb * O_tmem with ca = wa / (wa + wb) and
                    // cb = wb / ((wa + wb) l). A row that saw no key (l = 0) keeps
                    // its pair; the TMEM loads stay warp-wide either way.
                    const float la = a.lse[orow];
                    const float lb = l > 0.f ? m * a.scale + logf(l) : -INFINITY;
                    const float M = fmaxf(la, lb);
                    const bool fold = lb != -INFINITY;
                    const float wa = (fold && la != -INFINITY) ? expf(la - M) : 0.f;
                    const float wb = fold ? expf(lb - M) : 0.f;
                    const float ws = wa + wb;
                    const float ca = fold ? wa / ws : 1.f;
                    const float cb = fold ? wb / ws * inv : 0.f;
#pragma unroll 1
                    for (int cc = 0; cc < D; cc += 32) {
                        uint32_t ov[32];
                        tmem_ld32(tO + cc, ov);
                        if (!fold) continue;
#pragma unroll
                        for (int v4 = 0; v4 < 8; ++v4) {
                            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                            if (wa != 0.f) x = dst[cc / 4 + v4];
                            x.x = fmaf(ca, x.x, cb * __uint_as_float(ov[4 * v4]));
                            x.y = fmaf(ca, x.y, cb * __uint_as_float(ov[4 * v4 + 1]));
                            x.z = fmaf(ca, x.z, cb * __uint_as_float(ov[4 * v4 + 2]));
                            x.w = fmaf(ca, x.w, cb * __uint_as_float(ov[4 * v4 + 3]));
                            dst[cc / 4 + v4] = x;
                        }
                    }
                    if (fold) a.lse[orow] = M + logf(ws);
                    continue;
                }
#pragma unroll 1
                for (int cc = 0; cc < D; cc += 32) {
                    uint32_t ov[32];
                    tmem_ld32(tO + cc, ov);
#pragma unroll
                    for (int v4 = 0; v4 < 8; ++v4)
                        dst[cc / 4 + v4] = make_float4(__uint_as_float(ov[4 * v4]) * inv,
                                                       __uint_as_float(ov[4 * v4 + 1]) * inv,
                                                       __uint_as_float(ov[4 * v4 + 2]) * inv,
                                                       __uint_as_float(ov[4 * v4 + 3]) * inv);
                }
            } else {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + orow * D);
#pragma unroll 1
                for (int cc = 0; cc < D; cc += 32) {
                    uint32_t ov[32];
                    tmem_ld32(tO + cc, ov);
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        pk[c] = pack_bf16x2(__uint_as_float(ov[2 * c]) * inv,
                                            __uint_as_float(ov[2 * c + 1]) * inv);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4)
                        dst[cc / 8 + v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2],
                                                      pk[4 * v4 + 3]);
                }
            }
            a.lse[orow] = l > 0.f ? m * a.scale + logf(l) : -INFINITY;
        }
    }

    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D, int kMode>
cudaError_t launch(const TcArgs& a, int grid, const LaunchCtx& ctx) {
    constexpr int smem = Cfg<D>::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(ring_fwd_tc_kernel<D, kMode>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    ring_fwd_tc_kernel<D, kMode><<<grid, kThreads, smem, ctx.stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_tc(const AttnShape& sh, const void* q, const void* k, const void* v,
                          void* o, float* lse, const LaunchCtx& ctx) {
    TcArgs a{};
    cudaError_t e;
    const bool step = sh.mode == kStep;
    const int L = sh.S / sh.P;
    const int len = step ? L : sh.S;  // rows per head of q, k, v (one step: a rank's block)
    const uint64_t qrows = static_cast<uint64_t>(sh.B) * sh.H * len;
    const uint64_t kvrows = static_cast<uint64_t>(sh.B) * sh.Hkv * len;
    if ((e = make_tmap_bf16_rows(&a.tm_q, q, qrows, sh.D, kBM, 64)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16_rows(&a.tm_k, k, kvrows, sh.D, kBN, 64)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16_rows(&a.tm_v, v, kvrows, sh.D, kBN, 64)) != cudaSuccess) return e;
    a.o = o;
    a.lse = lse;
    a.status = ctx.status_word;
    a.timeout_ns = ctx.watchdog_ns;
    a.H = sh.H;
    a.Hkv = sh.Hkv;
    a.S = sh.S;
    a.P = sh.P;
    a.causal = sh.causal;
    a.G = sh.H / sh.Hkv;
    a.mk = MaskSpec{static_cast<const int4*>(sh.bounds), sh.S, sh.causal, sh.causal ? sh.window : 0};
    a.head_pair = (a.G % 2 == 0) ? 1 : 0;
    a.head_major = (!step && !sh.bounds && !a.mk.window) ? 1 : 0;
    a.n_units = a.head_pair ? len / kBM : len / (2 * kBM);
    a.n_head_units = sh.B * (a.head_pair ? sh.H / 2 : sh.H);
    a.n_items = a.n_units * a.n_head_units;
    a.scale = sh.scale;
    a.scale_log2 = sh.scale * 1.4426950408889634f;
    a.lay = RingLayout{sh.S, sh.P, sh.S / sh.P, sh.zigzag ? sh.S / (2 * sh.P) : sh.S / sh.P,
                       sh.zigzag};
    a.q_len = len;
    a.q_slot0 = step ? sh.rank * L : 0;
    a.kv_len = len;
    a.owner = step ? sh.owner : 0;
    a.merge = step ? sh.merge : 0;
    if ((e = next_work_counter(ctx, a.n_items, &a.work)) != cudaSuccess) return e;
    const int grid = std::min(a.n_items, ctx.num_sms);
    if (sh.D == 64) {
        if (sh.mode == kStep) return launch<64, kStep>(a, grid, ctx);
        if (sh.mode == kGathered) return launch<64, kGathered>(a, grid, ctx);
        return launch<64, kRing>(a, grid, ctx);
    }
    if (sh.mode == kStep) return launch<128, kStep>(a, grid, ctx);
    if (sh.mode == kGathered) return launch<128, kGathered>(a, grid, ctx);
    return launch<128, kRing>(a, grid, ctx);
}

}  // namespace rm
