// Ring attention backward, bf16 in / fp32 accumulate, on the sm_100a tensor
// cores (axolotl-ringmaster README: flash-style reverse-ring backward, fp32
// gradient accumulation across ring steps).
//
// Gradients of L = sum(dO * O), with P_ij = exp(scale q_i.k_j - LSE_i) over the
// visible keys and Delta_i = <dO_i, O_i>:
//   dV_j = sum_i P_ij dO_i            dS_ij = P_ij (<dO_i, v_j> - Delta_i)
//   dK_j = scale sum_i dS_ij q_i      dQ_i  = scale sum_j dS_ij k_j
// A KV head's dK/dV sum over the G query heads that share it.
//
// Three kernels, no atomics (every output element is written exactly once):
//   bwd_delta_kernel   Delta = rowsum(dO * O)                      (HBM-bound)
//   ring_bwd_dkdv      one 128-key tile of one KV head per work item (KV-
//                      stationary). The tile's block travels the ring backwards:
//                      at step t it visits the queries of rank (r + t) mod P,
//                      every head of the group. Per query tile:
//                        S^T = K Q^T, dP^T = V dO^T       (TMEM, fp32)
//                        P^T, dS^T -> bf16 back into TMEM (compute warps)
//                        dV += P^T dO, dK += dS^T Q       (TMEM A operand)
//   ring_bwd_dq        one 128-query tile per work item (Q-stationary), key
//                      tiles in ring order (i - t) mod P:
//                        S = Q K^T, dP = dO V^T; dS -> bf16 in TMEM;
//                        dQ += dS K
//                      S has two TMEM buffers (the kernel leaves 128 columns
//                      free), so S of tile j + 1 runs on the tensor pipe while
//                      the compute warps turn tile j's S, dP into dS.
// Warp roles as in the forward: warps 0-7 compute (two warpgroups splitting the
// 128 columns of S), warp 8 issues UMMA, warp 9 issues TMA. TMEM (512 cols):
// dK/dV: S^T [0,128), dP^T [128,256), dV at 256, dK at 384; dQ: S in two
// buffers [0,128) and [128,256), dP [256,384), dQ at 384. The elementwise step
// runs in two passes, P first (the MMA thread can start the product that needs
// only P) and dS second, and S and dP signal separately, so the compute warps
// start P while dP is still on the tensor pipe.
//
// One-step mode (`step`): the part of the backward that one rank of a ring
// across devices computes at one step. Its L local queries meet the L keys of
// one owner's block only: dQ of the rank and dK/dV of the block are ADDED to
// the arrays passed in (q-side arrays hold the rank's rows, k-side arrays the
// block's rows), so that dQ accumulates over the steps on the rank and dK/dV
// over the ranks the block visits. A tile that sees nothing of the other side
// is left untouched. Every element is still written by one CTA per launch, so
// the sums stay deterministic.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tmap.h"

namespace rm {

namespace {

constexpr int kT = 128;          // tile edge (rows of Q and of K/V)
constexpr int kThreads = 320;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr int kStages = 2;
constexpr int kKRing = 3;        // dQ kernel: K tiles in flight (S runs a tile ahead of dQ)
constexpr int kVRing = 2;        // dQ kernel: V tiles in flight
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BCfg {
    static constexpr int kTile = kT * D * 2;        // one bf16 tile
    static constexpr int kBoxes = D / 64;
    static constexpr int kBox = kT * 128;           // 16 KB swizzle box
    // dK/dV kernel: K, V resident; stages of Q + dO + LSE + Delta
    static constexpr int kStageKV = 2 * kTile + 2 * kT * 4;
    static constexpr int kKvBarOff = 2 * kTile + kStages * kStageKV;
    // dQ kernel: Q, dO resident; a ring of K tiles and a ring of V tiles
    static constexpr int kKRingOff = 2 * kTile;
    static constexpr int kVRingOff = kKRingOff + kKRing * kTile;
    static constexpr int kQBarOff = kVRingOff + kVRing * kTile;
    static constexpr int kSmemKV = kKvBarOff + 256 + 1024;
    static constexpr int kSmemQ = kQBarOff + 256 + 1024;
};

// TMEM column of K-step k (16 elements) of a bf16 operand written by the two
// compute warpgroups: warpgroup w packs its 64 columns into [64w, 64w+32).
__device__ __forceinline__ uint32_t packed_col(int k) { return k < 4 ? 8 * k : 64 + 8 * (k - 4); }

struct BwdArgs {
    CUtensorMap tm_q, tm_k, tm_v, tm_do;
    CUtensorMap tm_dq;  // fused kernel: fp32 dQ in 128-row x 32-column boxes (TMA reduce-add)
    const float* lse;
    const float* delta;
    float* dq;
    float* dk;
    float* dv;
    unsigned* status;
    WorkCounter work;  // this launch's work-item counter
    unsigned long long timeout_ns;
    int B, H, Hkv, S, P, causal, G, n_items;
    MaskSpec mk;     // which keys each query sees
    float scale, scale_log2;
    RingLayout lay;
    int step;        // one step: rank `rank`'s queries against `owner`'s block
    int rank, owner;
    int q_len;       // rows per head of q, dout, lse, delta, dq: S, or L for one step
    int kv_len;      // rows per head of k, v, dk, dv: S, or L for one step
    int head_major;  // item order: one head after another (see decode_kv_item)
};

constexpr int kItemReaders = 9;  // the MMA thread and one lane of each compute warp

struct Bars {
    ItemRing items;  // work items claimed by the producer (dynamic distribution)
    uint64_t res_full, res_empty, drain, acc_full;
    uint64_t st_full[kStages], st_empty[kStages];
    uint64_t s_full, dp_full;         // S^T in TMEM; dP^T in TMEM
    uint64_t p_half, p_full;          // P^T written; dS^T written
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// Barriers of the dQ kernel: separate rings for K and V tiles.
struct QBars {
    ItemRing items;
    uint64_t res_full, res_empty, drain, acc_full;
    uint64_t k_full[kKRing], k_empty[kKRing], v_full[kVRing], v_empty[kVRing];
    uint64_t s_full[2];   // S of buffer b is in TMEM (S runs up to two tiles ahead)
    uint64_t dp_full;     // dP of the next tile is in TMEM
    uint64_t p_full;      // dS written
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(QBars) <= 256, "barrier block");

// -------------------------------------------------------------------- dK / dV

struct KvItem {
    int b, g, kslot, kpos, rank;
};

// Key tiles in natural position order, earliest first (causal: they are seen
// by the most query tiles).
// One step: the tiles of the owner's block, in slot order; kslot is then the
// row within the block. head_major (whole-ring launches with plain causal or
// full masks): one head's key tiles after another, so the CTAs running at one
// time sweep one head's Q and dO, which stay in L2; otherwise (windows, packed
// documents, one step) the heads of one position are adjacent.
__device__ __forceinline__ KvItem decode_kv_item(const BwdArgs& a, int w) {
    KvItem it;
    const int nhu = a.B * a.Hkv, nu = a.kv_len / kT;
    const int hu = a.head_major ? w / nu : w % nhu;
    const int unit = a.head_major ? w - hu * nu : w / nhu;
    it.b = hu / a.Hkv;
    it.g = hu - it.b * a.Hkv;
    if (a.step) {
        it.kslot = unit * kT;
        it.kpos = a.lay.pos_of_slot(a.owner * a.lay.L + it.kslot);
        it.rank = a.owner;
    } else {
        it.kpos = unit * kT;
        it.kslot = a.lay.slot_of_pos(it.kpos);
        it.rank = it.kslot / a.lay.L;
    }
    return it;
}

// Query tiles (head, slot, class) that see a key tile, in reverse-ring order:
// step t visits rank (r + t) mod P; heads of the group innermost. A rank's
// block is one (contiguous) or two (zigzag) runs of consecutive positions. The
// queries that see any key of the tile form one interval [imin(first key),
// imax(last key)] (the bounds are monotone), so the query tiles to visit in a
// run are an interval too: O(1) work per returned tile, no division. qpos holds
// the natural position of the query tile last returned.
struct QIter {
    int rank, kpos, g, t, run, u, u_end, s0, p0, hh, cls, qslot, qpos;
    int2 cf, cl;  // {imin, imax} of the key tile's first and last key
    __device__ __forceinline__ QIter(const BwdArgs& a, const KvItem& it)
        : rank(it.rank), kpos(it.kpos), g(it.g), t(0), run(-1), u(0), u_end(0), s0(0), p0(0),
          hh(a.G), cls(kSkip), qslot(0), qpos(0) {
        cf = col_bounds(a.mk, it.kpos);
        cl = col_bounds(a.mk, it.kpos + kT - 1);
    }
    // `a` is the kernel's parameter block itself
    __device__ __forceinline__ bool next(const BwdArgs& a, int& h, int& slot, int& c) {
        const RingLayout& lay = a.lay;
        for (;;) {
            if (hh < a.G) {
                h = g * a.G + hh++;
                slot = qslot;
                c = cls;
                return true;
            }
            while (u >= u_end) {
                const int runs = lay.zigzag ? 2 : 1;
                if (++run == runs) {  // run starts at -1: the first call opens run 0 of step 0
                    run = 0;
                    // one step: the launching rank's runs only (t stays P after)
                    if (a.step || ++t == lay.P) {
                        run = runs - 1;
                        t = lay.P;
                        return false;
                    }
                }
                int i = a.step ? a.rank : rank + t;
                if (i >= lay.P) i -= lay.P;
                const int ctiles = (lay.zigzag ? lay.c : lay.L) / kT;
                s0 = (a.step ? 0 : i * lay.L) + run * lay.c;
                p0 = lay.zigzag ? (run == 0 ? i * lay.c : (2 * lay.P - 1 - i) * lay.c) : i * lay.L;
                // query tiles meeting [cf.x, cl.y]
                u = max(0, ceil_div128(cf.x - (kT - 1) - p0));
                u_end = min(ctiles, max(((cl.y - p0) >> 7) + 1, 0));
            }
            qslot = s0 + u * kT;
            qpos = p0 + u * kT;
            cls = class_from_cols(cf, cl, qpos);
            ++u;
            hh = 0;
        }
    }
};

template <int D>
__device__ __forceinline__ void issue_tile_product(uint32_t tmem_d, uint32_t a_smem, uint32_t b_smem) {
    // D[128 x 128] = A[128 x D] * B[128 x D]^T, both K-major in 128-byte swizzle boxes.
    constexpr uint32_t idesc = umma_idesc_bf16(kT, kT, 0, 0);
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * BCfg<D>::kBox + (k & 3) * 32;
        umma_ss(tmem_d, umma_desc_sw128(a_smem + off, 16, 1024), umma_desc_sw128(b_smem + off, 16, 1024),
                idesc, k > 0 ? 1u : 0u);
    }
}

template <int D>
__device__ __forceinline__ void issue_acc_product(uint32_t tmem_acc, uint32_t tmem_a, uint32_t b_smem,
                                                  bool accumulate) {
    // ACC[128 x D] += A[128 x 128] (bf16 in TMEM) * B[128 x D] (row-major tile, MN-major operand).
    constexpr uint32_t idesc = umma_idesc_bf16(kT, D, 0, 1);
#pragma unroll
    for (int k = 0; k < kT / 16; ++k)
        umma_ts(tmem_acc, tmem_a + packed_col(k), umma_desc_sw128(b_smem + k * 2048, BCfg<D>::kBox, 1024),
                idesc, (accumulate || k > 0) ? 1u : 0u);
}

// Stores N fp32 accumulator columns of this thread's TMEM row, times `mul`;
// with `add`, adds them to what dst holds.
template <int N>
__device__ __forceinline__ void store_cols(uint32_t taddr, float* dst, float mul, int add) {
#pragma unroll 1
    for (int cc = 0; cc < N; cc += 32) {
        uint32_t v[32];
        tmem_ld32(taddr + cc, v);
        float4* d4 = reinterpret_cast<float4*>(dst + cc);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            float4 x = make_float4(__uint_as_float(v[4 * c]) * mul, __uint_as_float(v[4 * c + 1]) * mul,
                                   __uint_as_float(v[4 * c + 2]) * mul, __uint_as_float(v[4 * c + 3]) * mul);
            if (add) {
                const float4 y = d4[c];
                x.x += y.x;
                x.y += y.y;
                x.z += y.z;
                x.w += y.w;
            }
            d4[c] = x;
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) ring_bwd_dkdv_kernel(const __grid_constant__ BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    Bars& bars = *reinterpret_cast<Bars*>(smem + BCfg<D>::kKvBarOff);
    const uint32_t k_smem = smem_u32(smem);
    const uint32_t v_smem = k_smem + BCfg<D>::kTile;
    const uint32_t st_smem = k_smem + 2 * BCfg<D>::kTile;  // stage s: Q, dO, LSE, Delta
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        bars.abort_flag = 0;
        item_ring_init(bars.items, kItemReaders);
        mbar_init(smem_u32(&bars.res_full), 1);
        mbar_init(smem_u32(&bars.res_empty), 1);
        mbar_init(smem_u32(&bars.drain), 1);
        mbar_init(smem_u32(&bars.acc_full), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&bars.st_full[s]), 1);
            mbar_init(smem_u32(&bars.st_empty[s]), 1);
        }
        mbar_init(smem_u32(&bars.s_full), 1);
        mbar_init(smem_u32(&bars.dp_full), 1);
        mbar_init(smem_u32(&bars.p_half), 256);
        mbar_init(smem_u32(&bars.p_full), 256);
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
        if (lane == 0) {
            prefetch_tmap(&a.tm_q);
            prefetch_tmap(&a.tm_k);
            prefetch_tmap(&a.tm_v);
            prefetch_tmap(&a.tm_do);
            uint32_t items = 0, fills = 0;  // items: those with at least one query tile
            bool ok = true;
            for (uint32_t k = 0; ok; ++k) {
                int w;
                ok = item_claim(bars.items, a.work, k, w, wd);
                if (!ok || w >= a.n_items) break;
                const KvItem it = decode_kv_item(a, w);
                QIter qi(a, it);
                int h, qslot, cls;
                bool more = qi.next(a, h, qslot, cls);
                if (!more) continue;  // one step: no query of the rank sees this tile
                if (items > 0) ok = mbar_wait(smem_u32(&bars.res_empty), (items - 1) & 1, wd);
                if (!ok) break;
                ++items;
                const int krow = (it.b * a.Hkv + it.g) * a.kv_len + it.kslot;
                mbar_arrive_expect_tx(smem_u32(&bars.res_full), 2 * BCfg<D>::kTile);
                for (int bx = 0; bx < BCfg<D>::kBoxes; ++bx) {
                    tma_load_2d(k_smem + bx * BCfg<D>::kBox, &a.tm_k, bx * 64, krow, smem_u32(&bars.res_full));
                    tma_load_2d(v_smem + bx * BCfg<D>::kBox, &a.tm_v, bx * 64, krow, smem_u32(&bars.res_full));
                }
                for (; ok && more; more = qi.next(a, h, qslot, cls)) {
                    const int st = fills % kStages;
                    const uint32_t use = fills / kStages;
                    if (use > 0) ok = mbar_wait(smem_u32(&bars.st_empty[st]), (use - 1) & 1, wd);
                    if (!ok) break;
                    const uint32_t base = st_smem + st * BCfg<D>::kStageKV;
                    const int qrow = (it.b * a.H + h) * a.q_len + qslot;
                    const uint32_t bar = smem_u32(&bars.st_full[st]);
                    mbar_arrive_expect_tx(bar, BCfg<D>::kStageKV);
                    for (int bx = 0; bx < BCfg<D>::kBoxes; ++bx) {
                        tma_load_2d(base + bx * BCfg<D>::kBox, &a.tm_q, bx * 64, qrow, bar);
                        tma_load_2d(base + BCfg<D>::kTile + bx * BCfg<D>::kBox, &a.tm_do, bx * 64, qrow, bar);
                    }
                    bulk_load(base + 2 * BCfg<D>::kTile, a.lse + qrow, kT * 4, bar);
                    bulk_load(base + 2 * BCfg<D>::kTile + kT * 4, a.delta + qrow, kT * 4, bar);
                    ++fills;
                }
            }
            if (!ok) {
                volatile int no_abort = 0;
                const Watchdog w2{a.status, &no_abort, a.timeout_ns};
                for (uint32_t i = fills > kStages ? fills - kStages : 0; i < fills; ++i)
                    (void)mbar_wait(smem_u32(&bars.st_full[i % kStages]), (i / kStages) & 1, w2);
                if (items > 0) (void)mbar_wait(smem_u32(&bars.res_full), (items - 1) & 1, w2);
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 384;
            uint32_t items = 0, uses = 0, p_cnt = 0;
            bool ok = true;
            for (uint32_t k = 0; ok; ++k) {
                int w;
                ok = item_read(bars.items, k, w, false, wd);
                if (!ok || w >= a.n_items) break;
                const KvItem it = decode_kv_item(a, w);
                QIter qi(a, it);
                int qh, qs, qc;
                if (!qi.next(a, qh, qs, qc)) continue;  // query tile 0 (one step may have none)
                ok = mbar_wait(smem_u32(&bars.res_full), items & 1, wd);
                if (!ok) break;
                ++items;
                tc_fence_after();
                // S^T of query tile j + 1 is issued right after dV of tile j (it
                // overwrites P^T, which dV has read: in-order pipe), so the next
                // tile's P^T pass runs while dK and dP^T finish on the tensor pipe.
                auto stage = [&](int& st) -> bool {
                    st = uses % kStages;
                    const bool r = mbar_wait(smem_u32(&bars.st_full[st]), (uses / kStages) & 1, wd);
                    ++uses;
                    tc_fence_after();
                    return r;
                };
                int st = 0;
                ok = stage(st);
                if (ok) {
                    const uint32_t q_addr = st_smem + st * BCfg<D>::kStageKV;
                    issue_tile_product<D>(tS, k_smem, q_addr);                     // S^T = K Q^T
                    umma_commit(smem_u32(&bars.s_full));
                    issue_tile_product<D>(tdP, v_smem, q_addr + BCfg<D>::kTile);   // dP^T = V dO^T
                    umma_commit(smem_u32(&bars.dp_full));
                }
                for (int j = 0; ok; ++j) {
                    const uint32_t q_addr = st_smem + st * BCfg<D>::kStageKV;
                    const uint32_t do_addr = q_addr + BCfg<D>::kTile;
                    // dV runs while the compute warps work out dS^T
                    ok = mbar_wait(smem_u32(&bars.p_half), p_cnt & 1, wd);
                    if (!ok) break;
                    tc_fence_after();
                    issue_acc_product<D>(tdV, tS, do_addr, j > 0);   // dV += P^T dO
                    const bool have_next = qi.next(a, qh, qs, qc);
                    int st_next = st;
                    if (have_next) {
                        ok = stage(st_next);
                        if (!ok) break;
                        issue_tile_product<D>(tS, k_smem, st_smem + st_next * BCfg<D>::kStageKV);
                        umma_commit(smem_u32(&bars.s_full));
                    }
                    ok = mbar_wait(smem_u32(&bars.p_full), (p_cnt++) & 1, wd);
                    if (!ok) break;
                    tc_fence_after();
                    issue_acc_product<D>(tdK, tdP, q_addr, j > 0);   // dK += dS^T Q
                    umma_commit(smem_u32(&bars.st_empty[st]));
                    if (!have_next) break;
                    // dP^T of the next tile overwrites dS^T after dK has read it
                    issue_tile_product<D>(tdP, v_smem, st_smem + st_next * BCfg<D>::kStageKV + BCfg<D>::kTile);
                    umma_commit(smem_u32(&bars.dp_full));
                    st = st_next;
                }
                if (!ok) break;
                umma_commit(smem_u32(&bars.acc_full));
                umma_commit(smem_u32(&bars.res_empty));
            }
            umma_commit(smem_u32(&bars.drain));
            volatile int no_abort = 0;
            const Watchdog w2{a.status, &no_abort, a.timeout_ns};
            (void)mbar_wait(smem_u32(&bars.drain), 0, w2);
        }
    } else {
        const int wg = warp >> 2;               // which 64 query columns
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;      // key row of the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_off + 64 * wg;
        const uint32_t tdP = tmem + lane_off + 128 + 64 * wg;
        constexpr int HC = D / 2;               // accumulator columns per warpgroup
        const uint32_t tdV = tmem + lane_off + 256 + HC * wg;
        const uint32_t tdK = tmem + lane_off + 384 + HC * wg;
        const float sl2 = a.scale_log2;
        uint32_t uses = 0, s_cnt = 0, items = 0;  // s_cnt counts tiles for s_full and dp_full
        bool ok = true;
        for (uint32_t k = 0; ok; ++k) {
            int w;
            ok = item_read(bars.items, k, w, true, wd);
            if (!ok || w >= a.n_items) break;
            const KvItem it = decode_kv_item(a, w);
            QIter qi(a, it);
            int h, qslot, cls, ntiles = 0;
            while (ok && qi.next(a, h, qslot, cls)) {
                ++ntiles;
                const int st = uses % kStages;
                ++uses;
                // key row r sees query column c iff imin(j) <= qpos + c <= imax(j)
                int lo = 0;
                unsigned wq = 0;
                if (cls == kMask) {
                    const int2 cb = col_bounds(a.mk, it.kpos + r);
                    lo = cb.x - qi.qpos;
                    wq = static_cast<unsigned>(cb.y - cb.x);
                }
                const float* lse_s = reinterpret_cast<const float*>(
                    smem + 2 * BCfg<D>::kTile + st * BCfg<D>::kStageKV + 2 * BCfg<D>::kTile);
                const float* del_s = lse_s + kT;
                ok = mbar_wait(smem_u32(&bars.s_full), s_cnt & 1, wd);
                if (!ok) break;
                tc_fence_after();
                // Two passes over two quarters of 32 query columns. Pass 1: P^T
                // from S^T and LSE, written as bf16 over S^T columns already
                // read (dV can start); pass 2: dS^T = P^T (dP^T - Delta) from the
                // fp32 P kept in registers, written over dP^T. LSE and Delta come
                // four at a time from shared memory; the arithmetic runs on
                // packed fp32 pairs.
                const uint64_t sl2x2 = pk2(sl2, sl2);
                const uint64_t nlog2e = pk2(-kLog2e, -kLog2e);
                uint64_t pp[32];  // P of this thread's 64 query columns, in pairs
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    uint32_t sv[32];
                    tmem_ld32(tS + 32 * qq, sv);
                    const float4* lse4 = reinterpret_cast<const float4*>(lse_s + 64 * wg + 32 * qq);
                    uint32_t pk[16];
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 L = lse4[c4];
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int c = 4 * c4 + 2 * hh;
                            const uint64_t lse2 = mul2(hh ? pk2(L.z, L.w) : pk2(L.x, L.y), nlog2e);
                            float x0, x1;
                            upk2(fma2(pk2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sl2x2, lse2), x0, x1);
                            float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                            if (cls == kMask) {
                                const int q0 = 64 * wg + 32 * qq + c;
                                if (static_cast<unsigned>(q0 - lo) > wq) p0 = 0.f;
                                if (static_cast<unsigned>(q0 + 1 - lo) > wq) p1 = 0.f;
                            }
                            pp[16 * qq + (c >> 1)] = pk2(p0, p1);
                            pk[c >> 1] = pack_bf16x2(p0, p1);
                        }
                    }
                    tmem_st16(tS + 16 * qq, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(smem_u32(&bars.p_half));
                ok = mbar_wait(smem_u32(&bars.dp_full), (s_cnt++) & 1, wd);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    uint32_t dpv[32];
                    tmem_ld32(tdP + 32 * qq, dpv);
                    const float4* del4 = reinterpret_cast<const float4*>(del_s + 64 * wg + 32 * qq);
                    uint32_t dsk[16];
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 Dl = del4[c4];
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int c = 4 * c4 + 2 * hh;
                            const uint64_t dd = mul2(pp[16 * qq + (c >> 1)],
                                                     sub2(pk2(__uint_as_float(dpv[c]), __uint_as_float(dpv[c + 1])),
                                                          hh ? pk2(Dl.z, Dl.w) : pk2(Dl.x, Dl.y)));
                            float d0, d1;
                            upk2(dd, d0, d1);
                            dsk[c >> 1] = pack_bf16x2(d0, d1);
                        }
                    }
                    tmem_st16(tdP + 16 * qq, dsk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(smem_u32(&bars.p_full));
            }
            if (!ok) break;
            if (ntiles == 0) continue;  // one step: the tile meets none of the rank's queries
            ok = mbar_wait(smem_u32(&bars.acc_full), items & 1, wd);
            if (!ok) break;
            ++items;
            tc_fence_after();
            const int64_t krow = (static_cast<int64_t>(it.b) * a.Hkv + it.g) * a.kv_len + it.kslot + r;
            store_cols<HC>(tdV, a.dv + krow * D + HC * wg, 1.0f, a.step);
            store_cols<HC>(tdK, a.dk + krow * D + HC * wg, a.scale, a.step);
        }
    }

    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// -------------------------------------------------------------------- fused

// One kernel for dK, dV and dQ: five products per tile pair instead of the
// seven of the two kernels (S and dP are computed once). It is KV-stationary
// like ring_bwd_dkdv_kernel; in addition the compute warps write dS^T as bf16
// to shared memory, where it is the A operand of both dK += dS^T Q (read
// K-major) and dQ_tile = dS K (the same bytes read MN-major, i.e. transposed).
// dQ_tile lands in the TMEM columns of dP^T, which the compute warps have read
// by then. They read it out, scale it, and write it 64 columns at a time to a
// 32 KB staging tile, which a reducer thread adds into global dQ with TMA
// reduce-add (fp32 additions at L2, whole 128-byte lines; per-thread vector
// reductions instead issue 4096 separate 16-byte requests per tile pair, which
// the SM's path to L2 cannot sustain). The order of those additions across
// CTAs depends on timing, so dQ varies in its last bits from run to run; dK
// and dV are written once per element. The two-kernel path is the
// deterministic option.
//
// Roles: warps 0-7 compute (two warpgroups, 64 query columns each), warp 8
// lane 0 issues UMMA, warp 9 lane 0 loads by TMA, warp 9 lane 1 issues the dQ
// reductions. TMEM: S^T [0,128) (bf16 P^T over it), dP^T then dQ_tile
// [128,256), dV at 256, dK at 384. Shared memory: K, V resident; two stages of
// Q + dO; the dQ staging tile (128 rows x 64 fp32, two 32-column boxes with
// the 128-byte swizzle). dS^T (128 x 128 bf16, laid out like a TMA tile) goes
// over the stage's dO once dV has read it when D = 128 (dO is then exactly
// its size); with D = 64 it has a buffer of its own. The LSE and Delta of
// each stage's 128 queries are loaded with it into the last 2 KB (every
// thread of a warpgroup reads the same 64 values of each).
constexpr int kDsBox = kT * 128;  // one 64-column box of the dS^T tile; one 32-column fp32 box

template <int D>
struct FCfg {
    static constexpr bool kDsInStage = D == 128;      // dS^T over the stage's dO
    static constexpr int kTile = kT * D * 2;
    static constexpr int kStage = 2 * kTile;          // Q + dO
    static constexpr int kStOff = 2 * kTile;
    static constexpr int kStgOff = kStOff + kStages * kStage;
    static constexpr int kDsOff = kStgOff + kT * 64 * 4;  // own dS^T buffer (D = 64)
    static constexpr int kBarOff = kDsOff + (kDsInStage ? 0 : kT * kT * 2);
    static constexpr int kLdOff = kBarOff + 256;   // LSE and Delta of stage s: 2 x 128 fp32
    static constexpr int kLdStage = 2 * kT * 4;
    static constexpr int kNeed = kLdOff + kStages * kLdStage;
    // The layout is 1024-byte aligned; what is allocated beyond kNeed (at most
    // the 227 KB a block may have) absorbs the dynamic base's misalignment.
    static constexpr int kSmem = kNeed + 1024 <= 232448 ? kNeed + 1024 : 232448;
    static constexpr int kSlack = kSmem - kNeed;
};
static_assert(FCfg<128>::kSlack >= 256, "shared memory of the fused backward");
static_assert(FCfg<64>::kSmem <= 232448, "shared memory of the fused backward");

struct FBars {
    ItemRing items;
    uint64_t res_full, res_empty, drain, acc_full;
    uint64_t st_full[kStages], st_empty[kStages];
    uint64_t s_full, dp_full;  // S^T, dP^T in TMEM
    uint64_t p_half;           // P^T written (256 arrivals)
    uint64_t dv_done;          // dV has read the stage's dO (dS^T may overwrite it)
    uint64_t ds_full;          // dS^T in shared memory and dP^T read out (256)
    uint64_t dq_full;          // dK and dQ_tile done: dQ_tile in TMEM, dS^T and the stage free
    uint64_t dq_empty;         // dQ_tile read out of TMEM (256)
    uint64_t stg_full;         // a 64-column round of dQ_tile staged (256)
    uint64_t stg_free;         // the reducer's TMA has read the staging tile (1)
    int stg_row;               // the round's first dQ row (-1: no more), and which round
    int stg_round;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(FBars) <= 256, "barrier block");

template <int D>
__device__ __forceinline__ void issue_dk_product(uint32_t tmem_acc, uint32_t ds_smem, uint32_t q_smem,
                                                 bool accumulate) {
    // dK[128 keys x D] += dS^T[128 keys x 128 queries] (K-major) * Q[128 queries x D] (MN-major)
    constexpr uint32_t idesc = umma_idesc_bf16(kT, D, 0, 1);
#pragma unroll
    for (int k = 0; k < kT / 16; ++k)
        umma_ss(tmem_acc, umma_desc_sw128(ds_smem + (k >> 2) * kDsBox + (k & 3) * 32, 16, 1024),
                umma_desc_sw128(q_smem + k * 2048, BCfg<D>::kBox, 1024), idesc,
                (accumulate || k > 0) ? 1u : 0u);
}

template <int D>
__device__ __forceinline__ void issue_dq_product(uint32_t tmem_acc, uint32_t ds_smem, uint32_t k_smem) {
    // dQ_tile[128 queries x D] = dS[128 queries x 128 keys] (MN-major: the dS^T
    // bytes) * K[128 keys x D] (MN-major)
    constexpr uint32_t idesc = umma_idesc_bf16(kT, D, 1, 1);
#pragma unroll
    for (int k = 0; k < kT / 16; ++k)
        umma_ss(tmem_acc, umma_desc_sw128(ds_smem + k * 2048, kDsBox, 1024),
                umma_desc_sw128(k_smem + k * 2048, BCfg<D>::kBox, 1024), idesc, k > 0 ? 1u : 0u);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) ring_bwd_fused_kernel(const __grid_constant__ BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    // D = 128 fills the block's shared memory but for 768 bytes: a dynamic base
    // further than that from a 1024-byte boundary (not seen on sm_100a) makes
    // the launch return at once with an error in the status word.
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    if (pad > static_cast<uint32_t>(FCfg<D>::kSlack)) {
        if (threadIdx.x == 0) atomicOr(a.status, kErrSmemLayout);
        return;
    }
    uint8_t* smem = smem_raw + pad;
    FBars& bars = *reinterpret_cast<FBars*>(smem + FCfg<D>::kBarOff);
    const uint32_t k_smem = smem_u32(smem);
    const uint32_t ld_smem = k_smem + FCfg<D>::kLdOff;  // stage s: LSE[128], Delta[128]
    const uint32_t v_smem = k_smem + FCfg<D>::kTile;
    const uint32_t st_smem = k_smem + FCfg<D>::kStOff;   // stage s: Q, dO
    const uint32_t stg_smem = k_smem + FCfg<D>::kStgOff;  // dQ staging (two 32-column fp32 boxes)
    // dS^T of a tile in stage st: over its dO (D = 128) or in the own buffer (D = 64)
    auto ds_of = [&](int st) -> uint32_t {
        return FCfg<D>::kDsInStage ? st_smem + st * FCfg<D>::kStage + FCfg<D>::kTile
                                   : k_smem + FCfg<D>::kDsOff;
    };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        bars.abort_flag = 0;
        item_ring_init(bars.items, kItemReaders);
        mbar_init(smem_u32(&bars.res_full), 1);
        mbar_init(smem_u32(&bars.res_empty), 1);
        mbar_init(smem_u32(&bars.drain), 1);
        mbar_init(smem_u32(&bars.acc_full), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&bars.st_full[s]), 1);
            mbar_init(smem_u32(&bars.st_empty[s]), 1);
        }
        mbar_init(smem_u32(&bars.s_full), 1);
        mbar_init(smem_u32(&bars.dp_full), 1);
        mbar_init(smem_u32(&bars.p_half), 256);
        mbar_init(smem_u32(&bars.dv_done), 1);
        mbar_init(smem_u32(&bars.ds_full), 256);
        mbar_init(smem_u32(&bars.dq_full), 1);
        mbar_init(smem_u32(&bars.dq_empty), 256);
        mbar_init(smem_u32(&bars.stg_full), 256);
        mbar_init(smem_u32(&bars.stg_free), 1);
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
        if (lane == 0) {
            // ------------------------------------------------------ producer
            prefetch_tmap(&a.tm_q);
            prefetch_tmap(&a.tm_k);
            prefetch_tmap(&a.tm_v);
            prefetch_tmap(&a.tm_do);
            uint32_t items = 0, fills = 0;
            bool ok = true;
            for (uint32_t k = 0; ok; ++k) {
                int w;
                ok = item_claim(bars.items, a.work, k, w, wd);
                if (!ok || w >= a.n_items) break;
                const KvItem it = decode_kv_item(a, w);
                QIter qi(a, it);
                int h, qslot, cls;
                bool more = qi.next(a, h, qslot, cls);
                if (!more) continue;  // one step: no query of the rank sees this tile
                if (items > 0) ok = mbar_wait(smem_u32(&bars.res_empty), (items - 1) & 1, wd);
                if (!ok) break;
                ++items;
                const int krow = (it.b * a.Hkv + it.g) * a.kv_len + it.kslot;
                mbar_arrive_expect_tx(smem_u32(&bars.res_full), 2 * FCfg<D>::kTile);
                for (int bx = 0; bx < BCfg<D>::kBoxes; ++bx) {
                    tma_load_2d(k_smem + bx * BCfg<D>::kBox, &a.tm_k, bx * 64, krow, smem_u32(&bars.res_full));
                    tma_load_2d(v_smem + bx * BCfg<D>::kBox, &a.tm_v, bx * 64, krow, smem_u32(&bars.res_full));
                }
                for (; ok && more; more = qi.next(a, h, qslot, cls)) {
                    const int st = fills % kStages;
                    const uint32_t use = fills / kStages;
                    if (use > 0) ok = mbar_wait(smem_u32(&bars.st_empty[st]), (use - 1) & 1, wd);
                    if (!ok) break;
                    const uint32_t base = st_smem + st * FCfg<D>::kStage;
                    const int qrow = (it.b * a.H + h) * a.q_len + qslot;
                    const uint32_t bar = smem_u32(&bars.st_full[st]);
                    mbar_arrive_expect_tx(bar, FCfg<D>::kStage + FCfg<D>::kLdStage);
                    for (int bx = 0; bx < BCfg<D>::kBoxes; ++bx) {
                        tma_load_2d(base + bx * BCfg<D>::kBox, &a.tm_q, bx * 64, qrow, bar);
                        tma_load_2d(base + FCfg<D>::kTile + bx * BCfg<D>::kBox, &a.tm_do, bx * 64, qrow, bar);
                    }
                    bulk_load(ld_smem + st * FCfg<D>::kLdStage, a.lse + qrow, kT * 4, bar);
                    bulk_load(ld_smem + st * FCfg<D>::kLdStage + kT * 4, a.delta + qrow, kT * 4, bar);
                    ++fills;
                }
            }
            if (!ok) {
                volatile int no_abort = 0;
                const Watchdog w2{a.status, &no_abort, a.timeout_ns};
                for (uint32_t i = fills > kStages ? fills - kStages : 0; i < fills; ++i)
                    (void)mbar_wait(smem_u32(&bars.st_full[i % kStages]), (i / kStages) & 1, w2);
                if (items > 0) (void)mbar_wait(smem_u32(&bars.res_full), (items - 1) & 1, w2);
            }
        } else if (lane == 1) {
            // ------------------------------------------------------ dQ reducer
            // Adds each staged 64-column round into global dQ (box 0 -> columns
            // 32 r, box 1 -> D/2 + 32 r for round r), and frees the staging tile
            // once the TMA has read it. Single-thread role: no warp-collective
            // operation here.
            prefetch_tmap(&a.tm_dq);
            for (uint32_t n = 0;; ++n) {
                if (!mbar_wait(smem_u32(&bars.stg_full), n & 1, wd)) break;
                const int row = *reinterpret_cast<volatile int*>(&bars.stg_row);
                const int round = *reinterpret_cast<volatile int*>(&bars.stg_round);
                if (row < 0) break;
                tma_reduce_add_2d(&a.tm_dq, 32 * round, row, stg_smem);
                tma_reduce_add_2d(&a.tm_dq, D / 2 + 32 * round, row, stg_smem + kDsBox);
                bulk_commit_group();
                bulk_wait_read_all();
                mbar_arrive(smem_u32(&bars.stg_free));
            }
            bulk_wait_all();  // every reduction issued has landed before the CTA exits
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            // ------------------------------------------------------ MMA issuer
            const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 384;
            uint32_t items = 0, uses = 0, p_cnt = 0, dq_cnt = 0;
            bool ok = true;
            for (uint32_t k = 0; ok; ++k) {
                int w;
                ok = item_read(bars.items, k, w, false, wd);
                if (!ok || w >= a.n_items) break;
                const KvItem it = decode_kv_item(a, w);
                QIter qi(a, it);
                int qh, qs, qc;
                if (!qi.next(a, qh, qs, qc)) continue;  // query tile 0 (one step may have none)
                ok = mbar_wait(smem_u32(&bars.res_full), items & 1, wd);
                if (!ok) break;
                ++items;
                tc_fence_after();
                auto stage = [&](int& st) -> bool {
                    st = uses % kStages;
                    const bool r = mbar_wait(smem_u32(&bars.st_full[st]), (uses / kStages) & 1, wd);
                    ++uses;
                    tc_fence_after();
                    return r;
                };
                int st = 0;
                ok = stage(st);
                if (ok) {
                    const uint32_t q_addr = st_smem + st * FCfg<D>::kStage;
                    issue_tile_product<D>(tS, k_smem, q_addr);  // S^T = K Q^T
                    umma_commit(smem_u32(&bars.s_full));
                    // dP^T goes where the previous tile's dQ was: it must be read out
                    if (dq_cnt > 0) ok = mbar_wait(smem_u32(&bars.dq_empty), (dq_cnt - 1) & 1, wd);
                    if (ok) {
                        tc_fence_after();
                        issue_tile_product<D>(tdP, v_smem, q_addr + FCfg<D>::kTile);  // dP^T = V dO^T
                        umma_commit(smem_u32(&bars.dp_full));
                    }
                }
                for (int j = 0; ok; ++j) {
                    const uint32_t q_addr = st_smem + st * FCfg<D>::kStage;
                    const uint32_t do_addr = q_addr + FCfg<D>::kTile;
                    ok = mbar_wait(smem_u32(&bars.p_half), p_cnt & 1, wd);
                    if (!ok) break;
                    tc_fence_after();
                    issue_acc_product<D>(tdV, tS, do_addr, j > 0);  // dV += P^T dO
                    umma_commit(smem_u32(&bars.dv_done));          // dO read: dS^T may go there
                    const bool have_next = qi.next(a, qh, qs, qc);
                    int st_next = st;
                    if (have_next) {  // S^T of the next tile overwrites P^T after dV read it
                        ok = stage(st_next);
                        if (!ok) break;
                        issue_tile_product<D>(tS, k_smem, st_smem + st_next * FCfg<D>::kStage);
                        umma_commit(smem_u32(&bars.s_full));
                    }
                    ok = mbar_wait(smem_u32(&bars.ds_full), (p_cnt++) & 1, wd);
                    if (!ok) break;
                    tc_fence_after();
                    issue_dk_product<D>(tdK, ds_of(st), q_addr, j > 0);  // dK += dS^T Q
                    issue_dq_product<D>(tdP, ds_of(st), k_smem);          // dQ_tile = dS K
                    umma_commit(smem_u32(&bars.st_empty[st]));            // Q and dS^T read
                    umma_commit(smem_u32(&bars.dq_full));
                    ++dq_cnt;
                    if (!have_next) break;
                    ok = mbar_wait(smem_u32(&bars.dq_empty), (dq_cnt - 1) & 1, wd);
                    if (!ok) break;
                    tc_fence_after();
                    issue_tile_product<D>(tdP, v_smem, st_smem + st_next * FCfg<D>::kStage + FCfg<D>::kTile);
                    umma_commit(smem_u32(&bars.dp_full));
                    st = st_next;
                }
                if (!ok) break;
                umma_commit(smem_u32(&bars.acc_full));
                umma_commit(smem_u32(&bars.res_empty));  // after dQ_tile, the last reader of K
            }
            umma_commit(smem_u32(&bars.drain));
            volatile int no_abort = 0;
            const Watchdog w2{a.status, &no_abort, a.timeout_ns};
            (void)mbar_wait(smem_u32(&bars.drain), 0, w2);
        }
    } else {
        // ---------------------------------------------------------- compute
        const int wg = warp >> 2;               // which 64 query columns (and D/2 dQ columns)
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;      // TMEM lane: key row (S^T, dP^T), query row (dQ)
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_off + 64 * wg;
        const uint32_t tdP = tmem + lane_off + 128 + 64 * wg;
        constexpr int HC = D / 2;               // accumulator columns per warpgroup
        const uint32_t tdQ = tmem + lane_off + 128 + HC * wg;
        const uint32_t tdV = tmem + lane_off + 256 + HC * wg;
        const uint32_t tdK = tmem + lane_off + 384 + HC * wg;
        const uint32_t stg_row = stg_smem + wg * kDsBox + r * 128;  // this thread's staging row
        const float sl2 = a.scale_log2;
        uint32_t uses = 0, s_cnt = 0, items = 0, dq_cnt = 0, rounds = 0;
        // dQ_tile of the tile before: waits for dK and dQ_tile, reads it out of
        // TMEM (then dP^T of the next tile may go there) and stages it, scaled,
        // 32 of this thread's columns per round, for the reducer.
        auto drain = [&](int row) -> bool {
            if (!mbar_wait(smem_u32(&bars.dq_full), dq_cnt & 1, wd)) return false;
            ++dq_cnt;
            tc_fence_after();
#pragma unroll
            for (int rd = 0; rd < HC / 32; ++rd) {
                uint32_t v[32];
                tmem_ld32(tdQ + 32 * rd, v);
                if (rd == HC / 32 - 1) {  // all of dQ_tile read out: dP^T may overwrite it
                    tc_fence_before();
                    mbar_arrive(smem_u32(&bars.dq_empty));
                }
                // the previous round's TMA has read the staging tile
                if (rounds > 0 && !mbar_wait(smem_u32(&bars.stg_free), (rounds - 1) & 1, wd)) return false;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    st_shared_v4(stg_row + ((c ^ (r & 7)) << 4),
                                 __float_as_uint(__uint_as_float(v[4 * c]) * a.scale),
                                 __float_as_uint(__uint_as_float(v[4 * c + 1]) * a.scale),
                                 __float_as_uint(__uint_as_float(v[4 * c + 2]) * a.scale),
                                 __float_as_uint(__uint_as_float(v[4 * c + 3]) * a.scale));
                fence_proxy_async_smem();
                if (threadIdx.x == 0) {
                    bars.stg_row = row;
                    bars.stg_round = rd;
                }
                mbar_arrive(smem_u32(&bars.stg_full));
                ++rounds;
            }
            return true;
        };
        bool ok = true;
        for (uint32_t k = 0; ok; ++k) {
            int w;
            ok = item_read(bars.items, k, w, true, wd);
            if (!ok || w >= a.n_items) break;
            const KvItem it = decode_kv_item(a, w);
            QIter qi(a, it);
            int h, qslot, cls, ntiles = 0, pend_row = -1;
            while (ok && qi.next(a, h, qslot, cls)) {
                const int st = uses % kStages;
                ++uses;
                // key row r sees query column c iff imin(j) <= qpos + c <= imax(j)
                int lo = 0;
                unsigned wq = 0;
                if (cls == kMask) {
                    const int2 cb = col_bounds(a.mk, it.kpos + r);
                    lo = cb.x - qi.qpos;
                    wq = static_cast<unsigned>(cb.y - cb.x);
                }
                const int qrow0 = (it.b * a.H + h) * a.q_len + qslot;
                // LSE and Delta of the tile's queries, loaded with the stage (an
                // L2 round trip per tile here measured 121 against 108 ms)
                const float4* lse4 = reinterpret_cast<const float4*>(
                    smem + FCfg<D>::kLdOff + st * FCfg<D>::kLdStage) + 16 * wg;
                const float4* del4 = lse4 + kT / 4;
                ok = mbar_wait(smem_u32(&bars.s_full), s_cnt & 1, wd);
                if (!ok) break;
                tc_fence_after();
                // P^T from S^T and LSE, bf16 over the S^T columns already read
                const uint64_t sl2x2 = pk2(sl2, sl2);
                const uint64_t nlog2e = pk2(-kLog2e, -kLog2e);
                uint64_t pp[32];  // P of this thread's 64 query columns, in pairs
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    uint32_t sv[32];
                    tmem_ld32(tS + 32 * qq, sv);
                    uint32_t pk[16];
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 L = lse4[8 * qq + c4];
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int c = 4 * c4 + 2 * hh;
                            const uint64_t lse2 = mul2(hh ? pk2(L.z, L.w) : pk2(L.x, L.y), nlog2e);
                            float x0, x1;
                            upk2(fma2(pk2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sl2x2, lse2), x0, x1);
                            float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                            if (cls == kMask) {
                                const int q0 = 64 * wg + 32 * qq + c;
                                if (static_cast<unsigned>(q0 - lo) > wq) p0 = 0.f;
                                if (static_cast<unsigned>(q0 + 1 - lo) > wq) p1 = 0.f;
                            }
                            pp[16 * qq + (c >> 1)] = pk2(p0, p1);
                            pk[c >> 1] = pack_bf16x2(p0, p1);
                        }
                    }
                    tmem_st16(tS + 16 * qq, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(smem_u32(&bars.p_half));
                // the previous tile's dQ_tile, while this tile's dV runs
                if (pend_row >= 0) {
                    ok = drain(pend_row);
                    if (!ok) break;
                }
                ok = mbar_wait(smem_u32(&bars.dp_full), (s_cnt++) & 1, wd);
                if (!ok) break;
                tc_fence_after();
                if constexpr (FCfg<D>::kDsInStage) {  // dS^T goes over dO: dV must have read it
                    ok = mbar_wait(smem_u32(&bars.dv_done), (s_cnt - 1) & 1, wd);
                    if (!ok) break;
                }
                // dS^T = P^T (dP^T - Delta), bf16, to shared memory (the swizzled
                // layout of a TMA tile: 16-byte chunk c of row r at c ^ (r % 8))
                const uint32_t ds_row = ds_of(st) + wg * kDsBox + r * 128;
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    uint32_t dpv[32];
                    tmem_ld32(tdP + 32 * qq, dpv);
                    uint32_t dsk[16];
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 Dl = del4[8 * qq + c4];
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int c = 4 * c4 + 2 * hh;
                            const uint64_t dd = mul2(pp[16 * qq + (c >> 1)],
                                                     sub2(pk2(__uint_as_float(dpv[c]), __uint_as_float(dpv[c + 1])),
                                                          hh ? pk2(Dl.z, Dl.w) : pk2(Dl.x, Dl.y)));
                            float d0, d1;
                            upk2(dd, d0, d1);
                            dsk[c >> 1] = pack_bf16x2(d0, d1);
                        }
                    }
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
                        st_shared_v4(ds_row + (((4 * qq + cc) ^ (r & 7)) << 4), dsk[4 * cc],
                                     dsk[4 * cc + 1], dsk[4 * cc + 2], dsk[4 * cc + 3]);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(smem_u32(&bars.ds_full));
                pend_row = qrow0;
                ++ntiles;
            }
            if (!ok) break;
            if (ntiles == 0) continue;  // one step: the tile meets none of the rank's queries
            ok = drain(pend_row);
            if (!ok) break;
            ok = mbar_wait(smem_u32(&bars.acc_full), items & 1, wd);
            if (!ok) break;
            ++items;
            tc_fence_after();
            const int64_t krow = (static_cast<int64_t>(it.b) * a.Hkv + it.g) * a.kv_len + it.kslot + r;
            store_cols<HC>(tdV, a.dv + krow * D + HC * wg, 1.0f, a.step);
            store_cols<HC>(tdK, a.dk + krow * D + HC * wg, a.scale, a.step);
        }
        if (ok) {  // no more work: the reducer stops at this sentinel
            if (rounds > 0) ok = mbar_wait(smem_u32(&bars.stg_free), (rounds - 1) & 1, wd);
            if (ok && threadIdx.x == 0) bars.stg_row = -1;
            if (ok) mbar_arrive(smem_u32(&bars.stg_full));
        }
    }

    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// -------------------------------------------------------------------- dQ

struct QItem {
    int b, h, g, slot, pos, rank;
};

// Query tiles, latest natural position first when causal (the most key tiles).
// One step: the rank's tiles, latest slot first; slot is then the row within
// the rank's arrays. head_major: one head's query tiles after another (its K
// and V stay in L2); otherwise the heads of one position are adjacent (the
// same choice as for the key tiles).
__device__ __forceinline__ QItem decode_q_item(const BwdArgs& a, int w) {
    QItem it;
    const int nhu = a.B * a.H, nq = a.q_len / kT;
    const int hu = a.head_major ? w / nq : w % nhu;
    const int unit = a.head_major ? w - hu * nq : w / nhu;
    it.b = hu / a.H;
    it.h = hu - it.b * a.H;
    it.g = it.h / a.G;
    const int nu = a.causal ? (a.q_len / kT) - 1 - unit : unit;
    if (a.step) {
        it.slot = nu * kT;
        it.pos = a.lay.pos_of_slot(a.rank * a.lay.L + it.slot);
        it.rank = a.rank;
    } else {
        it.pos = nu * kT;
        it.slot = a.lay.slot_of_pos(it.pos);
        it.rank = it.slot / a.lay.L;
    }
    return it;
}

// Key tiles a query tile sees, in ring order: step t visits owner (i - t) mod P.
// The keys the tile's rows see form one interval [lo(first row), hi(last
// row)], so within each run of an owner's block the tiles to visit are an
// interval. kpos holds the natural position of the tile last returned.
struct KIter {
    int rank, qpos, t, run, u, u_end, s0, p0, kpos;
    int2 rf, rl;  // {lo, hi} of the query tile's first and last row
    __device__ __forceinline__ KIter(const BwdArgs& a, const QItem& it)
        : rank(it.rank), qpos(it.pos), t(0), run(-1), u(0), u_end(0), s0(0), p0(0), kpos(0) {
        rf = row_bounds(a.mk, it.pos);
        rl = row_bounds(a.mk, it.pos + kT - 1);
    }
    __device__ __forceinline__ bool next(const BwdArgs& a, int& kslot, int& cls) {
        const RingLayout& lay = a.lay;
        while (u >= u_end) {
            const int runs = lay.zigzag ? 2 : 1;
            if (++run == runs) {
                run = 0;
                // one step: the owner's runs only (t stays P after)
                if (a.step || ++t == lay.P) {
                    run = runs - 1;
                    t = lay.P;
                    return false;
                }
            }
            const int r = a.step ? a.owner : lay.owner(rank, t);
            const int ctiles = (lay.zigzag ? lay.c : lay.L) / kT;
            s0 = (a.step ? 0 : r * lay.L) + run * lay.c;
            p0 = lay.zigzag ? (run == 0 ? r * lay.c : (2 * lay.P - 1 - r) * lay.c) : r * lay.L;
            // key tiles meeting [rf.x, rl.y]
            u = max(0, ceil_div128(rf.x - (kT - 1) - p0));
            u_end = min(ctiles, max(((rl.y - p0) >> 7) + 1, 0));
        }
        kslot = s0 + u * kT;
        kpos = p0 + u * kT;
        cls = class_from_rows(rf, rl, kpos);
        ++u;
        return true;
    }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1) ring_bwd_dq_kernel(const __grid_constant__ BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    QBars& bars = *reinterpret_cast<QBars*>(smem + BCfg<D>::kQBarOff);
    const uint32_t q_smem = smem_u32(smem);
    const uint32_t do_smem = q_smem + BCfg<D>::kTile;
    const uint32_t kr_smem = q_smem + BCfg<D>::kKRingOff;  // slot s: one K tile
    const uint32_t vr_smem = q_smem + BCfg<D>::kVRingOff;  // slot s: one V tile
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        bars.abort_flag = 0;
        item_ring_init(bars.items, kItemReaders);
        mbar_init(smem_u32(&bars.res_full), 1);
        mbar_init(smem_u32(&bars.res_empty), 1);
        mbar_init(smem_u32(&bars.drain), 1);
        mbar_init(smem_u32(&bars.acc_full), 1);
        for (int s = 0; s < kKRing; ++s) {
            mbar_init(smem_u32(&bars.k_full[s]), 1);
            mbar_init(smem_u32(&bars.k_empty[s]), 1);
        }
        for (int s = 0; s < kVRing; ++s) {
            mbar_init(smem_u32(&bars.v_full[s]), 1);
            mbar_init(smem_u32(&bars.v_empty[s]), 1);
        }
        mbar_init(smem_u32(&bars.s_full[0]), 1);
        mbar_init(smem_u32(&bars.s_full[1]), 1);
        mbar_init(smem_u32(&bars.dp_full), 1);
        mbar_init(smem_u32(&bars.p_full), 256);
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
        if (lane == 0) {
            prefetch_tmap(&a.tm_q);
            prefetch_tmap(&a.tm_k);
            prefetch_tmap(&a.tm_v);
            prefetch_tmap(&a.tm_do);
            uint32_t items = 0, kf = 0, vf = 0;
            bool ok = true;
            // one tile into slot (n % ring) of a ring, once its previous use is released
            auto fill = [&](uint64_t* full, uint64_t* empty, int ring, uint32_t n, uint32_t dst,
                            const CUtensorMap* map, int row) -> bool {
                const int slot = n % ring;
                if (n >= static_cast<uint32_t>(ring) &&
                    !mbar_wait(smem_u32(&empty[slot]), (n / ring - 1) & 1, wd))
                    return false;
                mbar_arrive_expect_tx(smem_u32(&full[slot]), BCfg<D>::kTile);
                for (int bx = 0; bx < BCfg<D>::kBoxes; ++bx)
                    tma_load_2d(dst + slot * BCfg<D>::kTile + bx * BCfg<D>::kBox, map, bx * 64, row,
                                smem_u32(&full[slot]));
                return true;
            };
            for (uint32_t k = 0; ok; ++k) {
                int w;
                ok = item_claim(bars.items, a.work, k, w, wd);
                if (!ok || w >= a.n_items) break;
                const QItem it = decode_q_item(a, w);
                KIter ki(a, it);
                int kslot, cls;
                bool more = ki.next(a, kslot, cls);
                if (!more) continue;  // one step: the tile sees no key of the block
                if (items > 0) ok = mbar_wait(smem_u32(&bars.res_empty), (items - 1) & 1, wd);
                if (!ok) break;
                ++items;
                const int qrow = (it.b * a.H + it.h) * a.q_len + it.slot;
                mbar_arrive_expect_tx(smem_u32(&bars.res_full), 2 * BCfg<D>::kTile);
                for (int bx = 0; bx < BCfg<D>::kBoxes; ++bx) {
                    tma_load_2d(q_smem + bx * BCfg<D>::kBox, &a.tm_q, bx * 64, qrow, smem_u32(&bars.res_full));
                    tma_load_2d(do_smem + bx * BCfg<D>::kBox, &a.tm_do, bx * 64, qrow, smem_u32(&bars.res_full));
                }
                for (; ok && more; more = ki.next(a, kslot, cls)) {
                    const int krow = (it.b * a.Hkv + it.g) * a.kv_len + kslot;
                    ok = fill(bars.k_full, bars.k_empty, kKRing, kf, kr_smem, &a.tm_k, krow);
                    if (!ok) break;
                    ++kf;
                    ok = fill(bars.v_full, bars.v_empty, kVRing, vf, vr_smem, &a.tm_v, krow);
                    if (!ok) break;
                    ++vf;
                }
            }
            if (!ok) {
                volatile int no_abort = 0;
                const Watchdog w2{a.status, &no_abort, a.timeout_ns};
                for (uint32_t i = kf > kKRing ? kf - kKRing : 0; i < kf; ++i)
                    (void)mbar_wait(smem_u32(&bars.k_full[i % kKRing]), (i / kKRing) & 1, w2);
                for (uint32_t i = vf > kVRing ? vf - kVRing : 0; i < vf; ++i)
                    (void)mbar_wait(smem_u32(&bars.v_full[i % kVRing]), (i / kVRing) & 1, w2);
                if (items > 0) (void)mbar_wait(smem_u32(&bars.res_full), (items - 1) & 1, w2);
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            const uint32_t tS[2] = {tmem, tmem + 128};
            const uint32_t tdP = tmem + 256, tdQ = tmem + 384;
            uint32_t items = 0, kc = 0, vc = 0, p_cnt = 0;
            bool ok = true;
            for (uint32_t k = 0; ok; ++k) {
                int w;
                ok = item_read(bars.items, k, w, false, wd);
                if (!ok || w >= a.n_items) break;
                const QItem it = decode_q_item(a, w);
                KIter ki(a, it);  // one tile ahead of the S products
                int ks, kcls;
                if (!ki.next(a, ks, kcls)) continue;  // tile 0 (one step may have none)
                ok = mbar_wait(smem_u32(&bars.res_full), items & 1, wd);
                if (!ok) break;
                ++items;
                const uint32_t bk = kc, bv = vc;
                // S_j = Q K_j^T into buffer j & 1
                auto score = [&](uint32_t j) -> bool {
                    const uint32_t n = bk + j;
                    if (!mbar_wait(smem_u32(&bars.k_full[n % kKRing]), (n / kKRing) & 1, wd)) return false;
                    tc_fence_after();
                    issue_tile_product<D>(tS[j & 1], q_smem, kr_smem + (n % kKRing) * BCfg<D>::kTile);
                    umma_commit(smem_u32(&bars.s_full[j & 1]));
                    return true;
                };
                // dP_j = dO V_j^T
                auto dprod = [&](uint32_t j) -> bool {
                    const uint32_t n = bv + j;
                    if (!mbar_wait(smem_u32(&bars.v_full[n % kVRing]), (n / kVRing) & 1, wd)) return false;
                    tc_fence_after();
                    issue_tile_product<D>(tdP, do_smem, vr_smem + (n % kVRing) * BCfg<D>::kTile);
                    umma_commit(smem_u32(&bars.v_empty[n % kVRing]));
                    umma_commit(smem_u32(&bars.dp_full));
                    return true;
                };
                bool have1 = ki.next(a, ks, kcls);
                ok = score(0) && dprod(0) && (!have1 || score(1));
                uint32_t j = 0;
                for (; ok; ++j) {
                    ok = mbar_wait(smem_u32(&bars.p_full), (p_cnt++) & 1, wd);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t n = bk + j;
                    issue_acc_product<D>(tdQ, tdP, kr_smem + (n % kKRing) * BCfg<D>::kTile, j > 0);  // dQ += dS K
                    umma_commit(smem_u32(&bars.k_empty[n % kKRing]));
                    if (!have1) break;
                    // dP of tile j + 1 overwrites dS_j after dQ has read it (in-order pipe)
                    ok = dprod(j + 1);
                    if (!ok) break;
                    const bool have2 = ki.next(a, ks, kcls);
                    if (have2) ok = score(j + 2);  // buffer j & 1: tile j's S has been read
                    have1 = have2;
                }
                if (!ok) break;
                kc = bk + j + 1;
                vc = bv + j + 1;
                umma_commit(smem_u32(&bars.acc_full));
                umma_commit(smem_u32(&bars.res_empty));
            }
            umma_commit(smem_u32(&bars.drain));
            volatile int no_abort = 0;
            const Watchdog w2{a.status, &no_abort, a.timeout_ns};
            (void)mbar_wait(smem_u32(&bars.drain), 0, w2);
        }
    } else {
        const int wg = warp >> 2;               // which 64 key columns
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;      // query row of the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tS0 = tmem + lane_off + 64 * wg;
        const uint32_t tdP = tmem + lane_off + 256 + 64 * wg;
        constexpr int HC = D / 2;
        const uint32_t tdQ = tmem + lane_off + 384 + HC * wg;
        const float sl2 = a.scale_log2;
        uint32_t s_cnt[2] = {0, 0}, dp_cnt = 0, items = 0;
        bool ok = true;
        for (uint32_t k = 0; ok; ++k) {
            int w;
            ok = item_read(bars.items, k, w, true, wd);
            if (!ok || w >= a.n_items) break;
            const QItem it = decode_q_item(a, w);
            const int64_t qrow = (static_cast<int64_t>(it.b) * a.H + it.h) * a.q_len + it.slot + r;
            const float lse2 = a.lse[qrow] * kLog2e;
            const float delta = a.delta[qrow];
            KIter ki(a, it);
            int kslot, cls;
            uint32_t j = 0;
            for (; ok && ki.next(a, kslot, cls); ++j) {
                // query row r sees key column c iff lo(i) <= kpos + c <= hi(i)
                int lo = 0;
                unsigned wk = 0;
                if (cls == kMask) {
                    const int2 rb = row_bounds(a.mk, it.pos + r);
                    lo = rb.x - ki.kpos;
                    wk = static_cast<unsigned>(rb.y - rb.x);
                }
                // P from S as soon as S is in (it may be a tile ahead of dP)
                const int b = j & 1;
                ok = mbar_wait(smem_u32(&bars.s_full[b]), (s_cnt[b]++) & 1, wd);
                if (!ok) break;
                tc_fence_after();
                uint64_t pp[32];
                {
                    uint32_t sv[64];
                    tmem_ld64(tS0 + 128 * b, sv);
                    const uint64_t sl2x2 = pk2(sl2, sl2), nlse2 = pk2(-lse2, -lse2);
#pragma unroll
                    for (int c = 0; c < 64; c += 2) {
                        const int k0 = 64 * wg + c;
                        float x0, x1;
                        upk2(fma2(pk2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sl2x2, nlse2), x0, x1);
                        float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                        if (cls == kMask) {
                            if (static_cast<unsigned>(k0 - lo) > wk) p0 = 0.f;
                            if (static_cast<unsigned>(k0 + 1 - lo) > wk) p1 = 0.f;
                        }
                        pp[c >> 1] = pk2(p0, p1);
                    }
                }
                // then dS = P (dP - Delta), written over dP
                ok = mbar_wait(smem_u32(&bars.dp_full), (dp_cnt++) & 1, wd);
                if (!ok) break;
                tc_fence_after();
                const uint64_t del2 = pk2(delta, delta);
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t dpv[32], dsk[16];
                    tmem_ld32(tdP + 32 * h2, dpv);
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        float d0, d1;
                        upk2(mul2(pp[16 * h2 + (c >> 1)],
                                  sub2(pk2(__uint_as_float(dpv[c]), __uint_as_float(dpv[c + 1])), del2)), d0, d1);
                        dsk[c >> 1] = pack_bf16x2(d0, d1);
                    }
                    tmem_st16(tdP + 16 * h2, dsk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(smem_u32(&bars.p_full));
            }
            if (!ok) break;
            if (j == 0) continue;  // one step: the tile sees no key of the block
            ok = mbar_wait(smem_u32(&bars.acc_full), items & 1, wd);
            if (!ok) break;
            ++items;
            tc_fence_after();
            store_cols<HC>(tdQ, a.dq + qrow * D + HC * wg, a.scale, a.step);
        }
    }

    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// -------------------------------------------------------------------- Delta

// Delta_i = <dO_i, O_i> in fp32 from the bf16 dO rows and the O rows (bf16, or
// fp32 as a ring across devices accumulates them); one warp per row.
template <int D, typename OT>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const OT* __restrict__ o,
                                                        const __nv_bfloat16* __restrict__ dout,
                                                        float* __restrict__ delta, int64_t rows) {
    constexpr int PER = D / 32;  // elements per lane
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * 256) >> 5;
    for (int64_t r = warp; r < rows; r += nwarps) {
        const OT* po = o + r * D + lane * PER;
        const __nv_bfloat16* pd = dout + r * D + lane * PER;
        float x[PER], y[PER];
        if constexpr (PER == 4) {
            const uint2 vd = *reinterpret_cast<const uint2*>(pd);
            const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&vd);
            const float2 y0 = __bfloat1622float2(b2[0]), y1 = __bfloat1622float2(b2[1]);
            y[0] = y0.x; y[1] = y0.y; y[2] = y1.x; y[3] = y1.y;
        } else {
            const float2 y0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(pd));
            y[0] = y0.x; y[1] = y0.y;
        }
        if constexpr (sizeof(OT) == 4) {
            if constexpr (PER == 4) {
                const float4 v = *reinterpret_cast<const float4*>(po);
                x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
            } else {
                const float2 v = *reinterpret_cast<const float2*>(po);
                x[0] = v.x; x[1] = v.y;
            }
        } else if constexpr (PER == 4) {
            const uint2 vo = *reinterpret_cast<const uint2*>(po);
            const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&vo);
            const float2 x0 = __bfloat1622float2(a2[0]), x1 = __bfloat1622float2(a2[1]);
            x[0] = x0.x; x[1] = x0.y; x[2] = x1.x; x[3] = x1.y;
        } else {
            const float2 x0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(po));
            x[0] = x0.x; x[1] = x0.y;
        }
        float acc = 0.f;
#pragma unroll
        for (int i = PER - 1; i >= 0; --i) acc = fmaf(x[i], y[i], acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) delta[r] = acc;
    }
}

template <int D, typename OT>
cudaError_t launch_delta(const void* o, const void* dout, float* delta, int64_t rows,
                         const LaunchCtx& ctx) {
    const int64_t dblocks = std::min<int64_t>((rows + 7) / 8, static_cast<int64_t>(ctx.num_sms) * 16);
    bwd_delta_kernel<D, OT><<<static_cast<unsigned>(dblocks), 256, 0, ctx.stream>>>(
        static_cast<const OT*>(o), static_cast<const __nv_bfloat16*>(dout), delta, rows);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_bwd_d(const AttnShape& sh, const BwdArgs& base, const void* o, const void* dout,
                         float* delta, const LaunchCtx& ctx) {
    cudaError_t e;
    if (!base.step) {  // one step reads the Delta its caller computed once per rank
        const int64_t rows = static_cast<int64_t>(sh.B) * sh.H * sh.S;
        if ((e = launch_delta<D, __nv_bfloat16>(o, dout, delta, rows, ctx)) != cudaSuccess) return e;
    }

    BwdArgs a = base;
    a.n_items = sh.B * sh.Hkv * (a.kv_len / kT);
    if ((e = next_work_counter(ctx, a.n_items, &a.work)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ring_bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  BCfg<D>::kSmemKV)) != cudaSuccess)
        return e;
    ring_bwd_dkdv_kernel<D><<<std::min(a.n_items, ctx.num_sms), kThreads, BCfg<D>::kSmemKV, ctx.stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    a.n_items = sh.B * sh.H * (a.q_len / kT);
    if ((e = next_work_counter(ctx, a.n_items, &a.work)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ring_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  BCfg<D>::kSmemQ)) != cudaSuccess)
        return e;
    ring_bwd_dq_kernel<D><<<std::min(a.n_items, ctx.num_sms), kThreads, BCfg<D>::kSmemQ, ctx.stream>>>(a);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_bwd_fused(const AttnShape& sh, const BwdArgs& base, const void* o,
                             const void* dout, float* delta, float* dq, const LaunchCtx& ctx) {
    cudaError_t e;
    if (!base.step) {
        const int64_t rows = static_cast<int64_t>(sh.B) * sh.H * sh.S;
        if ((e = launch_delta<D, __nv_bfloat16>(o, dout, delta, rows, ctx)) != cudaSuccess) return e;
        // dQ is a sum of reductions: it starts at zero (one step adds to the caller's)
        if ((e = cudaMemsetAsync(dq, 0, static_cast<size_t>(rows) * D * sizeof(float), ctx.stream)) !=
            cudaSuccess)
            return e;
    }
    BwdArgs a = base;
    a.n_items = sh.B * sh.Hkv * (a.kv_len / kT);
    if ((e = next_work_counter(ctx, a.n_items, &a.work)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ring_bwd_fused_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  FCfg<D>::kSmem)) != cudaSuccess)
        return e;
    ring_bwd_fused_kernel<D><<<std::min(a.n_items, ctx.num_sms), kThreads, FCfg<D>::kSmem, ctx.stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd(const AttnShape& sh, const void* q, const void* k, const void* v,
                       const void* o, const float* lse, const void* dout, float* dq, float* dk,
                       float* dv, float* delta, const LaunchCtx& ctx) {
    BwdArgs a{};
    cudaError_t e;
    const bool step = sh.mode == 2;
    const int len = step ? sh.S / sh.P : sh.S;  // rows per head (one step: a rank's block)
    const uint64_t qrows = static_cast<uint64_t>(sh.B) * sh.H * len;
    const uint64_t kvrows = static_cast<uint64_t>(sh.B) * sh.Hkv * len;
    if ((e = make_tmap_bf16_rows(&a.tm_q, q, qrows, sh.D, kT, 64)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16_rows(&a.tm_do, dout, qrows, sh.D, kT, 64)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16_rows(&a.tm_k, k, kvrows, sh.D, kT, 64)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16_rows(&a.tm_v, v, kvrows, sh.D, kT, 64)) != cudaSuccess) return e;
    a.lse = lse;
    a.delta = delta;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.status = ctx.status_word;
    a.timeout_ns = ctx.watchdog_ns;
    a.B = sh.B;
    a.H = sh.H;
    a.Hkv = sh.Hkv;
    a.S = sh.S;
    a.P = sh.P;
    a.causal = sh.causal;
    a.G = sh.H / sh.Hkv;
    a.mk = MaskSpec{static_cast<const int4*>(sh.bounds), sh.S, sh.causal, sh.causal ? sh.window : 0};
    a.scale = sh.scale;
    a.scale_log2 = sh.scale * kLog2e;
    a.lay = RingLayout{sh.S, sh.P, sh.S / sh.P, sh.zigzag ? sh.S / (2 * sh.P) : sh.S / sh.P, sh.zigzag};
    a.step = step ? 1 : 0;
    a.rank = step ? sh.rank : 0;
    a.owner = step ? sh.owner : 0;
    a.q_len = len;
    a.kv_len = len;
    a.head_major = (!step && !sh.bounds && !a.mk.window) ? 1 : 0;
    if (!sh.deterministic) {
        if ((e = make_tmap_f32_rows(&a.tm_dq, dq, qrows, sh.D, kT, 32)) != cudaSuccess) return e;
        return sh.D == 64 ? launch_bwd_fused<64>(sh, a, o, dout, delta, dq, ctx)
                          : launch_bwd_fused<128>(sh, a, o, dout, delta, dq, ctx);
    }
    return sh.D == 64 ? launch_bwd_d<64>(sh, a, o, dout, delta, ctx)
                      : launch_bwd_d<128>(sh, a, o, dout, delta, ctx);
}

cudaError_t launch_bwd_delta(const void* o, int o_fp32, const void* dout, float* delta,
                             int64_t rows, int D, const LaunchCtx& ctx) {
    if (D == 64)
        return o_fp32 ? launch_delta<64, float>(o, dout, delta, rows, ctx)
                      : launch_delta<64, __nv_bfloat16>(o, dout, delta, rows, ctx);
    return o_fp32 ? launch_delta<128, float>(o, dout, delta, rows, ctx)
                  : launch_delta<128, __nv_bfloat16>(o, dout, delta, rows, ctx);
}

}  // namespace rm
