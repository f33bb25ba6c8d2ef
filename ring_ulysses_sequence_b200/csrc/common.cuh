// Device helpers shared by the sm_100a kernels: ring layout arithmetic,
// bounded mbarrier waits, TMA tile loads, and tcgen05 (TMEM / UMMA) wrappers.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda.h>
#include <stdint.h>


namespace rm {

// ---------------------------------------------------------------------------
// Ring layout: rank-major slot <-> natural token position.
// ---------------------------------------------------------------------------

// Rank i's L tokens sit in slots [i*L, (i+1)*L). Contiguous order: slot s holds
// natural position s. Zigzag order (2P chunks of c tokens): rank i holds chunk
// i then chunk 2P-1-i.
struct RingLayout {
    int S, P, L, c, zigzag;

    __host__ __device__ __forceinline__ int pos_of_slot(int s) const {
        if (!zigzag) return s;
        int i = s / L, u = s - i * L;
        return u < c ? i * c + u : (2 * P - 1 - i) * c + (u - c);
    }
    __host__ __device__ __forceinline__ int slot_of_pos(int x) const {
        if (!zigzag) return x;
        int k = x / c, off = x - k * c;
        return k < P ? k * L + off : (2 * P - 1 - k) * L + c + off;
    }
    // Owner of the key/value block rank i holds at ring step t: blocks move one
    // rank forward per step, so it is (i - t) mod P.
    __host__ __device__ __forceinline__ int owner(int i, int t) const {
        int r = i - t;
        return r < 0 ? r + P : r;
    }
};

// Which keys each query sees, in natural token positions. A query at position
// i sees the keys lo(i) <= j <= hi(i); a key at position j is seen by the
// queries imin(j) <= i <= imax(j). All four bounds are non-decreasing in the
// position, so the visible pairs of any two tiles form a band. Without a table
// they follow from the mask: causal ("DeDLOC Guide", Best Practices, Causal
// Mask Handling) with an optional left window of W keys (axolotl-ringmaster
// README, Status: sliding-window attention), query i seeing i - W < j <= i, or
// no mask at all. With packed documents (the README's packing / varlen) a
// per-token table {lo, hi, imin, imax} holds them (rm_varlen_bounds).
struct MaskSpec {
    const int4* tab;  // per-token bounds, or null
    int S, causal, window;
};

// {lo(i), hi(i)}
__device__ __forceinline__ int2 row_bounds(const MaskSpec& m, int i) {
    if (m.tab) {
        const int4 t = m.tab[i];
        return make_int2(t.x, t.y);
    }
    return make_int2((m.causal && m.window) ? max(0, i - m.window + 1) : 0, m.causal ? i : m.S - 1);
}

// {imin(j), imax(j)}
__device__ __forceinline__ int2 col_bounds(const MaskSpec& m, int j) {
    if (m.tab) {
        const int4 t = m.tab[j];
        return make_int2(t.z, t.w);
    }
    return make_int2(m.causal ? j : 0,
                     (m.causal && m.window) ? min(m.S - 1, j + m.window - 1) : m.S - 1);
}

// Class of a (128-query tile, 128-key tile) pair. kSkip: no pair visible;
// kFull: every pair visible; kMask: mixed. From the query side: the bounds of
// the tile's first row (f) and last row (l) against the key tile at kpos.
enum : int { kSkip = 0, kMask = 1, kFull = 2 };
__device__ __forceinline__ int class_from_rows(int2 f, int2 l, int kpos) {
    if (kpos > l.y || kpos + 127 < f.x) return kSkip;
    return (kpos >= l.x && kpos + 127 <= f.y) ? kFull : kMask;
}
// The same pair from the key side: bounds of the key tile's first and last key
// against the query tile at qpos.
__device__ __forceinline__ int class_from_cols(int2 f, int2 l, int qpos) {
    if (qpos > l.y || qpos + 127 < f.x) return kSkip;
    return (qpos >= l.x && qpos + 127 <= f.y) ? kFull : kMask;
}

// ceil(x / 128) for any sign of x (the shift rounds toward minus infinity).
__host__ __device__ __forceinline__ int ceil_div128(int x) { return -((-x) >> 7); }

// ---------------------------------------------------------------------------
// Watchdog: every spin-wait is bounded in time.
// ---------------------------------------------------------------------------

enum : unsigned { kErrTimeout = 1u, kErrSlotReuse = 2u, kErrSmemLayout = 4u };

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

struct Watchdog {
    unsigned* err;          // device status word (global)
    volatile int* abort;    // CTA-wide abort flag (shared)
    uint64_t limit_ns;
};

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete. Gives up (returns
// false) when the CTA's abort flag is set or the time limit passes; in the
// latter case it raises the abort flag and the device status word.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const Watchdog& wd) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 16; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*wd.abort) return false;
        if (globaltimer_ns() - t0 > wd.limit_ns) {
            *wd.abort = 1;
            atomicOr(wd.err, kErrTimeout);
            return false;
        }
    }
}

// ---------------------------------------------------------------------------
// Dynamic work distribution inside a persistent CTA. The producer thread takes
// the next work-item index from the launch's counter in device memory (so a CTA
// that finishes early takes more work) and publishes it in a ring of
// kItemRing slots; the other roles read the k-th claimed index from slot
// k % kItemRing. An index >= the item count means no more work.
// ---------------------------------------------------------------------------

constexpr int kItemRing = 4;

struct ItemRing {
    uint64_t full[kItemRing], empty[kItemRing];
    int id[kItemRing];
};

// readers: the number of arrivals that release a slot.
__device__ __forceinline__ void item_ring_init(ItemRing& r, int readers) {
    for (int i = 0; i < kItemRing; ++i) {
        mbar_init(smem_u32(&r.full[i]), 1);
        mbar_init(smem_u32(&r.empty[i]), readers);
    }
}

// A launch's work-item counter: one of the library's counter slots, set to
// `base` on the launch's stream just before the launch. base carries the
// launch's generation in every byte (g * 0x01010101, g = 1..255), and two
// launches that use one slot one after the other have different generations.
// Every claim before the last returns an index below n_items and each CTA
// makes one claim past it, so a value outside [base, base + n_items + grid]
// means another launch has re-armed the slot while this one still runs.
struct WorkCounter {
    int* ptr;
    int base;
    int n_items;
};

// Claims the k-th item of this CTA (one thread). A launch that finds its slot
// re-armed by another raises kErrSlotReuse and stops (it publishes n_items,
// "no more work"). Its one claim per CTA has then advanced the other launch's
// counter, whose results are undefined too; the status word reports it. (A
// compare-and-swap claim would leave the other launch untouched, but 148
// producers starting at once serialise on it: it cost several percent on
// short launches.)
__device__ __forceinline__ bool item_claim(ItemRing& r, const WorkCounter& c, uint32_t k, int& w,
                                           const Watchdog& wd) {
    const int slot = k % kItemRing;
    if (k >= kItemRing && !mbar_wait(smem_u32(&r.empty[slot]), (k / kItemRing - 1) & 1, wd))
        return false;
    const int v = atomicAdd(c.ptr, 1) - c.base;
    const unsigned span = static_cast<unsigned>(c.n_items) + gridDim.x;
    if (static_cast<unsigned>(v) > span) {
        atomicOr(wd.err, kErrSlotReuse);
        w = c.n_items;
    } else {
        w = v;
    }
    r.id[slot] = w;
    mbar_arrive(smem_u32(&r.full[slot]));  // release: the index is visible first
    return true;
}

// Reads the k-th claimed item. A whole warp calls it with `warp_wide` set and
// its lane 0 releases the slot once every lane has read it; a single thread
// whose other lanes do not take part calls it with `warp_wide` clear and
// releases the slot itself (a warp-wide sync there would wait forever).
__device__ __forceinline__ bool item_read(ItemRing& r, uint32_t k, int& w, bool warp_wide,
                                          const Watchdog& wd) {
    const int slot = k % kItemRing;
    bool ok = mbar_wait(smem_u32(&r.full[slot]), (k / kItemRing) & 1, wd);
    if (warp_wide) ok = __all_sync(0xffffffffu, ok);  // the lanes leave together
    if (!ok) return false;
    w = *reinterpret_cast<volatile int*>(&r.id[slot]);
    if (warp_wide) {
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(smem_u32(&r.empty[slot]));
    } else {
        mbar_arrive(smem_u32(&r.empty[slot]));
    }
    return true;
}

// ---------------------------------------------------------------------------
// TMA (no multicast anywhere in this library)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tma_load_2d(uint32_t smem_dst, const CUtensorMap* map, int c0,
                                            int c1, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

// Non-tensor bulk copy global -> shared (16-byte aligned addresses, size a
// multiple of 16), completing on the mbarrier's transaction count.
__device__ __forceinline__ void bulk_load(uint32_t smem_dst, const void* gsrc, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_dst),
        "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(bar)
        : "memory");
}

// Element-wise add of a shared-memory tile into global memory through a tensor
// map (the addition happens at L2), tracked by the issuing thread's bulk group.
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, int c0, int c1,
                                                  uint32_t smem_src) {
    asm volatile(
        "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group"
        " [%0, {%1, %2}], [%3];" ::"l"(reinterpret_cast<uint64_t>(map)),
        "r"(c0), "r"(c1), "r"(smem_src)
        : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until the issuing thread's bulk groups have finished READING their
// shared-memory sources (the buffers may then be reused).
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Waits until the issuing thread's bulk groups have completed entirely.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy reads (UMMA operands, TMA stores) of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory and UMMA
// ---------------------------------------------------------------------------

// Warp-wide: allocates ncols TMEM columns (power of two >= 32) and writes the
// base address to shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t smem_dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_dst),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for UMMA with the 128-byte swizzle.
// Bit fields: start address >> 4 [0,14), leading byte offset >> 4 [16,30),
// stride byte offset >> 4 [32,46), version 1 at [46,48), layout type at
// [61,64) with 2 = SWIZZLE_128B.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 accumulation.
// c_format [4,6) = 1 (F32); a_format [7,10) = 1 (BF16); b_format [10,13) = 1;
// a_major bit 15, b_major bit 16 (0 = K-major, 1 = MN-major); N >> 3 at
// [17,23); M >> 4 at [24,29).
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, int a_mn_major,
                                                       int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn_major) << 15) |
           (static_cast<uint32_t>(b_mn_major) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives once on the mbarrier when every tcgen05 operation this thread issued
// before it has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp receives lane
// (lane base + t). The wait is inside the same asm so that no use of the
// registers can be scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// Two loads of 32 columns each, one wait (64 columns in flight together).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]),
          "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]),
          "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
          "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]),
          "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]),
          "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
}

// 32 lanes x 128 consecutive 32-bit columns in one load, then the wait.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x128.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%128];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
        "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
        "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]),
        "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Division by a run-time invariant divisor d in [1, 2^31] for n in [0, 2^31):
// q = (umulhi(n, m) + n) >> s with s = ceil(log2 d) and
// m = floor(2^32 (2^s - d) / d) + 1 (Granlund and Montgomery, "Division by
// invariant integers using multiplication", 1994).
// ---------------------------------------------------------------------------

struct FastDiv {
    uint32_t d, m, s;
    __host__ void init(uint32_t div) {
        d = div;
        s = 0;
        while ((1ull << s) < div) ++s;
        m = static_cast<uint32_t>(((1ull << 32) * ((1ull << s) - div)) / div + 1);
    }
    __device__ __forceinline__ uint32_t div(uint32_t n) const {
        return (__umulhi(n, m) + n) >> s;
    }
};

// ---------------------------------------------------------------------------
// Small math
// ---------------------------------------------------------------------------

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed fp32 pairs (sm_100 f32x2 instructions: one issue slot for two lanes).
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace rm
