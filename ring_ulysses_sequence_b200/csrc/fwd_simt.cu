// Ring attention forward in fp32 on the FMA pipes (no tensor cores: tf32 would
// round the inputs to 10 mantissa bits). One block = 64 query slots of one
// head; two threads per query row, each owning alternate 4-float chunks of D.
//
// The ring: the block's queries belong to rank i = slot / L. At step t they see
// the key/value block of owner r = (i - t) mod P ("Sequence Parallelism III:
// Ring Attention ...", duoan.github.io). Key tiles that the causal mask hides
// entirely are skipped ("DeDLOC Guide", Best Practices, Causal Mask Handling),
// and so are tiles outside every row's sliding window or document when those
// are set (axolotl-ringmaster README, Status); the online softmax runs on
// across step boundaries, which is the merge of the steps' partials ("DeDLOC
// Guide", section 3).
#include "common.cuh"
#include "internal.h"

namespace rm {

namespace {

constexpr int kRows = 64;   // query slots per block
constexpr int kKeys = 64;   // keys per tile
constexpr int kSub = 16;    // keys per online-softmax update

struct F32Args {
    const float* q;
    const float* k;
    const float* v;
    float* o;
    float* lse;
    int H, Hkv, S, P, causal;
    float scale;
    RingLayout lay;
    MaskSpec mk;  // which keys each query sees
};

template <int D>
__global__ void __launch_bounds__(128) fwd_fp32_kernel(const __grid_constant__ F32Args a) {
    constexpr int NC = D / 8;  // float4 chunks owned per thread
    extern __shared__ float4 smem4[];
    float4* Ks = smem4;                // [kKeys][D/4]
    float4* Vs = smem4 + kKeys * D / 4;
    const int row = threadIdx.x >> 1, half = threadIdx.x & 1;
    const int s0 = blockIdx.x * kRows;
    const int h = blockIdx.y, b = blockIdx.z, g = h / (a.H / a.Hkv);
    const int L = a.lay.L;
    const int rank = s0 / L;
    const int qpos0 = a.lay.pos_of_slot(s0);
    const int qpos = qpos0 + row;
    // key bounds of this row and of the block's first and last rows
    const int2 rb = row_bounds(a.mk, qpos);
    const int2 bf = row_bounds(a.mk, qpos0), bl = row_bounds(a.mk, qpos0 + kRows - 1);

    const float4* qrow =
        reinterpret_cast<const float4*>(a.q + ((static_cast<int64_t>(b) * a.H + h) * a.S + s0 + row) * D);
    float4 q[NC], o[NC];
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        q[j] = qrow[2 * j + half];
        o[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float m = -INFINITY, l = 0.f;
    const int64_t kv_head = (static_cast<int64_t>(b) * a.Hkv + g) * a.S;

    for (int t = 0; t < a.P; ++t) {
        const int r = a.lay.owner(rank, t);
        for (int u = 0; u < L / kKeys; ++u) {
            const int kslot = r * L + u * kKeys;
            const int kpos0 = a.lay.pos_of_slot(kslot);
            // no row sees a key of this tile: skip; every row sees all of it: no mask
            if (kpos0 > bl.y || kpos0 + kKeys - 1 < bf.x) continue;
            const bool full = kpos0 >= bl.x && kpos0 + kKeys - 1 <= bf.y;
            __syncthreads();
            const float4* kg = reinterpret_cast<const float4*>(a.k + (kv_head + kslot) * D);
            const float4* vg = reinterpret_cast<const float4*>(a.v + (kv_head + kslot) * D);
            for (int e = threadIdx.x; e < kKeys * D / 4; e += 128) {
                Ks[e] = kg[e];
                Vs[e] = vg[e];
            }
            __syncthreads();
            for (int kb = 0; kb < kKeys; kb += kSub) {
                float s[kSub];
                float mx = -INFINITY;
#pragma unroll
                for (int jj = 0; jj < kSub; ++jj) {
                    const float4* kr = Ks + (kb + jj) * (D / 4);
                    float acc = 0.f;
#pragma unroll
                    for (int j = 0; j < NC; ++j) {
                        const float4 kv = kr[2 * j + half];
                        acc = fmaf(q[j].x, kv.x, acc);
                        acc = fmaf(q[j].y, kv.y, acc);
                        acc = fmaf(q[j].z, kv.z, acc);
                        acc = fmaf(q[j].w, kv.w, acc);
                    }
                    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                    acc *= a.scale;
                    if (!full && (kpos0 + kb + jj < rb.x || kpos0 + kb + jj > rb.y)) acc = -INFINITY;
                    s[jj] = acc;
                    mx = fmaxf(mx, acc);
                }
                const float m_new = fmaxf(m, mx);
                if (m_new == -INFINITY) continue;  // nothing visible yet
                const float alpha = expf(m - m_new);
                l *= alpha;
#pragma unroll
                for (int j = 0; j < NC; ++j) {
                    o[j].x *= alpha; o[j].y *= alpha; o[j].z *= alpha; o[j].w *= alpha;
                }
#pragma unroll
                for (int jj = 0; jj < kSub; ++jj) {
                    const float p = expf(s[jj] - m_new);
                    l += p;
                    const float4* vr = Vs + (kb + jj) * (D / 4);
#pragma unroll
                    for (int j = 0; j < NC; ++j) {
                        const float4 vv = vr[2 * j + half];
                        o[j].x = fmaf(p, vv.x, o[j].x);
                        o[j].y = fmaf(p, vv.y, o[j].y);
                        o[j].z = fmaf(p, vv.z, o[j].z);
                        o[j].w = fmaf(p, vv.w, o[j].w);
                    }
                }
                m = m_new;
            }
        }
    }
    const float inv = l > 0.f ? 1.0f / l : 0.f;
    float4* orow =
        reinterpret_cast<float4*>(a.o + ((static_cast<int64_t>(b) * a.H + h) * a.S + s0 + row) * D);
#pragma unroll
    for (int j = 0; j < NC; ++j)
        orow[2 * j + half] = make_float4(o[j].x * inv, o[j].y * inv, o[j].z * inv, o[j].w * inv);
    if (half == 0)
        a.lse[(static_cast<int64_t>(b) * a.H + h) * a.S + s0 + row] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace

cudaError_t launch_fwd_fp32(const AttnShape& sh, const float* q, const float* k, const float* v,
                            float* o, float* lse, const LaunchCtx& ctx) {
    F32Args a{q, k, v, o, lse, sh.H, sh.Hkv, sh.S, sh.P, sh.causal, sh.scale,
              RingLayout{sh.S, sh.P, sh.S / sh.P, sh.zigzag ? sh.S / (2 * sh.P) : sh.S / sh.P,
                         sh.zigzag},
              MaskSpec{static_cast<const int4*>(sh.bounds), sh.S, sh.causal,
                       sh.causal ? sh.window : 0}};
    dim3 grid(sh.S / kRows, sh.H, sh.B);
    const size_t smem = 2 * static_cast<size_t>(kKeys) * sh.D * sizeof(float);
    if (sh.D == 64) {
        fwd_fp32_kernel<64><<<grid, 128, smem, ctx.stream>>>(a);
    } else {
        cudaError_t e = cudaFuncSetAttribute(fwd_fp32_kernel<128>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        fwd_fp32_kernel<128><<<grid, 128, smem, ctx.stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace rm
