// rma_decode: one decode token per sequence at one RMA layer.
//
// Computes, per sequence b, KV group g and query head h of g
// ("EdgeRock" model card, "How Rock Memory Anchors work"; ai-primer story
// "EdgeRock-4B fixes its attention KV cache at 72 MiB", operations 1-3):
//   local_h  = softmax over the window (ring rows [0, min(pos, R)) + current token)
//   anchor_h = softmax over the committed bank rows [0, bank_fill)
//   out_h    = local_h + tanh(q_h . w_g[h] + b_g[h]) * anchor_h
// then writes the current K/V into ring slot pos mod R and appends the
// candidate record to the pending buffer.
//
// Design (HBM-bound; ~2 FMA per byte streamed):
//   grid = (ring_splits + bank_splits, G, B).  Each CTA streams one contiguous
//   row range of one (b, g)'s ring or bank.  Rows are processed in tiles of 4;
//   warp w takes tiles w, w + W, w + 2W, ... and runs its OWN cp.async
//   pipeline (each lane copies, and later reads, exactly its own 16-byte
//   column of each row, so no block barrier is needed while streaming).
//   A lane holds 8 of the 256 dims for all 4 heads: QK^T is 32 FMAs per row
//   per lane, reduced across lanes by a 16-value reduce-scatter (16 shuffles
//   per 4 rows); the online softmax (log2 domain) and P.V run in FP32 with
//   packed FFMA2.  Warps merge in shared memory into one (m, l, acc) partial
//   per CTA; the last CTA of (b, g) to arrive (atomic ticket, no waiting)
//   merges all partials, adds the current token and the gate, writes the
//   output and performs the state writes after every read of the step; when
//   the step fills the pending buffer it also runs the admit for (b, g).
#include <cuda_bf16.h>
#include <math_constants.h>

#include <mutex>

#include "rma_admit_impl.cuh"
#include "rma_internal.cuh"

namespace rma {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 3;
constexpr int kTileRows = 4;
constexpr int kStageBytes = 2 * kTileRows * kRowBytes;          // K tile + V tile = 4 KiB
constexpr int kPipeBytes = kWarps * kStages * kStageBytes;       // 96 KiB
constexpr int kBcastFloats = 32;                                 // per warp: 16 p + 4 alpha (+pad)
constexpr int kMaxSplits = 64;                                   // ring_splits + bank_splits
constexpr int kSmemBytes = kPipeBytes + kWarps * kBcastFloats * 4 + (kMaxSplits + 1) * 4 * 4 + 16 * 4;

static_assert(kWarps == 8, "merger assigns 8 dot products to 8 warps");
static_assert(kStages * kStageBytes >= kPartialFloats * 4, "per-warp pipeline region must hold one warp partial");
static_assert(kPipeBytes >= admit_scratch_bytes(1, 4095), "the admit reuses the pipeline region (any A + P <= 4096)");

__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__device__ __forceinline__ float fast_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float dot8(const float2 (&q)[4], const uint4& k) {
    float2 d = __fmul2_rn(q[0], bf2_to_f2(k.x));
    d = __ffma2_rn(q[1], bf2_to_f2(k.y), d);
    d = __ffma2_rn(q[2], bf2_to_f2(k.z), d);
    d = __ffma2_rn(q[3], bf2_to_f2(k.w), d);
    return d.x + d.y;
}

// Reduce 16 per-lane partial sums across the warp so that lane L ends up
// with the full sum of value index (L >> 1) & 15 (lanes L and L^1 agree).
__device__ __forceinline__ float reduce_scatter16(float (&x)[16], int lane) {
    {
        const bool up = lane & 16;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float send = up ? x[i] : x[i + 8];
            float keep = up ? x[i + 8] : x[i];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
    }
    {
        const bool up = lane & 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float send = up ? x[i] : x[i + 4];
            float keep = up ? x[i + 4] : x[i];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
    }
    {
        const bool up = lane & 4;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float send = up ? x[i] : x[i + 2];
            float keep = up ? x[i + 2] : x[i];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
        }
    }
    {
        const bool up = lane & 2;
        float send = up ? x[0] : x[1];
        float keep = up ? x[1] : x[0];
        x[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    return x[0] + __shfl_xor_sync(0xffffffffu, x[0], 1);
}

__global__ void __launch_bounds__(kThreads, 2) decode_kernel(const __grid_constant__ DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.s.G;
    const int bg = b * G + g;
    const int n_splits = a.ring_splits + a.bank_splits;

    const int32_t* cnt = a.s.counters + bg * 4;
    int pos = cnt[0], bank_fill = cnt[1], pend_fill = cnt[2];
    if (pos < 0 || bank_fill < 0 || bank_fill > a.s.A || pend_fill < 0 || pend_fill > a.s.P) {
        // a corrupted state: never index outside the buffers
        if (threadIdx.x == 0 && split == 0) atomicOr(a.s.status, (unsigned)RMA_STATUS_BAD_COUNTERS);
        pos = max(pos, 0);
        bank_fill = min(max(bank_fill, 0), a.s.A);
        pend_fill = min(max(pend_fill, 0), a.s.P);
    }

    // ---- this CTA's row range ----
    const bool is_bank = split >= a.ring_splits;
    int nrows;
    const uint16_t* kbase;
    const uint16_t* vbase;
    if (!is_bank) {
        const int fill = min(pos, a.s.R);
        const int row0 = split * a.ring_chunk;
        nrows = max(0, min(a.ring_chunk, fill - row0));
        const size_t off = ((size_t)bg * a.s.R + row0) * kHeadDim;
        kbase = a.s.ring_k + off;
        vbase = a.s.ring_v + off;
    } else {
        const int row0 = (split - a.ring_splits) * a.bank_chunk;
        nrows = max(0, min(a.bank_chunk, bank_fill - row0));
        const size_t off = ((size_t)bg * a.s.A + row0) * kHeadDim;
        kbase = a.s.bank_k + off;
        vbase = a.s.bank_v + off;
    }

    // ---- per-warp cp.async pipeline over this warp's tiles ----
    uint8_t* wsm = smem + warp * (kStages * kStageBytes);
    const uint32_t wsm_a = smem_addr(wsm);
    float* bc = reinterpret_cast<float*>(smem + kPipeBytes) + warp * kBcastFloats;
    const int n_tiles = (nrows + kTileRows - 1) / kTileRows;
    const int my_n = n_tiles > warp ? (n_tiles - warp + kWarps - 1) / kWarps : 0;

    auto issue = [&](int i, int stage) {
        const int t = warp + i * kWarps;
        const uint32_t dst = wsm_a + stage * kStageBytes + lane * 16;
#pragma unroll
        for (int j = 0; j < kTileRows; ++j) {
            const int r = t * kTileRows + j;
            const bool ok = r < nrows;
            const size_t roff = (size_t)(ok ? r : 0) * kHeadDim + lane * 8;
            cp_async16(dst + j * kRowBytes, kbase + roff, ok ? 16 : 0);
            cp_async16(dst + (kTileRows + j) * kRowBytes, vbase + roff, ok ? 16 : 0);
        }
    };

#pragma unroll
    for (int s = 0; s < kStages; ++s) {
        if (s < my_n) issue(s, s);
        cp_commit();
    }

    // ---- q of the group's 4 heads, this lane's 8 dims, in the log2 domain (loaded while the
    //      first K/V tiles are in flight) ----
    float2 q2[kQPerGroup][4];
    const uint16_t* qg = a.q + ((size_t)b * G * kQPerGroup + (size_t)g * kQPerGroup) * kHeadDim;
#pragma unroll
    for (int h = 0; h < kQPerGroup; ++h) {
        const uint4 r = ld_nc_v4(qg + h * kHeadDim + lane * 8);
        const float2 s2 = make_float2(a.qscale, a.qscale);
        q2[h][0] = __fmul2_rn(bf2_to_f2(r.x), s2);
        q2[h][1] = __fmul2_rn(bf2_to_f2(r.y), s2);
        q2[h][2] = __fmul2_rn(bf2_to_f2(r.z), s2);
        q2[h][3] = __fmul2_rn(bf2_to_f2(r.w), s2);
    }


    float m_run = -CUDART_INF_F, l_run = 0.f;
    float2 acc[kQPerGroup][4];
#pragma unroll
    for (int h = 0; h < kQPerGroup; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[h][i] = make_float2(0.f, 0.f);

    const int my_j = (lane >> 3) & 3;   // row of the tile this lane's reduced score belongs to
    const int my_h = (lane >> 1) & 3;   // head of this lane's reduced score

    for (int i = 0; i < my_n; ++i) {
        cp_wait<kStages - 1>();
        const int stage = i % kStages;
        const uint8_t* ks = wsm + stage * kStageBytes + lane * 16;
        const uint8_t* vs = ks + kTileRows * kRowBytes;

        float x[16];
#pragma unroll
        for (int j = 0; j < kTileRows; ++j) {
            const uint4 kr = *reinterpret_cast<const uint4*>(ks + j * kRowBytes);
#pragma unroll
            for (int h = 0; h < kQPerGroup; ++h) x[j * 4 + h] = dot8(q2[h], kr);
        }
        float sc = reduce_scatter16(x, lane);
        const int row = (warp + i * kWarps) * kTileRows + my_j;
        if (row >= nrows) sc = -CUDART_INF_F;

        float mx = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_run, mx);
        const float m_use = (m_new == -CUDART_INF_F) ? 0.f : m_new;
        const float alpha = fast_ex2(m_run - m_use);
        const float p = fast_ex2(sc - m_use);
        float ps = p + __shfl_xor_sync(0xffffffffu, p, 8);
        ps += __shfl_xor_sync(0xffffffffu, ps, 16);
        l_run = l_run * alpha + ps;
        m_run = m_new;

        __syncwarp();
        if ((lane & 1) == 0) bc[(lane >> 1) & 15] = p;
        if ((lane & 0x19) == 0) bc[16 + my_h] = alpha;
        __syncwarp();
        const float4 al = *reinterpret_cast<const float4*>(bc + 16);
        const float alv[4] = {al.x, al.y, al.z, al.w};
#pragma unroll
        for (int h = 0; h < kQPerGroup; ++h) {
            const float2 a2 = make_float2(alv[h], alv[h]);
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[h][c] = __fmul2_rn(acc[h][c], a2);
        }
#pragma unroll
        for (int j = 0; j < kTileRows; ++j) {
            const float4 pj = *reinterpret_cast<const float4*>(bc + 4 * j);
            const float pv[4] = {pj.x, pj.y, pj.z, pj.w};
            const uint4 vr = *reinterpret_cast<const uint4*>(vs + j * kRowBytes);
            const float2 v0 = bf2_to_f2(vr.x), v1 = bf2_to_f2(vr.y), v2 = bf2_to_f2(vr.z), v3 = bf2_to_f2(vr.w);
#pragma unroll
            for (int h = 0; h < kQPerGroup; ++h) {
                const float2 p2 = make_float2(pv[h], pv[h]);
                acc[h][0] = __ffma2_rn(p2, v0, acc[h][0]);
                acc[h][1] = __ffma2_rn(p2, v1, acc[h][1]);
                acc[h][2] = __ffma2_rn(p2, v2, acc[h][2]);
                acc[h][3] = __ffma2_rn(p2, v3, acc[h][3]);
            }
        }
        if (i + kStages < my_n) issue(i + kStages, stage);
        cp_commit();
    }
    cp_wait<0>();

    // ---- merge the warps of this CTA (each warp's pipeline region holds its partial) ----
    float* wpart = reinterpret_cast<float*>(wsm);
    if ((lane & 0x19) == 0) {
        wpart[my_h] = m_run;
        wpart[4 + my_h] = l_run;
    }
#pragma unroll
    for (int h = 0; h < kQPerGroup; ++h) {
        float4* dst = reinterpret_cast<float4*>(wpart + 8 + h * kHeadDim + lane * 8);
        dst[0] = make_float4(acc[h][0].x, acc[h][0].y, acc[h][1].x, acc[h][1].y);
        dst[1] = make_float4(acc[h][2].x, acc[h][2].y, acc[h][3].x, acc[h][3].y);
    }
    __syncthreads();

    float* part = a.ws + ((size_t)bg * n_splits + split) * kPartialFloats;
    {
        const int h = tid >> 6;                 // 256 threads x 4 elements = 4 heads x 256 dims
        const int d = (tid & 63) * 4;
        float mw[kWarps];
        float M = -CUDART_INF_F;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            mw[w] = reinterpret_cast<const float*>(smem + w * (kStages * kStageBytes))[h];
            M = fmaxf(M, mw[w]);
        }
        const float Mu = (M == -CUDART_INF_F) ? 0.f : M;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float* wp = reinterpret_cast<const float*>(smem + w * (kStages * kStageBytes));
            const float c = fast_ex2(mw[w] - Mu);
            L += c * wp[4 + h];
            const float4 v = *reinterpret_cast<const float4*>(wp + 8 + h * kHeadDim + d);
            o.x += c * v.x; o.y += c * v.y; o.z += c * v.z; o.w += c * v.w;
        }
        *reinterpret_cast<float4*>(part + 8 + h * kHeadDim + d) = o;
        if ((tid & 63) == 0) {
            part[h] = M;
            part[4 + h] = L;
        }
    }
    __threadfence();
    __syncthreads();

    __shared__ int s_last;
    if (tid == 0) {
        const unsigned prev = atomicAdd(a.s.tickets + bg, 1u);
        s_last = (prev == (unsigned)(n_splits - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // ---- last CTA of (b, g): merge every split, add the current token, gate, write ----
    float* coef = reinterpret_cast<float*>(smem + kPipeBytes + kWarps * kBcastFloats * 4);  // [(n_splits+1)][4]
    float* misc = coef + (kMaxSplits + 1) * 4;                                             // scur[4], gate[4]
    const uint16_t* kc = a.k_cur + (size_t)bg * kHeadDim;
    const uint16_t* vc = a.v_cur + (size_t)bg * kHeadDim;
    const float* parts = a.ws + (size_t)bg * n_splits * kPartialFloats;
    // Every load the merge needs is issued before any of its results is used, so that the
    // merging CTA pays one L2 round trip instead of a chain of them: this thread's q / k_cur /
    // w_g pieces, every split's maxima and sums (into shared memory; the pipeline region is
    // free now) and the first 16 splits' accumulators for its 4 output dims.
    const int oh = tid >> 6, od = (tid & 63) * 4;          // this thread's output head and dims
    const float* pacc = parts + 8 + oh * kHeadDim + od;
    float4 pre[16];
#pragma unroll
    for (int u = 0; u < 16; ++u)
        if (u < n_splits) pre[u] = __ldcg(reinterpret_cast<const float4*>(pacc + (size_t)u * kPartialFloats));
    const int mh = warp & 3;                                // this warp's head for s_cur / gate
    const int head = g * kQPerGroup + mh;
    const uint4 qr = ld_nc_v4(qg + mh * kHeadDim + lane * 8);
    uint4 kr = make_uint4(0, 0, 0, 0);
    float4 w0 = make_float4(0.f, 0.f, 0.f, 0.f), w1 = w0;
    if (warp < 4) {
        kr = ld_nc_v4(kc + lane * 8);
    } else {
        w0 = __ldg(reinterpret_cast<const float4*>(a.w_g + (size_t)head * kHeadDim + lane * 8));
        w1 = __ldg(reinterpret_cast<const float4*>(a.w_g + (size_t)head * kHeadDim + lane * 8 + 4));
    }
    float* pml = reinterpret_cast<float*>(smem);   // [n_splits][8]
    for (int i = tid; i < n_splits * 8; i += kThreads)
        pml[i] = __ldcg(parts + (size_t)(i >> 3) * kPartialFloats + (i & 7));
    if (warp < 4) {
        // s_cur[h] = scale * log2(e) * q_h . k_cur
        const float2 s2 = make_float2(a.qscale, a.qscale);
        const float2 qh[4] = {__fmul2_rn(bf2_to_f2(qr.x), s2), __fmul2_rn(bf2_to_f2(qr.y), s2),
                              __fmul2_rn(bf2_to_f2(qr.z), s2), __fmul2_rn(bf2_to_f2(qr.w), s2)};
        const float sc = warp_sum(dot8(qh, kr));
        if (lane == 0) misc[mh] = sc;
    } else {
        // gate[h] = tanh(q_h . w_g[head] + b_g[head]), with the unscaled query
        const float2 q0 = bf2_to_f2(qr.x), q1 = bf2_to_f2(qr.y), qq2 = bf2_to_f2(qr.z), q3 = bf2_to_f2(qr.w);
        float dg = q0.x * w0.x + q0.y * w0.y + q1.x * w0.z + q1.y * w0.w +
                   qq2.x * w1.x + qq2.y * w1.y + q3.x * w1.z + q3.y * w1.w;
        dg = warp_sum(dg);
        if (lane == 0) misc[4 + mh] = tanhf(dg + a.b_g[head]);
    }
    __syncthreads();

    // Coefficients: warp w takes head w & 3 of the local softmax (ring splits and the current
    // token, w < 4) or of the anchor softmax (bank splits, scaled by the gate, w >= 4); its
    // lanes take the splits.
    {
        const int h = warp & 3;
        const bool local = warp < 4;
        const int sp0 = local ? 0 : a.ring_splits, sp1 = local ? a.ring_splits : n_splits;
        const float scur = misc[h];
        float M = local ? scur : -CUDART_INF_F;
        for (int sp = sp0 + lane; sp < sp1; sp += 32) M = fmaxf(M, pml[sp * 8 + h]);
        M = warp_max(M);
        const float Mu = (M == -CUDART_INF_F) ? 0.f : M;
        float L = 0.f;
        for (int sp = sp0 + lane; sp < sp1; sp += 32) L += fast_ex2(pml[sp * 8 + h] - Mu) * pml[sp * 8 + 4 + h];
        L = warp_sum(L);
        float scale;
        if (local) {
            L += fast_ex2(scur - Mu);
            scale = 1.f / L;
        } else {
            scale = (L > 0.f) ? misc[4 + h] / L : 0.f;
        }
        for (int sp = sp0 + lane; sp < sp1; sp += 32) coef[sp * 4 + h] = fast_ex2(pml[sp * 8 + h] - Mu) * scale;
        if (local && lane == 0) coef[n_splits * 4 + h] = fast_ex2(scur - Mu) * scale;
    }
    __syncthreads();

    {
        const int h = oh, d = od;
        const float cc = coef[n_splits * 4 + h];
        const uint2 vr = *reinterpret_cast<const uint2*>(vc + d);
        const float2 va = bf2_to_f2(vr.x), vb = bf2_to_f2(vr.y);
        float4 o = make_float4(cc * va.x, cc * va.y, cc * vb.x, cc * vb.y);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            if (u < n_splits) {
                const float c = coef[u * 4 + h];
                o.x += c * pre[u].x; o.y += c * pre[u].y; o.z += c * pre[u].z; o.w += c * pre[u].w;
            }
        }
        // the remaining splits' accumulators, sixteen loads in flight at a time (same summation order)
        int sp = 16;
        for (; sp + 16 <= n_splits; sp += 16) {
            float4 v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] = __ldcg(reinterpret_cast<const float4*>(pacc + (size_t)(sp + u) * kPartialFloats));
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const float c = coef[(sp + u) * 4 + h];
                o.x += c * v[u].x; o.y += c * v[u].y; o.z += c * v[u].z; o.w += c * v[u].w;
            }
        }
        for (; sp < n_splits; ++sp) {
            const float c = coef[sp * 4 + h];
            const float4 v = __ldcg(reinterpret_cast<const float4*>(pacc + (size_t)sp * kPartialFloats));
            o.x += c * v.x; o.y += c * v.y; o.z += c * v.z; o.w += c * v.w;
        }
        const __nv_bfloat162 o01 = __floats2bfloat162_rn(o.x, o.y);
        const __nv_bfloat162 o23 = __floats2bfloat162_rn(o.z, o.w);
        uint2 packed;
        packed.x = *reinterpret_cast<const uint32_t*>(&o01);
        packed.y = *reinterpret_cast<const uint32_t*>(&o23);
        const int ohead = g * kQPerGroup + h;
        *reinterpret_cast<uint2*>(a.out + ((size_t)b * G * kQPerGroup + ohead) * kHeadDim + d) = packed;
    }

    // ---- state writes: every split of (b, g) has finished reading ----
    const int slot = pos % a.s.R;
    const bool room = pend_fill < a.s.P;
    if (tid < 32) {
        reinterpret_cast<uint4*>(a.s.ring_k + ((size_t)bg * a.s.R + slot) * kHeadDim)[lane] =
            ld_nc_v4(kc + lane * 8);
    } else if (tid < 64) {
        reinterpret_cast<uint4*>(a.s.ring_v + ((size_t)bg * a.s.R + slot) * kHeadDim)[lane] =
            ld_nc_v4(vc + lane * 8);
    } else if (tid < 96) {
        if (room)
            reinterpret_cast<uint4*>(a.s.pend_k + ((size_t)bg * a.s.P + pend_fill) * kHeadDim)[lane] =
                ld_nc_v4(a.cand_k + (size_t)bg * kHeadDim + lane * 8);
    } else if (tid < 128) {
        if (room)
            reinterpret_cast<uint4*>(a.s.pend_v + ((size_t)bg * a.s.P + pend_fill) * kHeadDim)[lane] =
                ld_nc_v4(a.cand_v + (size_t)bg * kHeadDim + lane * 8);
    } else if (tid == 128) {
        if (room) a.s.pend_score[(size_t)bg * a.s.P + pend_fill] = a.cand_score[bg];
        else atomicOr(a.s.status, (unsigned)RMA_STATUS_PENDING_OVERFLOW);
        int32_t* c = a.s.counters + bg * 4;
        c[0] = pos + 1;
        c[2] = room ? pend_fill + 1 : pend_fill;
        a.s.tickets[bg] = 0u;
    }

    // ---- the admit, in this launch, when this step filled the pending buffer ----
    // Every split of (b, g) has finished reading the bank, so the bank may change now.
    if (room && pend_fill + 1 == a.s.P) {
        __syncthreads();   // the appended candidate and counters are visible to the whole CTA
        admit_group<kThreads>(a.s, bg, bank_fill, a.s.P, smem);
    }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    static SmemLimit limit(reinterpret_cast<const void*>(decode_kernel));
    const cudaError_t e = limit.ensure(kSmemBytes);
    if (e != cudaSuccess) return e;
    if (a.ring_splits + a.bank_splits > kMaxSplits) return cudaErrorInvalidValue;
    dim3 grid(a.ring_splits + a.bank_splits, a.s.G, a.s.B);
    decode_kernel<<<grid, kThreads, kSmemBytes, stream>>>(a);
    return cudaGetLastError();
}

int decode_max_splits() { return kMaxSplits; }

// ---------------------------------------------------------------------------
// Built-in decode scratch, for callers that cannot allocate device memory.
// A fixed 32 MiB array in the library's device image: every GPU that loads
// the library holds it until the process exits.  Host code must not pass the
// array's name to a kernel (on the host it is only a stand-in symbol); its
// device address is looked up once per device with cudaGetSymbolAddress,
// with that device current, and cached.  All calls on a device share it.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticDecodeScratchBytes];

cudaError_t static_decode_scratch(void** ptr) {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *ptr = addr[dev];
    return cudaSuccess;
}

}  // namespace rma
