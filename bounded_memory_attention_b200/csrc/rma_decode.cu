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
// Design (HBM-bound: every K/V byte is read once, ~2 FLOP per byte):
//   grid = (ring_splits + bank_splits, G, B).  Each CTA streams one contiguous
//   row range of one (b, g)'s ring or bank in tiles of 16 rows.  Warp w takes
//   tiles w, w + 8, w + 16, ... with its own K slot and V slot in shared
//   memory: the lanes copy a tile's rows with one 512-byte bulk copy each
//   (completion counted on the slot's mbarrier) into rows padded to 528 bytes,
//   so that the tensor-core fragment loads below are free of bank conflicts.
//   The next tile's K is requested as soon as this tile's Q K^T has read its
//   K slot, its V as soon as P V has read the V slot.
//   Both products run on the tensor cores (mma.sync m16n8k16, BF16 operands,
//   FP32 accumulation), with the 16 keys of the tile in M and the group's
//   heads in N (4 of the 8 columns used):
//     S^T [16 keys x 8]  = K [16 x 256] . Q^T [256 x 8]     (K from ldmatrix)
//     O^T [256 x 8]     += V^T [256 x 16] . P^T [16 x 8]    (V from ldmatrix.trans)
//   The softmax runs on S^T in registers (log2 domain, FP32; the running max
//   moves, and O is rescaled, only when a tile raises it); P is rounded to
//   BF16 and turned from the S^T accumulator layout into the P^T operand
//   layout with movmatrix.  Warps merge in shared memory into one (m, l, acc)
//   partial per CTA; the last CTA of (b, g) to arrive (atomic ticket, no
//   waiting) merges all partials, adds the current token and the gate, writes
//   the output and performs the state writes after every read of the step;
//   when the step fills the pending buffer it also runs the admit for (b, g).
#include <cuda_bf16.h>
#include <math_constants.h>

#include "rma_admit_impl.cuh"
#include "rma_internal.cuh"
#include "sm100_ptx.cuh"

namespace rma {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTile = 16;                                        // keys per tensor-core tile
constexpr int kRowStride = kRowBytes + 16;                       // 528: padded shared-memory row
constexpr int kSlotBytes = kTile * kRowStride;                   // 8,448: one K or V tile
constexpr int kWarpRegion = 2 * kSlotBytes;                      // this warp's K slot + V slot
constexpr int kPipeBytes = kWarps * kWarpRegion;                 // 135,168
constexpr int kMaxSplits = 64;                                   // ring_splits + bank_splits
constexpr int kCoefOff = kPipeBytes;                             // [(kMaxSplits + 1)][4] floats
constexpr int kMiscOff = kCoefOff + (kMaxSplits + 1) * 4 * 4;    // scur[4], gate[4] (+ pad)
constexpr int kBarOff = kMiscOff + 16 * 4;                       // [kWarps][2] mbarriers
constexpr int kSmemBytes = kBarOff + kWarps * 2 * 8;

static_assert(kWarps == 8, "merger assigns 8 dot products to 8 warps");
static_assert(kSlotBytes >= kPartialFloats * 4, "a warp's K slot must hold one warp partial");
static_assert(kPipeBytes >= (int)admit_scratch_bytes(1, 4095), "the admit reuses the pipeline region (any A + P <= 4096)");
static_assert((kBarOff & 7) == 0, "mbarriers are 8-byte aligned");

__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__device__ __forceinline__ float fast_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t ld_nc_u32(const void* p) {
    uint32_t r;
    asm volatile("ld.global.nc.u32 %0, [%1];\n" : "=r"(r) : "l"(p));
    return r;
}

// `bytes` (a multiple of 16) from global memory to this CTA's shared memory, counted as tx
// bytes on the mbarrier `bar`; a plain copy into this CTA (no multicast).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// Four 8x8 BF16 matrices from shared memory (lane L gives the address of row L & 7 of matrix L >> 3).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

// D (16x8 FP32) += A (16x16 BF16, row) . B (16x8 BF16, col)
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Transpose an 8x8 matrix of 16-bit values held one row pair per lane in the mma fragment layout.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
    return y;
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

// Bounded wait on an mbarrier phase (about two seconds); on timeout sets RMA_STATUS_TIMEOUT and
// returns false.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, uint32_t* status) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > ptx::kWaitLimitCycles) {
            atomicOr(status, (unsigned)RMA_STATUS_TIMEOUT);
            return false;
        }
    }
    return true;
}

__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.s.G;
    const int bg = b * G + g;
    const int n_splits = a.ring_splits + a.bank_splits;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
    if (tid < 2 * kWarps) ptx::mbar_init(&bars[tid], 1);
    ptx::fence_mbar_init();

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
    __syncthreads();   // the mbarriers are initialised

    // ---- this warp's tiles: w, w + 8, ...; K slot and V slot, one mbarrier each ----
    uint8_t* wsm = smem + warp * kWarpRegion;
    const uint32_t kslot = ptx::smem_u32(wsm), vslot = kslot + kSlotBytes;
    uint64_t* kbar = &bars[2 * warp];
    uint64_t* vbar = &bars[2 * warp + 1];
    const int n_tiles = (nrows + kTile - 1) / kTile;
    const int my_n = n_tiles > warp ? (n_tiles - warp + kWarps - 1) / kWarps : 0;

    // rows of tile i of this warp -> one slot: lane r < rows copies row r (512 bytes)
    auto issue = [&](int i, bool v_half) {
        const int r0 = (warp + i * kWarps) * kTile;
        const int nv = min(kTile, nrows - r0);
        uint64_t* bar = v_half ? vbar : kbar;
        if (lane == 0) ptx::mbar_arrive_expect_tx(bar, (uint32_t)(nv * kRowBytes));
        __syncwarp();
        if (lane < nv)
            bulk_g2s((v_half ? vslot : kslot) + lane * kRowStride, (v_half ? vbase : kbase) + (size_t)(r0 + lane) * kHeadDim,
                     kRowBytes, ptx::smem_u32(bar));
    };
    if (my_n > 0) {
        issue(0, false);
        issue(0, true);
    }

    // ---- Q^T fragments (the B operand of S^T = K Q^T), loaded while the first tiles are in flight:
    //      lane (gq = lane / 4, tq = lane % 4) holds head gq's dims 16 c + 2 tq (+1) and 16 c + 2 tq + 8 (+9);
    //      heads 4..7 of the 8 columns are zero ----
    const int gq = lane >> 2, tq = lane & 3;
    const uint16_t* qg = a.q + ((size_t)b * G * kQPerGroup + (size_t)g * kQPerGroup) * kHeadDim;
    uint32_t qf[16][2];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        qf[c][0] = gq < kQPerGroup ? ld_nc_u32(qg + gq * kHeadDim + 16 * c + 2 * tq) : 0u;
        qf[c][1] = gq < kQPerGroup ? ld_nc_u32(qg + gq * kHeadDim + 16 * c + 2 * tq + 8) : 0u;
    }

    // ldmatrix row addresses: lane L feeds row L & 7 of matrix L >> 3
    const int lr = lane & 7, lm = lane >> 3;
    // K (A operand, rows = keys): matrices (keys 0-7 | 8-15) x (dims +0-7 | +8-15)
    const uint32_t k_addr = kslot + (uint32_t)((lr + 8 * (lm & 1)) * kRowStride + 16 * (lm >> 1));
    // V^T (A operand via .trans, rows = dims): matrices (dims +0-7 | +8-15) x (keys 0-7 | 8-15)
    const uint32_t v_addr = vslot + (uint32_t)((lr + 8 * (lm >> 1)) * kRowStride + 16 * (lm & 1));

    // running softmax of heads 2 tq and 2 tq + 1 (lanes with tq >= 2 carry the unused columns)
    float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.f, l1 = 0.f;
    float acc[16][4];
#pragma unroll
    for (int mt = 0; mt < 16; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    const float qs = a.qscale;
    bool ok = true;
    int k_issued = my_n > 0 ? 1 : 0, v_issued = k_issued;

    for (int i = 0; i < my_n && ok; ++i) {
        const int r0 = (warp + i * kWarps) * kTile;
        const int nv = min(kTile, nrows - r0);
        // ---- S^T = K Q^T: 16 MMAs in four independent chains ----
        if (!wait_phase(kbar, i & 1, a.s.status)) { ok = false; break; }
        float s[4][4];
#pragma unroll
        for (int c = 0; c < 4; ++c) s[c][0] = s[c][1] = s[c][2] = s[c][3] = 0.f;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            uint32_t af[4];
            ldsm_x4(k_addr + 32 * c, af);
            mma_16816(s[c & 3], af, qf[c][0], qf[c][1]);
        }
        __syncwarp();
        if (i + 1 < my_n) {   // the K slot has been read: request the next tile's K
            issue(i + 1, false);
            ++k_issued;
        }
        // ---- softmax on S^T: x0 = (key gq, head 2tq), x1 = (gq, 2tq+1), x2 = (gq+8, 2tq), x3 = (gq+8, 2tq+1) ----
        const bool va = gq < nv, vb = gq + 8 < nv;
        const float x0 = va ? ((s[0][0] + s[1][0]) + (s[2][0] + s[3][0])) * qs : -CUDART_INF_F;
        const float x1 = va ? ((s[0][1] + s[1][1]) + (s[2][1] + s[3][1])) * qs : -CUDART_INF_F;
        const float x2 = vb ? ((s[0][2] + s[1][2]) + (s[2][2] + s[3][2])) * qs : -CUDART_INF_F;
        const float x3 = vb ? ((s[0][3] + s[1][3]) + (s[2][3] + s[3][3])) * qs : -CUDART_INF_F;
        float t0 = fmaxf(x0, x2), t1 = fmaxf(x1, x3);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, o));
            t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, o));
        }
        const bool up0 = t0 > m0, up1 = t1 > m1;
        if (__any_sync(0xffffffffu, up0 || up1)) {
            // the running max grew: rescale what this lane holds of those heads
            const float f0 = up0 ? (m0 == -CUDART_INF_F ? 0.f : fast_ex2(m0 - t0)) : 1.f;
            const float f1 = up1 ? (m1 == -CUDART_INF_F ? 0.f : fast_ex2(m1 - t1)) : 1.f;
            m0 = up0 ? t0 : m0;
            m1 = up1 ? t1 : m1;
            l0 *= f0;
            l1 *= f1;
#pragma unroll
            for (int mt = 0; mt < 16; ++mt) {
                acc[mt][0] *= f0;
                acc[mt][1] *= f1;
                acc[mt][2] *= f0;
                acc[mt][3] *= f1;
            }
        }
        const float p0 = fast_ex2(x0 - m0), p1 = fast_ex2(x1 - m1);
        const float p2 = fast_ex2(x2 - m0), p3 = fast_ex2(x3 - m1);
        l0 += p0 + p2;
        l1 += p1 + p3;
        // P^T operand (k = key, n = head): transpose the two 8x8 BF16 blocks of P^T's rows
        const uint32_t pb0 = movmatrix_trans(pack_bf16(p0, p1));
        const uint32_t pb1 = movmatrix_trans(pack_bf16(p2, p3));
        // ---- O^T += V^T P^T: 16 MMAs, one per 16 dims ----
        if (!wait_phase(vbar, i & 1, a.s.status)) { ok = false; break; }
        if (nv < kTile) {
            // rows past the range hold stale bytes: zero them so that 0 x stale stays 0
            for (int e = lane; e < (kTile - nv) * (kRowBytes / 16); e += 32)
                *reinterpret_cast<uint4*>(wsm + kSlotBytes + (nv + e / (kRowBytes / 16)) * kRowStride +
                                          16 * (e % (kRowBytes / 16))) = make_uint4(0, 0, 0, 0);
            __syncwarp();
        }
#pragma unroll
        for (int mt = 0; mt < 16; ++mt) {
            uint32_t af[4];
            ldsm_x4_trans(v_addr + 32 * mt, af);
            mma_16816(acc[mt], af, pb0, pb1);
        }
        __syncwarp();
        if (i + 1 < my_n) {   // the V slot has been read: request the next tile's V
            issue(i + 1, true);
            ++v_issued;
        }
    }
    if (!ok) {
        // a wait ran out: let the copies this warp already requested land before its slots are reused
        if (k_issued > 0) wait_phase(kbar, (k_issued - 1) & 1, a.s.status);
        if (v_issued > 0) wait_phase(vbar, (v_issued - 1) & 1, a.s.status);
    }
    // row sums over the 8 key rows of the fragment
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }

    // ---- this warp's partial (m, l, acc) into its K slot: lanes with tq < 2 hold heads 0..3 ----
    __syncwarp();
    float* wpart = reinterpret_cast<float*>(wsm);
    if (tq < 2) {
        const int h0 = 2 * tq, h1 = 2 * tq + 1;
        if (gq == 0) {
            wpart[h0] = m0;
            wpart[h1] = m1;
            wpart[4 + h0] = l0;
            wpart[4 + h1] = l1;
        }
#pragma unroll
        for (int mt = 0; mt < 16; ++mt) {
            wpart[8 + h0 * kHeadDim + 16 * mt + gq] = acc[mt][0];
            wpart[8 + h1 * kHeadDim + 16 * mt + gq] = acc[mt][1];
            wpart[8 + h0 * kHeadDim + 16 * mt + gq + 8] = acc[mt][2];
            wpart[8 + h1 * kHeadDim + 16 * mt + gq + 8] = acc[mt][3];
        }
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
            mw[w] = reinterpret_cast<const float*>(smem + w * kWarpRegion)[h];
            M = fmaxf(M, mw[w]);
        }
        const float Mu = (M == -CUDART_INF_F) ? 0.f : M;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float* wp = reinterpret_cast<const float*>(smem + w * kWarpRegion);
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
    float* coef = reinterpret_cast<float*>(smem + kCoefOff);   // [(n_splits+1)][4]
    float* misc = reinterpret_cast<float*>(smem + kMiscOff);   // scur[4], gate[4]
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
// device address is looked up with cudaGetSymbolAddress, on every call, in
// the CUDA context current on the calling thread (so a device reset or a
// second context on the same device never sees a stale address).  All calls
// on a device share it.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticDecodeScratchBytes];

cudaError_t static_decode_scratch(void** ptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    *ptr = p;
    return cudaSuccess;
}

}  // namespace rma
