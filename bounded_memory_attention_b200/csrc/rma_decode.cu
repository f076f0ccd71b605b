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
//
// FP8 storage (a state with kv_format RMA_KV_FP8_E4M3): the same structure on
// E4M3 codes and per-row power-of-two scale exponents.  A tile's 16 K rows
// and 16 V rows (256 bytes each, contiguous in the state) arrive with one bulk
// copy each, plus one for each set of 16 exponent bytes, two tiles in flight
// per warp.  The K
// codes become the FP16 A operand in registers (cvt e4m3x2 -> f16x2, exact);
// Q is scaled per head by a power of two into FP16 range (exact for every
// value the FP32 products can resolve); the K exponents scale S per key.  The
// V codes are converted into an FP16 tile for ldmatrix.trans, and the V
// exponents fold into P: O is accumulated against its own running maximum of
// (logit + V exponent), so P V stays in [0, 1] x code range, and is brought
// back to the softmax's reference at the end.  The ring write and candidate
// append quantise the rows (one warp per row: amax, exponent, cvt to E4M3).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
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
constexpr int kMaxSplits = 64;                                   // ring_splits + bank_splits
// FP8 storage, per warp: two stages of (K codes + exponents, V codes + exponents), then the FP16 V tile.
// A tile's 16 code rows are contiguous in the state, so each slot arrives with one bulk copy for
// the codes and one for the exponents (four requests per tile, not one per row).
constexpr int kF8Hdr = 64;                                       // a slot's 16 exponent bytes (+ pad)
constexpr int kF8Row = kHeadDim;                                 // 256 code bytes per row, unpadded
constexpr int kF8KSlot = kF8Hdr + kTile * kF8Row;                // 4,160
constexpr int kF8VSlot = kF8Hdr + kTile * kF8Row;                // 4,160
constexpr int kF8Stage = kF8KSlot + kF8VSlot;                    // 8,320
constexpr int kF8Stages = 2;
constexpr int kF8WarpRegion = kF8Stages * kF8Stage + kSlotBytes; // 25,088

// Shared-memory layout of a storage: the warps' regions, the merge's coefficients and scalars, mbarriers.
template <bool kFp8>
struct Smem {
    static constexpr int kRegion = kFp8 ? kF8WarpRegion : kWarpRegion;
    static constexpr int kPipe = kWarps * kRegion;
    static constexpr int kCoef = kPipe;                          // [(kMaxSplits + 1)][4] floats
    static constexpr int kMisc = kCoef + (kMaxSplits + 1) * 4 * 4;   // scur[4], gate[4] (+ pad)
    static constexpr int kBars = kMisc + 16 * 4;                 // [kWarps][2 or 4] mbarriers
    static constexpr int kNumBars = kWarps * (kFp8 ? 4 : 2);
    static constexpr int kBytes = kBars + kNumBars * 8;
    static_assert(kRegion >= kPartialFloats * 4, "a warp's region must hold one warp partial");
    static_assert(kPipe >= (int)admit_scratch_bytes(1, 4095), "the admit reuses the pipeline region (any A + P <= 4096)");
    static_assert((kBars & 7) == 0, "mbarriers are 8-byte aligned");
    static_assert(kBytes <= 227 * 1024, "shared memory per CTA");
};

static_assert(kWarps == 8, "merger assigns 8 dot products to 8 warps");

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

__device__ __forceinline__ uint2 ld_nc_v2(const void* p) {
    uint2 r;
    asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];\n" : "=r"(r.x), "=r"(r.y) : "l"(p));
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

// D (16x8 FP32) += A (16x16 FP16, row) . B (16x8 FP16, col)
__device__ __forceinline__ void mma_16816_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two E4M3 codes (low byte first) -> two FP16 values (low half first); exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
    uint32_t r;
    const unsigned short v = (unsigned short)(two_codes & 0xffffu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;\n" : "=r"(r) : "h"(v));
    return r;
}

// Two FP32 values -> two E4M3 codes (lo in the low byte), round to nearest even (|x| <= 448 here).
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;\n" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// 2^e as FP32 for e in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float pow2i(int e) {
    return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(0x00400000u >> (-127 - e));
}

// The scale exponent of an FP8 row: the smallest e in [-127, 127] with amax <= 448 * 2^e (0 for
// amax == 0).  With amax = 1.M * 2^(E - 127) and 448 = 1.75 * 2^8: e = E - 135, plus one when
// 1.M > 1.75 (M > 0x600000); amax below the normal range gives -127.
__device__ __forceinline__ int fp8_row_exponent(float amax) {
    if (amax == 0.f) return 0;
    const uint32_t u = __float_as_uint(amax);
    const int E = (int)(u >> 23);
    if (E == 0) return -127;
    return max(-127, min(127, E - 135 + ((u & 0x7FFFFFu) > 0x600000u ? 1 : 0)));
}

// Quantise one BF16 row of 256 values (a warp: lane L takes values 8 L .. 8 L + 7) into 256
// E4M3 codes at dst and its scale exponent at *dexp.
__device__ __forceinline__ void quantize_row_warp(const uint16_t* src, uint8_t* dst, int8_t* dexp, int lane) {
    const uint4 r = ld_nc_v4(src + lane * 8);
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
    float f[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        f[2 * k] = __uint_as_float(w[k] << 16);
        f[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
    float am = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) am = fmaxf(am, fabsf(f[k]));
    am = warp_max(am);
    const int e = fp8_row_exponent(am);
    const float sc = pow2i(-e);   // an exact power-of-two scaling
    const uint32_t lo = f32x2_to_e4m3x2(f[0] * sc, f[1] * sc) | (f32x2_to_e4m3x2(f[2] * sc, f[3] * sc) << 16);
    const uint32_t hi = f32x2_to_e4m3x2(f[4] * sc, f[5] * sc) | (f32x2_to_e4m3x2(f[6] * sc, f[7] * sc) << 16);
    *reinterpret_cast<uint2*>(dst + lane * 8) = make_uint2(lo, hi);
    if (lane == 0) *dexp = (int8_t)e;
}

// Transpose an 8x8 matrix of 16-bit values held one row pair per lane in the mma fragment layout.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
    return y;
}

__device__ __forceinline__ float dot8(const float2 (&q)[4], const uint4& k) {
    float2 d = __fmul2_rn(q[0], bf2_to_f2(k.x));
    d = __ffma2_rn(q[1], bf2_to_f2(k.y), d);
    d = __ffma2_rn(q[2], bf2_to_f2(k.z), d);
    d = __ffma2_rn(q[3], bf2_to_f2(k.w), d);
    return d.x + d.y;
}

// Programmatic dependent launch: wait until the previous kernel in the stream has completed and
// its writes are visible; let the next kernel's CTAs be scheduled.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

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

// BF16 storage: stream this warp's tiles of the CTA's row range and leave the warp's running
// softmax of heads 2 tq and 2 tq + 1 (lanes with tq >= 2 carry the unused columns) in m0, m1,
// l0, l1 (row sums already reduced over the fragment's key rows) and acc (O^T fragments).
__device__ __forceinline__ void stream_bf16(const DecodeArgs& a, uint8_t* smem, uint64_t* bars, int warp, int lane,
                                            int nrows, const uint16_t* kbase, const uint16_t* vbase,
                                            const uint16_t* qg, float& m0, float& m1, float& l0, float& l1,
                                            float (&acc)[16][4]) {
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
    if (a.early) {   // the first tile is requested: now wait for the previous kernel (see decode_kernel)
        grid_dep_wait();
        grid_dep_launch();
    }

    // ---- Q^T fragments (the B operand of S^T = K Q^T), loaded while the first tiles are in flight:
    //      lane (gq = lane / 4, tq = lane % 4) holds head gq's dims 16 c + 2 tq (+1) and 16 c + 2 tq + 8 (+9);
    //      heads 4..7 of the 8 columns are zero ----
    const int gq = lane >> 2, tq = lane & 3;
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

}

// FP8 storage: the same contract as stream_bf16 on E4M3 codes with per-row scale exponents
// (kexp / vexp: the exponents of the range's rows, 16-byte aligned).
__device__ __forceinline__ void stream_fp8(const DecodeArgs& a, uint8_t* smem, uint64_t* bars, int warp, int lane,
                                           int nrows, const uint8_t* kcodes, const uint8_t* vcodes,
                                           const int8_t* kexp, const int8_t* vexp, const uint16_t* qg, float& m0,
                                           float& m1, float& l0, float& l1, float (&acc)[16][4]) {
    uint8_t* wsm = smem + warp * kF8WarpRegion;
    uint8_t* vt = wsm + kF8Stages * kF8Stage;      // the FP16 V tile (16 rows x 528 bytes)
    uint64_t* kb = &bars[4 * warp];                // K of stage 0 / 1
    uint64_t* vb = &bars[4 * warp + 2];            // V of stage 0 / 1
    const int n_tiles = (nrows + kTile - 1) / kTile;
    const int my_n = n_tiles > warp ? (n_tiles - warp + kWarps - 1) / kWarps : 0;

    // tile i of this warp -> stage i & 1: lane 0 copies its K code rows (one contiguous range) and
    // the 16 K exponents, lane 16 its V code rows and V exponents
    auto issue = [&](int i) {
        const int st = i & 1;
        const int r0 = (warp + i * kWarps) * kTile;
        const int nv = min(kTile, nrows - r0);
        uint8_t* ks = wsm + st * kF8Stage;
        uint8_t* vs = ks + kF8KSlot;
        if (lane == 0) {
            ptx::mbar_arrive_expect_tx(&kb[st], (uint32_t)(nv * kF8Row + 16));
            bulk_g2s(ptx::smem_u32(ks + kF8Hdr), kcodes + (size_t)r0 * kF8Row, (uint32_t)(nv * kF8Row),
                     ptx::smem_u32(&kb[st]));
            bulk_g2s(ptx::smem_u32(ks), kexp + r0, 16, ptx::smem_u32(&kb[st]));
        } else if (lane == 16) {
            ptx::mbar_arrive_expect_tx(&vb[st], (uint32_t)(nv * kF8Row + 16));
            bulk_g2s(ptx::smem_u32(vs + kF8Hdr), vcodes + (size_t)r0 * kF8Row, (uint32_t)(nv * kF8Row),
                     ptx::smem_u32(&vb[st]));
            bulk_g2s(ptx::smem_u32(vs), vexp + r0, 16, ptx::smem_u32(&vb[st]));
        }
        __syncwarp();
    };
    if (my_n > 0) issue(0);
    if (my_n > 1) issue(1);
    int issued = min(my_n, 2);
    if (a.early) {   // the first tiles are requested: now wait for the previous kernel (see decode_kernel)
        grid_dep_wait();
        grid_dep_launch();
    }

    // ---- Q^T fragments in FP16.  Chunk c = 4 j + i of the contraction takes, for lane (gq, tq),
    //      dims 64 j + 16 tq + 4 i + {0, 1} as k = 2 tq, 2 tq + 1 and + {2, 3} as k = 2 tq + 8, 2 tq + 9
    //      (the K fragments below use the same order), so that each lane reads its K bytes with
    //      16-byte loads.  Head gq's values are scaled by 2^-eq, eq putting its largest magnitude
    //      in [2^14, 2^15); the logits take 2^eq back. ----
    const int gq = lane >> 2, tq = lane & 3;
    uint2 qraw[16];
    float am = 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        qraw[c] = gq < kQPerGroup ? ld_nc_v2(qg + gq * kHeadDim + 64 * (c >> 2) + 16 * tq + 4 * (c & 3))
                                  : make_uint2(0u, 0u);
        am = fmaxf(am, fmaxf(fmaxf(fabsf(__uint_as_float(qraw[c].x << 16)), fabsf(__uint_as_float(qraw[c].x & 0xffff0000u))),
                             fmaxf(fabsf(__uint_as_float(qraw[c].y << 16)), fabsf(__uint_as_float(qraw[c].y & 0xffff0000u)))));
    }
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
    const int eq = am == 0.f ? 0 : max(-126, min(126, (int)(__float_as_uint(am) >> 23) - 141));
    const float qsc = pow2i(-eq);
    uint32_t qf[16][2];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        qf[c][0] = pack_f16(__uint_as_float(qraw[c].x << 16) * qsc, __uint_as_float(qraw[c].x & 0xffff0000u) * qsc);
        qf[c][1] = pack_f16(__uint_as_float(qraw[c].y << 16) * qsc, __uint_as_float(qraw[c].y & 0xffff0000u) * qsc);
    }
    // logit scale of this lane's S^T columns (heads 2 tq, 2 tq + 1; their Q lives in lanes 8 tq, 8 tq + 4)
    const float qs0 = a.qscale * pow2i(__shfl_sync(0xffffffffu, eq, (8 * tq) & 31));
    const float qs1 = a.qscale * pow2i(__shfl_sync(0xffffffffu, eq, (8 * tq + 4) & 31));

    const int lr = lane & 7, lm = lane >> 3;
    const uint32_t v_addr = ptx::smem_u32(vt) + (uint32_t)((lr + 8 * (lm >> 1)) * kRowStride + 16 * (lm & 1));
    // O is accumulated against its own reference n (running max of logit + V exponent)
    float n0 = -CUDART_INF_F, n1 = -CUDART_INF_F;
    bool ok = true;
    int i = 0;
    for (; i < my_n; ++i) {
        const int st = i & 1;
        const uint32_t par = (i >> 1) & 1;
        const int r0 = (warp + i * kWarps) * kTile;
        const int nv = min(kTile, nrows - r0);
        uint8_t* ks = wsm + st * kF8Stage;
        uint8_t* vs = ks + kF8KSlot;
        // ---- S^T = K Q^T on the codes: 16 FP16 MMAs in four chains ----
        if (!wait_phase(&kb[st], par, a.s.status)) { ok = false; break; }
        float s[4][4];
#pragma unroll
        for (int c = 0; c < 4; ++c) s[c][0] = s[c][1] = s[c][2] = s[c][3] = 0.f;
        const uint8_t* klo = ks + kF8Hdr + gq * kF8Row + 16 * tq;
        const uint8_t* khi = klo + 8 * kF8Row;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 ra = *reinterpret_cast<const uint4*>(klo + 64 * j);
            const uint4 rb = *reinterpret_cast<const uint4*>(khi + 64 * j);
            const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w}, wb[4] = {rb.x, rb.y, rb.z, rb.w};
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) {
                uint32_t af[4];
                af[0] = e4m3x2_to_f16x2(wa[i4]);
                af[1] = e4m3x2_to_f16x2(wb[i4]);
                af[2] = e4m3x2_to_f16x2(wa[i4] >> 16);
                af[3] = e4m3x2_to_f16x2(wb[i4] >> 16);
                mma_16816_f16(s[i4], af, qf[4 * j + i4][0], qf[4 * j + i4][1]);
            }
        }
        const float ks_lo = pow2i((int)(int8_t)ks[gq]), ks_hi = pow2i((int)(int8_t)ks[gq + 8]);
        // ---- logits x (log2 domain): (key gq | gq + 8) x (head 2 tq | 2 tq + 1); the softmax sums l ----
        const bool va = gq < nv, vb2 = gq + 8 < nv;
        const float x0 = va ? (((s[0][0] + s[1][0]) + (s[2][0] + s[3][0])) * qs0) * ks_lo : -CUDART_INF_F;
        const float x1 = va ? (((s[0][1] + s[1][1]) + (s[2][1] + s[3][1])) * qs1) * ks_lo : -CUDART_INF_F;
        const float x2 = vb2 ? (((s[0][2] + s[1][2]) + (s[2][2] + s[3][2])) * qs0) * ks_hi : -CUDART_INF_F;
        const float x3 = vb2 ? (((s[0][3] + s[1][3]) + (s[2][3] + s[3][3])) * qs1) * ks_hi : -CUDART_INF_F;
        float t0 = fmaxf(x0, x2), t1 = fmaxf(x1, x3);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, o));
            t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, o));
        }
        if (t0 > m0) {
            l0 *= (m0 == -CUDART_INF_F) ? 0.f : fast_ex2(m0 - t0);
            m0 = t0;
        }
        if (t1 > m1) {
            l1 *= (m1 == -CUDART_INF_F) ? 0.f : fast_ex2(m1 - t1);
            m1 = t1;
        }
        l0 += fast_ex2(x0 - m0) + fast_ex2(x2 - m0);
        l1 += fast_ex2(x1 - m1) + fast_ex2(x3 - m1);
        // ---- V codes -> the FP16 tile (rows past the range become zero); the stage is then free ----
        if (!wait_phase(&vb[st], par, a.s.status)) { ok = false; break; }
        const float ev_lo = (float)(int8_t)vs[gq], ev_hi = (float)(int8_t)vs[gq + 8];
        {
            // pass k: the warp reads 512 contiguous code bytes (rows 2k and 2k + 1), lane L the 16
            // codes at columns 16 (L % 16) of row 2k + L / 16
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int vr = 2 * k + (lane >> 4), col = 16 * (lane & 15);
                const uint4 u = vr < nv ? *reinterpret_cast<const uint4*>(vs + kF8Hdr + vr * kF8Row + col)
                                        : make_uint4(0u, 0u, 0u, 0u);
                uint8_t* dst = vt + vr * kRowStride + 2 * col;
                *reinterpret_cast<uint4*>(dst) = make_uint4(e4m3x2_to_f16x2(u.x), e4m3x2_to_f16x2(u.x >> 16),
                                                            e4m3x2_to_f16x2(u.y), e4m3x2_to_f16x2(u.y >> 16));
                *reinterpret_cast<uint4*>(dst + 16) = make_uint4(e4m3x2_to_f16x2(u.z), e4m3x2_to_f16x2(u.z >> 16),
                                                                 e4m3x2_to_f16x2(u.w), e4m3x2_to_f16x2(u.w >> 16));
            }
        }
        __syncwarp();
        if (i + 2 < my_n) {   // both slots of this stage have been read: request tile i + 2
            issue(i + 2);
            ++issued;
        }
        // ---- P' = 2^(x + V exponent - n), O^T += V^T P'^T on the codes ----
        const float y0 = x0 + ev_lo, y1 = x1 + ev_lo, y2 = x2 + ev_hi, y3 = x3 + ev_hi;
        float u0 = fmaxf(y0, y2), u1 = fmaxf(y1, y3);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            u0 = fmaxf(u0, __shfl_xor_sync(0xffffffffu, u0, o));
            u1 = fmaxf(u1, __shfl_xor_sync(0xffffffffu, u1, o));
        }
        const bool up0 = u0 > n0, up1 = u1 > n1;
        if (__any_sync(0xffffffffu, up0 || up1)) {
            const float f0 = up0 ? (n0 == -CUDART_INF_F ? 0.f : fast_ex2(n0 - u0)) : 1.f;
            const float f1 = up1 ? (n1 == -CUDART_INF_F ? 0.f : fast_ex2(n1 - u1)) : 1.f;
            n0 = up0 ? u0 : n0;
            n1 = up1 ? u1 : n1;
#pragma unroll
            for (int mt = 0; mt < 16; ++mt) {
                acc[mt][0] *= f0;
                acc[mt][1] *= f1;
                acc[mt][2] *= f0;
                acc[mt][3] *= f1;
            }
        }
        const uint32_t pb0 = movmatrix_trans(pack_f16(fast_ex2(y0 - n0), fast_ex2(y1 - n1)));
        const uint32_t pb1 = movmatrix_trans(pack_f16(fast_ex2(y2 - n0), fast_ex2(y3 - n1)));
#pragma unroll
        for (int mt = 0; mt < 16; ++mt) {
            uint32_t af[4];
            ldsm_x4_trans(v_addr + 32 * mt, af);
            mma_16816_f16(acc[mt], af, pb0, pb1);
        }
        __syncwarp();   // the FP16 tile has been read before the next tile's conversion
    }
    if (!ok) {
        // a wait ran out: let every copy this warp requested land before its slots are reused
        for (int t = i; t < issued; ++t) {
            wait_phase(&kb[t & 1], (t >> 1) & 1, a.s.status);
            wait_phase(&vb[t & 1], (t >> 1) & 1, a.s.status);
        }
    }
    // O back to the softmax's reference: acc = O * 2^(n - m)
    const float f0 = (m0 == -CUDART_INF_F) ? 0.f : fast_ex2(n0 - m0);
    const float f1 = (m1 == -CUDART_INF_F) ? 0.f : fast_ex2(n1 - m1);
#pragma unroll
    for (int mt = 0; mt < 16; ++mt) {
        acc[mt][0] *= f0;
        acc[mt][1] *= f1;
        acc[mt][2] *= f0;
        acc[mt][3] *= f1;
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeArgs a) {
    using L = Smem<kFp8>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.s.G;
    const int bg = b * G + g;
    const int n_splits = a.ring_splits + a.bank_splits;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
    if (tid < L::kNumBars) ptx::mbar_init(&bars[tid], 1);
    ptx::fence_mbar_init();

    // The launch may begin before the previous kernel in the stream has finished.  By default
    // nothing in global memory is touched before that kernel has completed.  With `early` (the host
    // found that kernel to be a decode of this library on another layer or another state) the
    // counters are read and the first ring / bank tiles requested first, and the wait comes before
    // anything else is read or written (the inputs come after it, whoever produced them).  Either
    // way this launch lets its own dependents start only after its wait, so a launch never overlaps
    // more than the one before it.
    if (!a.early) {
        grid_dep_wait();
        grid_dep_launch();
    }

    const int32_t* cnt = a.s.counters + bg * 4;
    int pos = cnt[0], bank_fill = cnt[1], pend_fill = cnt[2];
    if (pos < 0 || bank_fill < 0 || bank_fill > a.s.A || pend_fill < 0 || pend_fill > a.s.P) {
        // a corrupted state: never index outside the buffers
        if (threadIdx.x == 0 && split == 0) atomicOr(a.s.status, (unsigned)RMA_STATUS_BAD_COUNTERS);
        pos = max(pos, 0);
        bank_fill = min(max(bank_fill, 0), a.s.A);
        pend_fill = min(max(pend_fill, 0), a.s.P);
    }

    // ---- this CTA's row range: rows [row0, row0 + nrows) of the ring or the bank ----
    const bool is_bank = split >= a.ring_splits;
    int nrows, row0;
    if (!is_bank) {
        row0 = split * a.ring_chunk;
        nrows = max(0, min(a.ring_chunk, min(pos, a.s.R) - row0));
    } else {
        row0 = (split - a.ring_splits) * a.bank_chunk;
        nrows = max(0, min(a.bank_chunk, bank_fill - row0));
    }
    const size_t row_index = (size_t)bg * (is_bank ? a.s.A : a.s.R) + row0;
    __syncthreads();   // the mbarriers are initialised

    const uint16_t* qg = a.q + ((size_t)b * G * kQPerGroup + (size_t)g * kQPerGroup) * kHeadDim;
    float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.f, l1 = 0.f;
    float acc[16][4];
#pragma unroll
    for (int mt = 0; mt < 16; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    if constexpr (kFp8) {
        const uint8_t* kc8 = reinterpret_cast<const uint8_t*>(is_bank ? a.s.bank_k : a.s.ring_k) + row_index * kHeadDim;
        const uint8_t* vc8 = reinterpret_cast<const uint8_t*>(is_bank ? a.s.bank_v : a.s.ring_v) + row_index * kHeadDim;
        const size_t erow = (size_t)bg * (is_bank ? a.s.AE : a.s.RE) + row0;
        stream_fp8(a, smem, bars, warp, lane, nrows, kc8, vc8, (is_bank ? a.s.bank_ke : a.s.ring_ke) + erow,
                   (is_bank ? a.s.bank_ve : a.s.ring_ve) + erow, qg, m0, m1, l0, l1, acc);
    } else {
        stream_bf16(a, smem, bars, warp, lane, nrows, (is_bank ? a.s.bank_k : a.s.ring_k) + row_index * kHeadDim,
                    (is_bank ? a.s.bank_v : a.s.ring_v) + row_index * kHeadDim, qg, m0, m1, l0, l1, acc);
    }
    const int gq = lane >> 2, tq = lane & 3;
    uint8_t* wsm = smem + warp * L::kRegion;

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
            mw[w] = reinterpret_cast<const float*>(smem + w * L::kRegion)[h];
            M = fmaxf(M, mw[w]);
        }
        const float Mu = (M == -CUDART_INF_F) ? 0.f : M;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float* wp = reinterpret_cast<const float*>(smem + w * L::kRegion);
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
    float* coef = reinterpret_cast<float*>(smem + L::kCoef);   // [(n_splits+1)][4]
    float* misc = reinterpret_cast<float*>(smem + L::kMisc);   // scur[4], gate[4]
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
    if constexpr (kFp8) {
        // one warp per row: quantise into codes and a scale exponent
        uint8_t* rk = reinterpret_cast<uint8_t*>(a.s.ring_k) + ((size_t)bg * a.s.R + slot) * kHeadDim;
        uint8_t* rv = reinterpret_cast<uint8_t*>(a.s.ring_v) + ((size_t)bg * a.s.R + slot) * kHeadDim;
        uint8_t* pk = reinterpret_cast<uint8_t*>(a.s.pend_k) + ((size_t)bg * a.s.P + pend_fill) * kHeadDim;
        uint8_t* pv = reinterpret_cast<uint8_t*>(a.s.pend_v) + ((size_t)bg * a.s.P + pend_fill) * kHeadDim;
        if (warp == 0) {
            quantize_row_warp(kc, rk, a.s.ring_ke + (size_t)bg * a.s.RE + slot, lane);
        } else if (warp == 1) {
            quantize_row_warp(vc, rv, a.s.ring_ve + (size_t)bg * a.s.RE + slot, lane);
        } else if (warp == 2) {
            if (room) quantize_row_warp(a.cand_k + (size_t)bg * kHeadDim, pk, a.s.pend_ke + (size_t)bg * a.s.PE + pend_fill, lane);
        } else if (warp == 3) {
            if (room) quantize_row_warp(a.cand_v + (size_t)bg * kHeadDim, pv, a.s.pend_ve + (size_t)bg * a.s.PE + pend_fill, lane);
        }
    } else {
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
        }
    }
    if (tid == 128) {
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

// Every row of every array of one layer, one warp per row: BF16 -> E4M3 codes + exponent.
__global__ void __launch_bounds__(256) quantize_kernel(const __grid_constant__ LayerView d,
                                                       const __grid_constant__ LayerView s) {
    const int lane = threadIdx.x & 31;
    const long long nbg = (long long)s.B * s.G;
    const long long n_ring = nbg * s.R, n_bank = nbg * s.A, n_pend = nbg * s.P;
    const long long total = 2 * (n_ring + n_bank + n_pend);
    for (long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); w < total; w += (long long)gridDim.x * 8) {
        long long r = w;
        const uint16_t* src;
        uint8_t* dst;
        int8_t* dexp;
        if (r < 2 * n_ring) {
            const bool v = r >= n_ring;
            const long long idx = v ? r - n_ring : r;
            src = (v ? s.ring_v : s.ring_k) + idx * kHeadDim;
            dst = reinterpret_cast<uint8_t*>(v ? d.ring_v : d.ring_k) + idx * kHeadDim;
            dexp = (v ? d.ring_ve : d.ring_ke) + (idx / s.R) * d.RE + idx % s.R;
        } else if ((r -= 2 * n_ring) < 2 * n_bank) {
            const bool v = r >= n_bank;
            const long long idx = v ? r - n_bank : r;
            src = (v ? s.bank_v : s.bank_k) + idx * kHeadDim;
            dst = reinterpret_cast<uint8_t*>(v ? d.bank_v : d.bank_k) + idx * kHeadDim;
            dexp = (v ? d.bank_ve : d.bank_ke) + (idx / s.A) * d.AE + idx % s.A;
        } else {
            r -= 2 * n_bank;
            const bool v = r >= n_pend;
            const long long idx = v ? r - n_pend : r;
            src = (v ? s.pend_v : s.pend_k) + idx * kHeadDim;
            dst = reinterpret_cast<uint8_t*>(v ? d.pend_v : d.pend_k) + idx * kHeadDim;
            dexp = (v ? d.pend_ve : d.pend_ke) + (idx / s.P) * d.PE + idx % s.P;
        }
        quantize_row_warp(src, dst, dexp, lane);
    }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    if (a.ring_splits + a.bank_splits > kMaxSplits) return cudaErrorInvalidValue;
    // launched with programmatic stream serialisation: the kernel's griddepcontrol.wait keeps it
    // correct after any kernel, and after a decode it overlaps that kernel's tail
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.ring_splits + a.bank_splits, a.s.G, a.s.B);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (a.s.fp8) {
        static SmemLimit limit(reinterpret_cast<const void*>(decode_kernel<true>));
        const cudaError_t e = limit.ensure(Smem<true>::kBytes);
        if (e != cudaSuccess) return e;
        cfg.dynamicSmemBytes = Smem<true>::kBytes;
        return cudaLaunchKernelEx(&cfg, decode_kernel<true>, a);
    }
    static SmemLimit limit(reinterpret_cast<const void*>(decode_kernel<false>));
    const cudaError_t e = limit.ensure(Smem<false>::kBytes);
    if (e != cudaSuccess) return e;
    cfg.dynamicSmemBytes = Smem<false>::kBytes;
    return cudaLaunchKernelEx(&cfg, decode_kernel<false>, a);
}

cudaError_t launch_quantize_layer(const LayerView& dst, const LayerView& src, cudaStream_t stream) {
    const long long rows = 2LL * src.B * src.G * ((long long)src.R + src.A + src.P);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long blocks = std::min<long long>((rows + 7) / 8, (long long)sms * 8);
    quantize_kernel<<<(unsigned)blocks, 256, 0, stream>>>(dst, src);
    cudaError_t e = cudaGetLastError();
    const size_t nbg = (size_t)src.B * src.G;
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(dst.bank_score, src.bank_score, nbg * src.A * 4, cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(dst.pend_score, src.pend_score, nbg * src.P * 4, cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(dst.counters, src.counters, nbg * 16, cudaMemcpyDeviceToDevice, stream);
    return e;
}

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
