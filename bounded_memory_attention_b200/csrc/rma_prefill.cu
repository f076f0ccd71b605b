// rma_prefill_block: a block of n tokens per sequence at one RMA layer.
//
// ("EdgeRock" model card, FAQ "How do Rock Memory Anchors preserve distant
// information?": reads use the committed bank and updates take effect at the
// next block; ai-primer story "EdgeRock-4B fixes its attention KV cache at
// 72 MiB", operations 1-3.)  With block start s = pos, query i (position
// s + i) attends causally to positions [s + i - R, s + i] (ring slots for
// those below s, the block's own K/V for the rest) and to the committed bank
// as it was before the block; out = local + tanh(q . w_g + b_g) anchor.
// Then the block's K/V go into the ring, its candidates into pending, and
// the admit runs forced.
//
// Three launches, in stream order:
//  1. prefill_attn_kernel (tensor cores).  One CTA per (sequence, group,
//     tile of 32 tokens, phase): phase 0 = local window, phase 1 = bank.  The
//     tile's 128 rows are 32 tokens x the group's 4 query heads, which share
//     every key, so one K/V chunk feeds all 4 heads.  TMA brings the Q tile
//     and 64-key K/V chunks into 128B-swizzled shared memory; one thread
//     issues tcgen05.mma for S = Q K^T into tensor memory; a 128-thread
//     softmax warpgroup (one thread per row) reads S, masks it by position,
//     keeps the online max/sum in FP32 and writes P (BF16) back into the same
//     tensor-memory columns; tcgen05.mma then accumulates O += P V with P
//     read from tensor memory and V as an MN-major shared-memory operand.
//     Each CTA writes its normalised FP32 rows to the workspace.
//  2. prefill_finish_kernel: out = local + gate * anchor (BF16), then the
//     block's K/V into ring slots (s + i) mod R and its candidates into
//     pending (if they fit).  Runs after every read of launch 1.
//  3. the admit kernel, forced, which also advances pos and pend_fill.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <mutex>

#include "rma_internal.cuh"
#include "sm100_ptx.cuh"

namespace rma {
namespace {

constexpr int kTileTok = 32;                          // tokens per tile
constexpr int kRows = kTileTok * kQPerGroup;          // 128 MMA rows
constexpr int kChunk = 64;                            // keys per chunk
constexpr int kSlabQ = kRows * 128;                   // 128 rows x 64 dims (bf16) = 16 KiB
constexpr int kSlabKV = kChunk * 128;                 // 64 keys x 64 dims = 8 KiB
constexpr int kQBytes = 4 * kSlabQ;                   // 64 KiB
constexpr int kKVBytes = 4 * kSlabKV;                 // 32 KiB per K or V chunk
constexpr int kSmemQ = 0;
constexpr int kSmemK = kQBytes;                       // 2 stages
constexpr int kSmemV = kSmemK + 2 * kKVBytes;         // 2 stages
constexpr int kSmemBar = kSmemV + 2 * kKVBytes;       // 192 KiB
constexpr int kSmemBytes = kSmemBar + 256 + 1024;     // barriers + 1 KiB for alignment
constexpr int kThreads = 192;                         // warps 0-3 softmax, 4 TMA, 5 MMA
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS0 = 256, kColS1 = 320;

struct Tmaps {
    CUtensorMap q, k, v, ring_k, ring_v, bank_k, bank_v;
};

struct AttnParams {
    const int32_t* counters;   // [B][G][4] of this layer
    float* ws;                 // [B][G][ntiles][2][128][256]
    uint32_t* status;
    int B, G, R, A, n, ntiles;
    float qscale;
};

enum Bar { kQFull = 0, kKFull = 1, kVFull = 3, kKVEmpty = 5, kSFull = 7, kPFull = 9, kODone = 11, kNumBars = 12 };

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ float fast_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__global__ void __launch_bounds__(kThreads, 1)
    prefill_attn_kernel(const __grid_constant__ Tmaps tm, const __grid_constant__ AttnParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int T = blockIdx.x >> 1, phase = blockIdx.x & 1;
    const int g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bg = b * p.G + g;

    int s = p.counters[bg * 4 + 0];
    int bank_fill = p.counters[bg * 4 + 1];
    s = max(s, 0);
    bank_fill = min(max(bank_fill, 0), p.A);
    const int fill = min(s, p.R);

    int n_ring = 0, n_blk = 0, n_bank = 0;
    if (phase == 0) {
        n_ring = (fill + kChunk - 1) / kChunk;
        n_blk = (kTileTok * T + kTileTok - 1) / kChunk + 1;
    } else {
        n_bank = (bank_fill + kChunk - 1) / kChunk;
    }
    const int nchunks = n_ring + n_blk + n_bank;
    float* out_rows = p.ws + (((size_t)bg * p.ntiles + T) * 2 + phase) * (size_t)kRows * kHeadDim;

    if (nchunks == 0) {   // empty bank: the anchor read is 0
        for (int e = tid; e < kRows * kHeadDim / 4; e += kThreads)
            reinterpret_cast<float4*>(out_rows)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        return;
    }

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBar);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kNumBars + 1);

    if (tid == 0) {
        ptx::mbar_init(&bars[kQFull], 1);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&bars[kKFull + i], 1);
            ptx::mbar_init(&bars[kVFull + i], 1);
            ptx::mbar_init(&bars[kKVEmpty + i], 1);
            ptx::mbar_init(&bars[kSFull + i], 1);
            ptx::mbar_init(&bars[kPFull + i], 4);
        }
        ptx::mbar_init(&bars[kODone], 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 5) {
        ptx::tmem_alloc(tmem_holder, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 4) {
        // ---------------- TMA producer (the whole warp loops; lane 0 issues) ----------------
        if (lane == 0) {
            ptx::prefetch_tmap(&tm.q);
            ptx::mbar_arrive_expect_tx(&bars[kQFull], kQBytes);
            for (int slab = 0; slab < 4; ++slab)
                ptx::tma_load_3d(smem + kSmemQ + slab * kSlabQ, &tm.q, &bars[kQFull], 64 * slab, kQPerGroup * g,
                                 b * p.n + kTileTok * T);
        }
        __syncwarp();
        const int zreg = b * p.G + g;
        for (int j = 0; j < nchunks; ++j) {
            const int st = j & 1;
            if (j >= 2 && !ptx::mbar_wait_warp(&bars[kKVEmpty + st], ((j >> 1) - 1) & 1, abort_flag, p.status))
                break;
            if (lane == 0) {
                const CUtensorMap* mk;
                const CUtensorMap* mv;
                int y, z;
                if (j < n_ring) {
                    mk = &tm.ring_k; mv = &tm.ring_v; y = kChunk * j; z = zreg;
                } else if (j < n_ring + n_blk) {
                    mk = &tm.k; mv = &tm.v; y = g; z = b * p.n + kChunk * (j - n_ring);
                } else {
                    mk = &tm.bank_k; mv = &tm.bank_v; y = kChunk * (j - n_ring - n_blk); z = zreg;
                }
                ptx::mbar_arrive_expect_tx(&bars[kKFull + st], kKVBytes);
                for (int slab = 0; slab < 4; ++slab)
                    ptx::tma_load_3d(smem + kSmemK + st * kKVBytes + slab * kSlabKV, mk, &bars[kKFull + st],
                                     64 * slab, y, z);
                ptx::mbar_arrive_expect_tx(&bars[kVFull + st], kKVBytes);
                for (int slab = 0; slab < 4; ++slab)
                    ptx::tma_load_3d(smem + kSmemV + st * kKVBytes + slab * kSlabKV, mv, &bars[kVFull + st],
                                     64 * slab, y, z);
            }
            __syncwarp();
        }
    } else if (warp == 5) {
        // ---------------- MMA issuer (lane 0) ----------------
        constexpr uint32_t idesc_qk = ptx::idesc_bf16_f32(kRows, kChunk, false, false);
        constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(kRows, kHeadDim, false, true);
        const uint32_t q_base = ptx::smem_u32(smem + kSmemQ);
        bool ok = ptx::mbar_wait_warp(&bars[kQFull], 0, abort_flag, p.status);
        for (int j = 0; ok && j <= nchunks; ++j) {
            if (j < nchunks) {
                const int st = j & 1;
                if (!ptx::mbar_wait_warp(&bars[kKFull + st], (j >> 1) & 1, abort_flag, p.status)) break;
                ptx::tc_fence_after();
                if (lane == 0) {
                    const uint32_t k_base = ptx::smem_u32(smem + kSmemK + st * kKVBytes);
                    const uint32_t d = tmem + (st ? kColS1 : kColS0);
                    for (int ks = 0; ks < kHeadDim / 16; ++ks) {
                        const uint32_t within = (ks & 3) * 32;   // 16 dims = 32 bytes inside the swizzle atom
                        const uint64_t ad = ptx::smem_desc(q_base + (ks >> 2) * kSlabQ + within, 16, 1024,
                                                           ptx::kSwizzle128B);
                        const uint64_t bd = ptx::smem_desc(k_base + (ks >> 2) * kSlabKV + within, 16, 1024,
                                                           ptx::kSwizzle128B);
                        ptx::mma_ss(d, ad, bd, idesc_qk, ks > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(&bars[kSFull + st]);
                }
                __syncwarp();
            }
            if (j >= 1) {
                const int jj = j - 1, st = jj & 1;
                if (!ptx::mbar_wait_warp(&bars[kPFull + st], (jj >> 1) & 1, abort_flag, p.status)) break;
                if (!ptx::mbar_wait_warp(&bars[kVFull + st], (jj >> 1) & 1, abort_flag, p.status)) break;
                // rows of this chunk past the valid keys may hold stale bytes: zero them so
                // that P = 0 times V stays 0
                int nvalid;
                if (jj < n_ring) nvalid = fill - kChunk * jj;
                else if (jj < n_ring + n_blk) nvalid = p.n - kChunk * (jj - n_ring);
                else nvalid = bank_fill - kChunk * (jj - n_ring - n_blk);
                if (nvalid < kChunk) {
                    uint8_t* vst = smem + kSmemV + st * kKVBytes;
                    const int nz = (kChunk - nvalid) * 8;   // 16-byte pieces per slab
                    for (int e = lane; e < 4 * nz; e += 32) {
                        const int slab = e / nz, piece = e % nz;
                        reinterpret_cast<uint4*>(vst + slab * kSlabKV + nvalid * 128)[piece] = make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                }
                __syncwarp();
                ptx::tc_fence_after();
                if (lane == 0) {
                    const uint32_t v_base = ptx::smem_u32(smem + kSmemV + st * kKVBytes);
                    const uint32_t a_col = tmem + (st ? kColS1 : kColS0);
                    for (int ks = 0; ks < kChunk / 16; ++ks) {
                        const uint64_t bd = ptx::smem_desc(v_base + ks * 16 * 128, kSlabKV, 1024, ptx::kSwizzle128B);
                        ptx::mma_ts(tmem + kColO, a_col + 8 * ks, bd, idesc_pv, (jj > 0 || ks > 0) ? 1u : 0u);
                    }
                    ptx::mma_commit(&bars[kKVEmpty + st]);
                    ptx::mma_commit(&bars[kODone]);
                }
                __syncwarp();
            }
        }
        // the producer never waits on the last two kv_empty phases: consume them here so no
        // commit is still pending when the CTA exits
        for (int jj = max(0, nchunks - 2); ok && jj < nchunks; ++jj)
            if (!ptx::mbar_wait_warp(&bars[kKVEmpty + (jj & 1)], (jj >> 1) & 1, abort_flag, p.status)) break;
    } else {
        // ---------------- softmax warpgroup: thread = row ----------------
        const int row = 32 * warp + lane;
        const int tok = kTileTok * T + (row >> 2);     // token index within the block
        const int pq = s + tok;                        // query position
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * warp) << 16);
        const int w = (s - 1) % p.R;                   // slot of position s - 1 (when s >= 1)
        const int base_pos = s - 1 - w;
        float m_used = -CUDART_INF_F, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nchunks; ++j) {
            const int st = j & 1;
            if (!ptx::mbar_wait_warp(&bars[kSFull + st], (j >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            ptx::tc_fence_after();
            uint32_t sr0[32], sr1[32];
            ptx::tmem_ld32(lane_addr + (st ? kColS1 : kColS0), sr0);
            ptx::tmem_ld32(lane_addr + (st ? kColS1 : kColS0) + 32, sr1);
            ptx::tmem_wait_ld();
            float x[kChunk];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                x[i] = __uint_as_float(sr0[i]);
                x[32 + i] = __uint_as_float(sr1[i]);
            }
            float mloc = -CUDART_INF_F;
            if (j < n_ring) {
                const int slot0 = kChunk * j;
#pragma unroll
                for (int i = 0; i < kChunk; ++i) {
                    const int slot = slot0 + i;
                    const int pk = base_pos + slot - (slot > w ? p.R : 0);
                    const bool vis = (slot < fill) && (pk >= pq - p.R);
                    x[i] = vis ? x[i] * p.qscale : -CUDART_INF_F;
                    mloc = fmaxf(mloc, x[i]);
                }
            } else if (j < n_ring + n_blk) {
                const int t0 = kChunk * (j - n_ring);
#pragma unroll
                for (int i = 0; i < kChunk; ++i) {
                    const bool vis = (t0 + i < p.n) && (t0 + i <= tok);
                    x[i] = vis ? x[i] * p.qscale : -CUDART_INF_F;
                    mloc = fmaxf(mloc, x[i]);
                }
            } else {
                const int a0 = kChunk * (j - n_ring - n_blk);
#pragma unroll
                for (int i = 0; i < kChunk; ++i) {
                    const bool vis = (a0 + i < bank_fill);
                    x[i] = vis ? x[i] * p.qscale : -CUDART_INF_F;
                    mloc = fmaxf(mloc, x[i]);
                }
            }
            // lazy reference point: move it only when the chunk max exceeds it by more than 2^8
            float m_new = m_used;
            bool resc = false;
            if (mloc > m_used + 8.f) {
                resc = (m_used != -CUDART_INF_F);
                m_new = mloc;
            }
            const float fac = resc ? fast_ex2(m_used - m_new) : 1.f;
            const float mref = (m_new == -CUDART_INF_F) ? 0.f : m_new;
            m_used = m_new;
            float sum = 0.f;
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float a = fast_ex2(x[2 * i] - mref), c = fast_ex2(x[2 * i + 1] - mref);
                sum += a + c;
                pk[i] = pack_bf16(a, c);
            }
            l = l * fac + sum;
            if (j >= 1 && !ptx::mbar_wait_warp(&bars[kODone], (j - 1) & 1, abort_flag, p.status)) { ok = false; break; }
            ptx::tc_fence_after();
            if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
                for (int c = 0; c < kHeadDim / 32; ++c) {
                    uint32_t o[32];
                    ptx::tmem_ld32(lane_addr + kColO + 32 * c, o);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * fac);
                    ptx::tmem_st32(lane_addr + kColO + 32 * c, o);
                }
            }
            ptx::tmem_st32(lane_addr + (st ? kColS1 : kColS0), pk);
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars[kPFull + st]);
        }
        if (ok && ptx::mbar_wait_warp(&bars[kODone], (nchunks - 1) & 1, abort_flag, p.status)) {
            ptx::tc_fence_after();
            const float inv = (l > 0.f) ? 1.f / l : 0.f;
            float4* dst = reinterpret_cast<float4*>(out_rows + (size_t)row * kHeadDim);
#pragma unroll 1
            for (int c = 0; c < kHeadDim / 32; ++c) {
                uint32_t o[32];
                ptx::tmem_ld32(lane_addr + kColO + 32 * c, o);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[c * 8 + i] = make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                                 __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// out = local + tanh(q . w_g + b_g) * anchor for the tile's 128 rows; then the
// tile's 32 tokens go into the ring and (if they fit) the pending buffer.
__global__ void __launch_bounds__(128) prefill_finish_kernel(const __grid_constant__ PrefillArgs a, int ntiles) {
    const int T = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.s.G, HQ = G * kQPerGroup, n = a.n_tok;
    const int bg = b * G + g;
    const float* loc = a.ws + (((size_t)bg * ntiles + T) * 2 + 0) * (size_t)kRows * kHeadDim;
    const float* anc = loc + (size_t)kRows * kHeadDim;
    for (int r = warp; r < kRows; r += 4) {
        const int i = kTileTok * T + (r >> 2), h = r & 3, head = g * kQPerGroup + h;
        const size_t qoff = ((size_t)(b * n + i) * HQ + head) * kHeadDim + lane * 8;
        const uint4 qr = *reinterpret_cast<const uint4*>(a.q + qoff);
        const float4 w0 = *reinterpret_cast<const float4*>(a.w_g + (size_t)head * kHeadDim + lane * 8);
        const float4 w1 = *reinterpret_cast<const float4*>(a.w_g + (size_t)head * kHeadDim + lane * 8 + 4);
        const uint32_t qw[4] = {qr.x, qr.y, qr.z, qr.w};
        const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            d += __uint_as_float(qw[e] << 16) * wv[2 * e] + __uint_as_float(qw[e] & 0xffff0000u) * wv[2 * e + 1];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        const float gate = tanhf(d + a.b_g[head]);
        const float4 l0 = *reinterpret_cast<const float4*>(loc + (size_t)r * kHeadDim + lane * 8);
        const float4 l1 = *reinterpret_cast<const float4*>(loc + (size_t)r * kHeadDim + lane * 8 + 4);
        const float4 c0 = *reinterpret_cast<const float4*>(anc + (size_t)r * kHeadDim + lane * 8);
        const float4 c1 = *reinterpret_cast<const float4*>(anc + (size_t)r * kHeadDim + lane * 8 + 4);
        uint4 o;
        o.x = pack_bf16(l0.x + gate * c0.x, l0.y + gate * c0.y);
        o.y = pack_bf16(l0.z + gate * c0.z, l0.w + gate * c0.w);
        o.z = pack_bf16(l1.x + gate * c1.x, l1.y + gate * c1.y);
        o.w = pack_bf16(l1.z + gate * c1.z, l1.w + gate * c1.w);
        *reinterpret_cast<uint4*>(a.out + qoff) = o;
    }
    // state writes for this tile's tokens (launch 1 has finished every read)
    const int32_t* cnt = a.s.counters + bg * 4;
    const int s = max(cnt[0], 0);
    const int pf = min(max(cnt[2], 0), a.s.P);
    const bool fits = pf + n <= a.s.P;
    for (int t = warp; t < kTileTok; t += 4) {
        const int i = kTileTok * T + t;
        const size_t src = ((size_t)(b * n + i) * G + g) * kHeadDim;
        const int slot = (s + i) % a.s.R;
        const size_t dst = ((size_t)bg * a.s.R + slot) * kHeadDim;
        reinterpret_cast<uint4*>(a.s.ring_k + dst)[lane] = reinterpret_cast<const uint4*>(a.k + src)[lane];
        reinterpret_cast<uint4*>(a.s.ring_v + dst)[lane] = reinterpret_cast<const uint4*>(a.v + src)[lane];
        if (fits) {
            const size_t pd = ((size_t)bg * a.s.P + pf + i) * kHeadDim;
            reinterpret_cast<uint4*>(a.s.pend_k + pd)[lane] = reinterpret_cast<const uint4*>(a.cand_k + src)[lane];
            reinterpret_cast<uint4*>(a.s.pend_v + pd)[lane] = reinterpret_cast<const uint4*>(a.cand_v + src)[lane];
            if (lane == 0)
                a.s.pend_score[(size_t)bg * a.s.P + pf + i] = a.cand_score[(size_t)(b * n + i) * G + g];
        }
    }
}

// ---- host side: tensor maps through the driver entry point ----

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D BF16 tensor [d2][d1][256] with the given strides (bytes) for dims 1 and 2,
// box (64, box1, box2), 128-byte swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap* m, const void* base, uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2,
              uint32_t box1, uint32_t box2) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)d1, (cuuint64_t)d2};
    const cuuint64_t strides[2] = {(cuuint64_t)stride1, (cuuint64_t)stride2};
    const cuuint32_t box[3] = {64, box1, box2};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t prefill_workspace_bytes(const rma_config& cfg, int n_tok) {
    const size_t ntiles = (size_t)(n_tok + kTileTok - 1) / kTileTok;
    return (size_t)cfg.batch * cfg.n_groups * ntiles * 2 * kRows * kHeadDim * sizeof(float);
}

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream) {
    const LayerView& s = a.s;
    const int B = s.B, G = s.G, n = a.n_tok, HQ = G * kQPerGroup;
    if (n % kTileTok != 0 || n > s.R) return cudaErrorNotSupported;
    const int ntiles = n / kTileTok;
    Tmaps tm;
    const uint64_t row = (uint64_t)kHeadDim * 2;
    bool ok = make_map(&tm.q, a.q, HQ, (uint64_t)B * n, row, row * HQ, kQPerGroup, kTileTok) &&
              make_map(&tm.k, a.k, G, (uint64_t)B * n, row, row * G, 1, kChunk) &&
              make_map(&tm.v, a.v, G, (uint64_t)B * n, row, row * G, 1, kChunk) &&
              make_map(&tm.ring_k, s.ring_k, s.R, (uint64_t)B * G, row, row * s.R, kChunk, 1) &&
              make_map(&tm.ring_v, s.ring_v, s.R, (uint64_t)B * G, row, row * s.R, kChunk, 1) &&
              make_map(&tm.bank_k, s.bank_k, s.A, (uint64_t)B * G, row, row * s.A, kChunk, 1) &&
              make_map(&tm.bank_v, s.bank_v, s.A, (uint64_t)B * G, row, row * s.A, kChunk, 1);
    if (!ok) return cudaErrorInvalidValue;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemBytes);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    AttnParams p;
    p.counters = s.counters;
    p.ws = a.ws;
    p.status = s.status;
    p.B = B;
    p.G = G;
    p.R = s.R;
    p.A = s.A;
    p.n = n;
    p.ntiles = ntiles;
    p.qscale = a.qscale;
    prefill_attn_kernel<<<dim3(2 * ntiles, G, B), kThreads, kSmemBytes, stream>>>(tm, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    prefill_finish_kernel<<<dim3(ntiles, G, B), 128, 0, stream>>>(a, ntiles);
    return cudaGetLastError();
}

}  // namespace rma
