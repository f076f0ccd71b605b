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
// One launch.  One CTA per (sequence, group, tile of 32 tokens, phase):
// phase 0 reads the local window, phase 1 the bank.  The tile's 128 rows are
// 32 tokens x the group's 4 query heads, which share every key, so one K/V
// chunk feeds all 4 heads.
//   * tensor memory (512 columns): O [0,256) FP32, S/P double buffer
//     [256,320) and [320,384), Q [384,512) as packed BF16 (the A operand of
//     Q K^T comes from tensor memory, which leaves shared memory to a
//     three-stage ring of 64-key K/V chunks);
//   * warp 8 (TMA) loads 128B-swizzled K and V chunks: ring slots, then the
//     block's own keys, or bank slots;
//   * warp 9 issues tcgen05.mma: S = Q K^T (M 128, N 64, K 256) and
//     O += P V (M 128, N 256, K 64; P from tensor memory, V an MN-major
//     shared-memory operand);
//   * warps 0-7 are the softmax: two warpgroups, each thread one row and one
//     half of the chunk's keys (and of Q and O's columns).  They load Q into
//     tensor memory, then per chunk read their half of S, mask it by
//     position (whole halves that are all visible or all hidden skip the
//     per-key test), exchange the row max through shared memory, keep the
//     online max / sum in FP32 (moving the reference max only when it grows by
//     more than 2^8), write BF16 P over S, and finally normalise O.
// Tail, through a per-(sequence, group) ticket word: each CTA writes its
// normalised rows to the workspace; the second CTA of a tile's pair adds
// them as local + gate * anchor and writes the BF16 output; the last CTA of
// the (sequence, group) writes the block into the ring and pending buffer
// (every read of the block is finished by then) and runs the forced admit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <mutex>

#include "rma_admit_impl.cuh"
#include "rma_internal.cuh"
#include "sm100_ptx.cuh"

namespace rma {
namespace {

constexpr int kTileTok = 32;                          // tokens per tile
constexpr int kRows = kTileTok * kQPerGroup;          // 128 MMA rows
constexpr int kChunk = 64;                            // keys per chunk
constexpr int kMaxTiles = 8;                          // ticket word: 2 bits per tile below bit 16
constexpr int kSlabKV = kChunk * 128;                 // 64 keys x 64 dims (bf16) = 8 KiB
constexpr int kKVBytes = 4 * kSlabKV;                 // 32 KiB per K or V chunk
constexpr int kStages = 3;
constexpr int kSmemK = 0;
constexpr int kSmemV = kStages * kKVBytes;
constexpr int kSmemBar = 2 * kStages * kKVBytes;      // 192 KiB
constexpr int kSmemXch = kSmemBar + 256;             // softmax exchange: max [2][2][128], sums/gate [2][128]
constexpr int kSmemBytes = kSmemXch + 4096 + 1024;    // + 1 KiB for alignment
constexpr int kSoftmaxThreads = 256;                  // warps 0-7
constexpr int kWarpTma = 8, kWarpMma = 9;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS0 = 256, kColS1 = 320, kColQ = 384;

static_assert(kSmemBar >= (int)admit_scratch_bytes(1, 4095), "the tail's admit reuses the K/V stages");

struct Tmaps {
    CUtensorMap k, v, ring_k, ring_v, bank_k, bank_v;
};

enum Bar {
    kQReady = 0,
    kKFull = 1,                 // [3]
    kVFull = 4,                 // [3]
    kKVEmpty = 7,               // [3]
    kSFull = 10,                // [2]
    kPFull = 12,                // [2]
    kODone = 14,
    kNumBars = 15
};

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
    prefill_kernel(const __grid_constant__ Tmaps tm, const __grid_constant__ PrefillArgs a, int ntiles) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const LayerView& S = a.s;
    const int T = blockIdx.x >> 1, phase = blockIdx.x & 1;
    const int g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = S.G, HQ = G * kQPerGroup, n = a.n_tok;
    const int bg = b * G + g;

    const int32_t* cnt = S.counters + bg * 4;
    const int s = max(cnt[0], 0);
    const int bank_fill = min(max(cnt[1], 0), S.A);
    const int pend_fill = min(max(cnt[2], 0), S.P);
    const int fill = min(s, S.R);

    int n_ring = 0, n_blk = 0, n_bank = 0;
    if (phase == 0) {
        n_ring = (fill + kChunk - 1) / kChunk;
        n_blk = (kTileTok * T + kTileTok - 1) / kChunk + 1;
    } else {
        n_bank = (bank_fill + kChunk - 1) / kChunk;
    }
    const int nchunks = n_ring + n_blk + n_bank;
    const bool has_work = nchunks > 0;
    float* own_rows = a.ws + (((size_t)bg * ntiles + T) * 2 + phase) * (size_t)kRows * kHeadDim;
    const float* partner_rows = a.ws + (((size_t)bg * ntiles + T) * 2 + (phase ^ 1)) * (size_t)kRows * kHeadDim;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBar);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kNumBars + 1);
    int* tail_flags = reinterpret_cast<int*>(bars + kNumBars + 2);   // [0] partner done, [1] last of all

    // softmax-thread identity (warps 0-7): row, and which half of keys / columns
    const int row = 32 * (warp & 3) + lane;
    const int wg = (warp >> 2) & 1;
    const int tok = kTileTok * T + (row >> 2);    // token within the block
    const int head = g * kQPerGroup + (row & 3);
    float* xch = reinterpret_cast<float*>(smem + kSmemXch);
    float l = 0.f;
    uint32_t tmem = 0;

    if (has_work) {
        if (tid == 0) {
            ptx::mbar_init(&bars[kQReady], 8);
            for (int i = 0; i < kStages; ++i) {
                ptx::mbar_init(&bars[kKFull + i], 1);
                ptx::mbar_init(&bars[kVFull + i], 1);
                ptx::mbar_init(&bars[kKVEmpty + i], 1);
            }
            for (int i = 0; i < 2; ++i) {
                ptx::mbar_init(&bars[kSFull + i], 1);
                ptx::mbar_init(&bars[kPFull + i], 8);
            }
            ptx::mbar_init(&bars[kODone], 1);
            *abort_flag = 0;
            ptx::fence_mbar_init();
        }
        if (warp == kWarpMma) {
            ptx::tmem_alloc(tmem_holder, kTmemCols);
            ptx::tmem_relinquish();
        }
        ptx::tc_fence_before();
        __syncthreads();
        ptx::tc_fence_after();
        tmem = *tmem_holder;

        if (warp == kWarpTma) {
            // ---------------- TMA producer (whole warp loops; lane 0 issues) ----------------
            const int zreg = b * G + g;
            for (int j = 0; j < nchunks; ++j) {
                const int st = j % kStages;
                if (j >= kStages &&
                    !ptx::mbar_wait_warp(&bars[kKVEmpty + st], ((j / kStages) - 1) & 1, abort_flag, S.status))
                    break;
                if (lane == 0) {
                    const CUtensorMap* mk;
                    const CUtensorMap* mv;
                    int y, z;
                    if (j < n_ring) {
                        mk = &tm.ring_k; mv = &tm.ring_v; y = kChunk * j; z = zreg;
                    } else if (j < n_ring + n_blk) {
                        mk = &tm.k; mv = &tm.v; y = g; z = b * n + kChunk * (j - n_ring);
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
        } else if (warp == kWarpMma) {
            // ---------------- MMA issuer (whole warp loops; lane 0 issues) ----------------
            // tcgen05.mma instructions from one thread execute in issue order, so Q K^T of
            // chunk j + 2 (issued after P V of chunk j) cannot overwrite P_j before it is read.
            constexpr uint32_t idesc_qk = ptx::idesc_bf16_f32(kRows, kChunk, false, false);
            constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(kRows, kHeadDim, false, true);
            bool ok = ptx::mbar_wait_warp(&bars[kQReady], 0, abort_flag, S.status);
            ptx::tc_fence_after();
            for (int j = 0; ok && j <= nchunks; ++j) {
                if (j < nchunks) {
                    const int st = j % kStages;
                    if (!ptx::mbar_wait_warp(&bars[kKFull + st], (j / kStages) & 1, abort_flag, S.status)) break;
                    ptx::tc_fence_after();
                    if (lane == 0) {
                        const uint32_t k_base = ptx::smem_u32(smem + kSmemK + st * kKVBytes);
                        const uint32_t d = tmem + ((j & 1) ? kColS1 : kColS0);
                        for (int ks = 0; ks < kHeadDim / 16; ++ks) {
                            // 16 dims = 32 bytes inside the 128-byte swizzle atom of slab ks / 4
                            const uint64_t bd = ptx::smem_desc(k_base + (ks >> 2) * kSlabKV + (ks & 3) * 32, 16,
                                                               1024, ptx::kSwizzle128B);
                            ptx::mma_ts(d, tmem + kColQ + 8 * ks, bd, idesc_qk, ks > 0 ? 1u : 0u);
                        }
                        ptx::mma_commit(&bars[kSFull + (j & 1)]);
                    }
                    __syncwarp();
                }
                if (j >= 1) {
                    const int jj = j - 1, st = jj % kStages;
                    if (!ptx::mbar_wait_warp(&bars[kPFull + (jj & 1)], (jj >> 1) & 1, abort_flag, S.status)) break;
                    if (!ptx::mbar_wait_warp(&bars[kVFull + st], (jj / kStages) & 1, abort_flag, S.status)) break;
                    // rows past the valid keys may hold stale bytes: zero them so P = 0 times V stays 0
                    int nvalid;
                    if (jj < n_ring) nvalid = fill - kChunk * jj;
                    else if (jj < n_ring + n_blk) nvalid = n - kChunk * (jj - n_ring);
                    else nvalid = bank_fill - kChunk * (jj - n_ring - n_blk);
                    if (nvalid < kChunk) {
                        uint8_t* vst = smem + kSmemV + st * kKVBytes;
                        const int nz = (kChunk - nvalid) * 8;   // 16-byte pieces per slab
                        for (int e = lane; e < 4 * nz; e += 32) {
                            const int slab = e / nz, piece = e % nz;
                            reinterpret_cast<uint4*>(vst + slab * kSlabKV + nvalid * 128)[piece] =
                                make_uint4(0, 0, 0, 0);
                        }
                        ptx::fence_proxy_async_smem();
                    }
                    __syncwarp();
                    ptx::tc_fence_after();
                    if (lane == 0) {
                        const uint32_t v_base = ptx::smem_u32(smem + kSmemV + st * kKVBytes);
                        const uint32_t a_col = tmem + ((jj & 1) ? kColS1 : kColS0);
                        for (int ks = 0; ks < kChunk / 16; ++ks) {
                            const uint64_t bd =
                                ptx::smem_desc(v_base + ks * 16 * 128, kSlabKV, 1024, ptx::kSwizzle128B);
                            ptx::mma_ts(tmem + kColO, a_col + 8 * ks, bd, idesc_pv, (jj > 0 || ks > 0) ? 1u : 0u);
                        }
                        ptx::mma_commit(&bars[kKVEmpty + st]);
                        ptx::mma_commit(&bars[kODone]);
                    }
                    __syncwarp();
                }
            }
            // the producer never waits on the last stages' kv_empty phases: consume them here
            // so that no commit is still pending when the CTA moves on
            for (int jj = max(0, nchunks - kStages); ok && jj < nchunks; ++jj)
                if (!ptx::mbar_wait_warp(&bars[kKVEmpty + jj % kStages], (jj / kStages) & 1, abort_flag, S.status))
                    break;
        } else {
            // ---------------- softmax: thread = (row, half) ----------------
            const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
            {
                // this half of the Q row -> tensor memory columns [384 + 64 wg, +64) as packed BF16
                const uint4* qrow =
                    reinterpret_cast<const uint4*>(a.q + ((size_t)(b * n + tok) * HQ + head) * kHeadDim) + 16 * wg;
                uint32_t r0[32], r1[32];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint4 v0 = __ldg(qrow + e), v1 = __ldg(qrow + 8 + e);
                    r0[4 * e] = v0.x; r0[4 * e + 1] = v0.y; r0[4 * e + 2] = v0.z; r0[4 * e + 3] = v0.w;
                    r1[4 * e] = v1.x; r1[4 * e + 1] = v1.y; r1[4 * e + 2] = v1.z; r1[4 * e + 3] = v1.w;
                }
                ptx::tmem_st32(lane_addr + kColQ + 64 * wg, r0);
                ptx::tmem_st32(lane_addr + kColQ + 64 * wg + 32, r1);
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&bars[kQReady]);
            }
            const int pq = s + tok;                    // query position
            const int w = (s - 1) % S.R;               // slot of position s - 1 (s >= 1)
            const int base_pos = s - 1 - w;
            const float qs = a.qscale;
            float m_used = -CUDART_INF_F;
            bool ok = true;
            // Every softmax thread runs every iteration and every named barrier, also after an
            // abort (then without touching tensor memory), so no thread is left waiting at one.
            for (int j = 0; j < nchunks; ++j) {
                const int sb = j & 1;
                if (ok) ok = ptx::mbar_wait_warp(&bars[kSFull + sb], (j >> 1) & 1, abort_flag, S.status);
                ok = __all_sync(0xffffffffu, ok);
                uint32_t sr[32];
                if (ok) {
                    ptx::tc_fence_after();
                    ptx::tmem_ld32(lane_addr + (sb ? kColS1 : kColS0) + 32 * wg, sr);
                    ptx::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) sr[i] = 0u;
                }
                // visibility of this thread's 32 keys: 0 all visible, 1 none, 2 per key
                int mode;
                uint32_t vis = 0;
                if (j < n_ring) {
                    const int slot0 = kChunk * j + 32 * wg;
                    if (slot0 >= fill) {
                        mode = 1;
                    } else {
                        const bool all_valid = slot0 + 31 < fill;
                        const bool wraps = (slot0 <= w) && (w < slot0 + 31) && (fill == S.R);
                        const int first = wraps ? w + 1 : slot0;            // the oldest slot of the range
                        const int pk_min = base_pos + first - (first > w ? S.R : 0);
                        mode = (all_valid && pk_min >= pq - S.R) ? 0 : 2;
                        if (mode == 2) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) {
                                const int slot = slot0 + i;
                                const int pk = base_pos + slot - (slot > w ? S.R : 0);
                                vis |= (uint32_t)((slot < fill) && (pk >= pq - S.R)) << i;
                            }
                        }
                    }
                } else if (j < n_ring + n_blk) {
                    const int t0 = kChunk * (j - n_ring) + 32 * wg;
                    if (t0 > tok || t0 >= n) {
                        mode = 1;
                    } else if (t0 + 31 <= tok && t0 + 31 < n) {
                        mode = 0;
                    } else {
                        mode = 2;
#pragma unroll
                        for (int i = 0; i < 32; ++i) vis |= (uint32_t)((t0 + i <= tok) && (t0 + i < n)) << i;
                    }
                } else {
                    const int a0 = kChunk * (j - n_ring - n_blk) + 32 * wg;
                    if (a0 >= bank_fill) {
                        mode = 1;
                    } else if (a0 + 31 < bank_fill) {
                        mode = 0;
                    } else {
                        mode = 2;
                        vis = (bank_fill - a0 >= 32) ? 0xffffffffu : ((1u << (bank_fill - a0)) - 1u);
                    }
                }
                if (mode == 0) vis = 0xffffffffu;
                // the row max over both halves (raw scores; the scale is positive)
                float m4[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
                if (mode != 1) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float v = ((vis >> i) & 1u) ? __uint_as_float(sr[i]) : -CUDART_INF_F;
                        m4[i & 3] = fmaxf(m4[i & 3], v);
                    }
                }
                float mloc = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * qs;
                xch[(sb * 2 + wg) * 128 + row] = mloc;
                ptx::named_bar_sync(1, kSoftmaxThreads);
                mloc = fmaxf(mloc, xch[(sb * 2 + (wg ^ 1)) * 128 + row]);
                float m_new = m_used;
                bool resc = false;
                if (mloc > m_used + 8.f) {
                    resc = (m_used != -CUDART_INF_F);
                    m_new = mloc;
                }
                const float fac = resc ? fast_ex2(m_used - m_new) : 1.f;
                const float mref = (m_new == -CUDART_INF_F) ? 0.f : m_new;
                m_used = m_new;
                float s4[4] = {0.f, 0.f, 0.f, 0.f};
                uint32_t pk[16];
                if (mode == 1) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = 0u;
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float e0 = fast_ex2(fmaf(__uint_as_float(sr[2 * i]), qs, -mref));
                        float e1 = fast_ex2(fmaf(__uint_as_float(sr[2 * i + 1]), qs, -mref));
                        e0 = ((vis >> (2 * i)) & 1u) ? e0 : 0.f;
                        e1 = ((vis >> (2 * i + 1)) & 1u) ? e1 : 0.f;
                        s4[i & 3] += e0 + e1;
                        pk[i] = pack_bf16(e0, e1);
                    }
                }
                l = l * fac + ((s4[0] + s4[1]) + (s4[2] + s4[3]));
                if (ok && j >= 1) ok = ptx::mbar_wait_warp(&bars[kODone], (j - 1) & 1, abort_flag, S.status);
                if (!ok) continue;
                ptx::tc_fence_after();
                if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        const uint32_t col = kColO + 128 * wg + 32 * c;
                        ptx::tmem_ld32(lane_addr + col, o);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * fac);
                        ptx::tmem_st32(lane_addr + col, o);
                    }
                }
                ptx::tmem_st16(lane_addr + (sb ? kColS1 : kColS0) + 16 * wg, pk);
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&bars[kPFull + sb]);
            }
            // both halves of a row used the same reference max: the row sum is the sum of halves
            xch[(4 + wg) * 128 + row] = l;
            ptx::named_bar_sync(1, kSoftmaxThreads);
            l += xch[(4 + (wg ^ 1)) * 128 + row];
            if (ok && ptx::mbar_wait_warp(&bars[kODone], (nchunks - 1) & 1, abort_flag, S.status)) {
                ptx::tc_fence_after();
                const float inv = (l > 0.f) ? 1.f / l : 0.f;
                float4* dst = reinterpret_cast<float4*>(own_rows + (size_t)row * kHeadDim + 128 * wg);
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    ptx::tmem_ld32(lane_addr + kColO + 128 * wg + 32 * c, o);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[c * 8 + i] =
                            make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                        __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
                }
                l = inv;   // from here on: the row's normalisation factor
            }
        }
    } else if (warp < 8) {
        // nothing to read (empty bank): this CTA's rows are zero
        float4* dst = reinterpret_cast<float4*>(own_rows + (size_t)row * kHeadDim + 128 * wg);
        for (int c = 0; c < 32; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }

    // ---------------- tail ----------------
    __threadfence();
    ptx::tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        const unsigned old = atomicAdd(S.tickets + bg, (1u << (2 * T)) + (1u << 16));
        tail_flags[0] = ((old >> (2 * T)) & 3u) != 0u;
        tail_flags[1] = (int)(old >> 16) == 2 * ntiles - 1;
    }
    __syncthreads();
    const bool partner_done = tail_flags[0] != 0, last_all = tail_flags[1] != 0;
    if (partner_done && warp < 8) {
        // out = local + gate * anchor; this thread: one row, one half of the dims
        __threadfence();
        ptx::tc_fence_after();
        const size_t qoff = ((size_t)(b * n + tok) * HQ + head) * kHeadDim;
        const uint4* qrow = reinterpret_cast<const uint4*>(a.q + qoff) + 16 * wg;
        const float4* wrow = reinterpret_cast<const float4*>(a.w_g + (size_t)head * kHeadDim + 128 * wg);
        float d = 0.f;
#pragma unroll 4
        for (int e = 0; e < 16; ++e) {
            const uint4 qv = __ldg(qrow + e);
            const float4 w0 = __ldg(wrow + 2 * e), w1 = __ldg(wrow + 2 * e + 1);
            d += __uint_as_float(qv.x << 16) * w0.x + __uint_as_float(qv.x & 0xffff0000u) * w0.y +
                 __uint_as_float(qv.y << 16) * w0.z + __uint_as_float(qv.y & 0xffff0000u) * w0.w +
                 __uint_as_float(qv.z << 16) * w1.x + __uint_as_float(qv.z & 0xffff0000u) * w1.y +
                 __uint_as_float(qv.w << 16) * w1.z + __uint_as_float(qv.w & 0xffff0000u) * w1.w;
        }
        xch[(6 + wg) * 128 + row] = d;
        ptx::named_bar_sync(1, kSoftmaxThreads);
        d += xch[(6 + (wg ^ 1)) * 128 + row];
        const float gate = tanhf(d + a.b_g[head]);
        // own result scaled by its normalisation (0 when there was nothing to read)
        const float c_own = (phase == 0 ? 1.f : gate) * (has_work ? l : 0.f);
        const float c_par = phase == 0 ? gate : 1.f;
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        const float4* prow = reinterpret_cast<const float4*>(partner_rows + (size_t)row * kHeadDim + 128 * wg);
        uint4* orow = reinterpret_cast<uint4*>(a.out + qoff) + 16 * wg;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            if (has_work) {
                ptx::tmem_ld32(lane_addr + kColO + 128 * wg + 32 * c, o);
                ptx::tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = 0u;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float4 p0 = __ldcg(prow + 8 * c + 2 * e), p1 = __ldcg(prow + 8 * c + 2 * e + 1);
                const float* ov = reinterpret_cast<const float*>(o) + 8 * e;
                uint4 r;
                r.x = pack_bf16(c_own * ov[0] + c_par * p0.x, c_own * ov[1] + c_par * p0.y);
                r.y = pack_bf16(c_own * ov[2] + c_par * p0.z, c_own * ov[3] + c_par * p0.w);
                r.z = pack_bf16(c_own * ov[4] + c_par * p1.x, c_own * ov[5] + c_par * p1.y);
                r.w = pack_bf16(c_own * ov[6] + c_par * p1.z, c_own * ov[7] + c_par * p1.w);
                orow[4 * c + e] = r;
            }
        }
    }
    if (has_work) {
        ptx::tc_fence_before();
        __syncthreads();
        if (warp == kWarpMma) {
            ptx::tc_fence_after();
            ptx::tmem_dealloc(tmem, kTmemCols);
        }
    }
    if (!last_all) return;

    // ---------------- last CTA of (b, g): commit the block, then the forced admit ----------------
    __threadfence();
    const bool fits = pend_fill + n <= S.P;
    constexpr int kPieces = kRowBytes / 16;   // 32 per row
    for (int e = tid; e < n * kPieces; e += kThreads) {
        const int i = e / kPieces, c = e % kPieces;
        const size_t src = ((size_t)(b * n + i) * G + g) * kHeadDim;
        const int slot = (s + i) % S.R;
        const size_t dst = ((size_t)bg * S.R + slot) * kHeadDim;
        reinterpret_cast<uint4*>(S.ring_k + dst)[c] = reinterpret_cast<const uint4*>(a.k + src)[c];
        reinterpret_cast<uint4*>(S.ring_v + dst)[c] = reinterpret_cast<const uint4*>(a.v + src)[c];
        if (fits) {
            const size_t pd = ((size_t)bg * S.P + pend_fill + i) * kHeadDim;
            reinterpret_cast<uint4*>(S.pend_k + pd)[c] = reinterpret_cast<const uint4*>(a.cand_k + src)[c];
            reinterpret_cast<uint4*>(S.pend_v + pd)[c] = reinterpret_cast<const uint4*>(a.cand_v + src)[c];
        }
    }
    if (fits)
        for (int i = tid; i < n; i += kThreads)
            S.pend_score[(size_t)bg * S.P + pend_fill + i] = a.cand_score[(size_t)(b * n + i) * G + g];
    const int np = fits ? pend_fill + n : pend_fill;
    __syncthreads();
    if (tid == 0) {
        int32_t* c = S.counters + bg * 4;
        c[0] = s + n;
        c[2] = np;
        if (!fits) atomicOr(S.status, (unsigned)RMA_STATUS_PREFILL_PENDING_OVERFLOW);
    }
    if (np > 0) admit_group<kThreads>(S, bg, bank_fill, np, smem);
    if (tid == 0) S.tickets[bg] = 0u;
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
    const int B = s.B, G = s.G, n = a.n_tok;
    if (n % kTileTok != 0 || n > kMaxTiles * kTileTok || n > s.R) return cudaErrorNotSupported;
    const int ntiles = n / kTileTok;
    Tmaps tm;
    const uint64_t row = (uint64_t)kHeadDim * 2;
    bool ok = make_map(&tm.k, a.k, G, (uint64_t)B * n, row, row * G, 1, kChunk) &&
              make_map(&tm.v, a.v, G, (uint64_t)B * n, row, row * G, 1, kChunk) &&
              make_map(&tm.ring_k, s.ring_k, s.R, (uint64_t)B * G, row, row * s.R, kChunk, 1) &&
              make_map(&tm.ring_v, s.ring_v, s.R, (uint64_t)B * G, row, row * s.R, kChunk, 1) &&
              make_map(&tm.bank_k, s.bank_k, s.A, (uint64_t)B * G, row, row * s.A, kChunk, 1) &&
              make_map(&tm.bank_v, s.bank_v, s.A, (uint64_t)B * G, row, row * s.A, kChunk, 1);
    if (!ok) return cudaErrorInvalidValue;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    prefill_kernel<<<dim3(2 * ntiles, G, B), kThreads, kSmemBytes, stream>>>(tm, a, ntiles);
    return cudaGetLastError();
}

}  // namespace rma
