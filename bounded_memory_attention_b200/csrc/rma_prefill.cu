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
// One launch.  A CTA owns 128 query rows (32 tokens x the group's 4 query
// heads, which share every key) and one phase: the local window (phase 0) or
// the bank (phase 1).  Four CTAs form a thread-block cluster:
//   rank 0: tile 2p, local     rank 1: tile 2p+1, local
//   rank 2: tile 2p, anchor    rank 3: tile 2p+1, anchor
// A block may hold any n from 1 to 256 tokens: the grid covers ceil(n / 64)
// pairs of tiles, rows past the last token repeat its query and are not
// stored, and keys past it are masked (their V rows cleared).
// Ranks (0,1) and (2,3) are CTA pairs for the 2-SM tensor-core MMA
// (tcgen05 cta_group::2, M = 256): both tiles of a pair read exactly the same
// keys, so each CTA loads only half of every 64-key K/V chunk (K rows split
// by key, V split by dimension), which halves the K/V bytes per FLOP.
//   * tensor memory (512 columns, the pair allocates together): O [0,256)
//     FP32, S double buffer [256,320) and [320,384) (chunk j in S_(j & 1)),
//     Q [384,512) packed BF16 (Q K^T takes A from tensor memory); shared
//     memory holds a five-stage ring of K/V half-chunks and one BF16 P buffer
//     per softmax group (the UMMA K-major layout, 128-byte swizzle);
//   * warp 8 of each CTA loads its half of each chunk with TMA (128B swizzle);
//   * in the even CTA, warps 9 and 11 issue S = Q K^T (N 64, K 256) for even
//     and odd chunks and warp 10 issues O += P V (N 256, K 64, P and V from
//     shared memory, V an MN-major operand), committing to the barriers of both
//     CTAs; the tensor pipe queues few instructions, and three issuers keep it
//     fed while any one waits.  Warp 9 of the odd CTA checks its half landed,
//     clears stale V rows and signals the even CTA;
//   * warps 0-7 of each CTA are the softmax for its own rows: two
//     warpgroups that take alternate chunks, each thread a whole 64-key row;
//     they load Q into tensor memory (and compute the gate), read S, release
//     its columns for Q K^T of chunk j + 2, mask by position (32-key halves
//     that are all visible skip the per-key test), hand the reference max from
//     chunk to chunk through shared memory (moving it only when a chunk's max
//     exceeds it by more than 2^8, then rescaling O), write P to shared memory,
//     keep one row sum per group and finally normalise O.
// Tail: every CTA writes its normalised rows into its own shared memory and
// pushes the 64 rows the other CTA of its tile (local <-> anchor) combines into
// that CTA's free stage area with one bulk copy (no multicast); each combines
// its half: out = local + gate * anchor in FP32, rounded once to BF16.  Each CTA
// appends its share of the candidates to pending; local pairs write the block's
// K/V into the ring as soon as every earlier pair has finished reading it; the
// last CTA of the (sequence, group) runs the forced admit.  No load is
// multicast: every CTA reads its own data.
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

constexpr int kTileTok = 32;                          // tokens per CTA
constexpr int kRows = kTileTok * kQPerGroup;          // 128 rows per CTA, 256 per pair
constexpr int kChunk = 64;                            // keys per chunk
constexpr int kHalfKeys = kChunk / 2;                 // K rows each CTA of a pair loads
constexpr int kSlabK = kHalfKeys * 128;               // 32 keys x 64 dims (bf16) = 4 KiB
constexpr int kSlabV = kChunk * 128;                  // 64 keys x 64 dims = 8 KiB
constexpr int kKHalfBytes = 4 * kSlabK;               // 16 KiB: this CTA's keys, all 256 dims
constexpr int kVHalfBytes = 2 * kSlabV;               // 16 KiB: all 64 keys, this CTA's 128 dims
constexpr int kStageBytes = kKHalfBytes + kVHalfBytes;
constexpr int kStages = 5;
constexpr int kSmemP = kStages * kStageBytes;         // 160 KiB: P of the two softmax groups
constexpr int kPBytes = 128 * 128;                    // 128 rows x 64 keys (BF16), 128-byte swizzle
constexpr int kSmemBar = kSmemP + 2 * kPBytes;        // 192 KiB
// softmax exchange (floats): the reference max handed between the groups [128] at 0, each
// group's final reference max [2][128] at 128 and row sum [2][128] at 512, the gate [128] at 768
// (first the two halves' partial dot products [2][128], then the gate itself in the first)
constexpr int kSmemXch = kSmemBar + 512;
constexpr int kSmemW = kSmemXch + 4096;               // w_g rows of the group's 4 heads (FP32)
constexpr int kSmemBytes = kSmemW + 4096 + 1024;      // + 1 KiB for alignment
constexpr int kXchEndM = 128, kXchEndL = 512, kXchGate = 768;
constexpr int kSoftmaxThreads = 256;                  // warps 0-7
// warp 8: TMA producer; warps 9 and 11: Q K^T issuers for even and odd chunks (even CTA;
// in the odd CTA warp 9 is the stale-row cleaner); warp 10: P V issuer (even CTA).  The
// tensor pipe queues few instructions, so it idles whenever its only issuer waits on a
// barrier; three issuing warps keep it fed while any one of them waits.
constexpr int kWarpTma = 8, kWarpQK = 9, kWarpPV = 10, kWarpQK2 = 11;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS0 = 256, kColS1 = 320, kColQ = 384;
constexpr int kTilesPerCluster = 2;

static_assert(kSmemBar >= kRows * 1024, "the result rows reuse the K/V stages");
static_assert(kSmemBar >= (int)admit_scratch_bytes(1, 4095), "the tail's admit reuses the K/V stages");

struct Tmaps {
    CUtensorMap k, v, ring_k, ring_v, bank_k, bank_v;   // K maps: 32-row boxes; V maps: 64-row boxes
};

enum Bar {
    kQReady = 0,                // even CTA: 16 arrivals (8 warps x 2 CTAs)
    kFull = 1,                  // [5] both: this CTA's own loads of the stage landed (tx bytes)
    kEmpty = 6,                 // [5] both: the MMA commit after P V of the chunk in that stage (the stage,
                                //     that P buffer and O are free to reuse)
    kSFull = 11,                // [2] both, one per softmax group: MMA commit after Q K^T
    kPFull = 13,                // [2] even CTA, per group: P is in shared memory, 8 arrivals (4 warps x 2 CTAs)
    kSFree = 15,                // [2] even CTA, per group: S has been read, 8 arrivals
    kXfer = 17,                 // both: the other CTA's half-result rows have landed (tx bytes)
    kOFinal = 18,               // both: MMA commit after the last P V (one phase)
    kPeer = 19,                 // [5] even CTA: the odd CTA's half of the stage landed and its stale V rows
                                //     are cleared (one remote arrival)
    kDrain = 24,                // both: one commit from each of the even CTA's three MMA-issuing warps after
                                //     its last MMA: every tensor-core operation of the pair has completed
    kNumBars = 25
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

__global__ void __cluster_dims__(4, 1, 1) __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ Tmaps tm, const __grid_constant__ PrefillArgs a, int ntiles) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const LayerView& S = a.s;
    const uint32_t rank = ptx::cluster_ctarank();
    const int pr = rank & 1;                     // 0: the pair's MMA-issuing CTA
    const int phase = rank >> 1;
    const int T = kTilesPerCluster * (blockIdx.x >> 2) + pr;
    const int g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = S.G, HQ = G * kQPerGroup, n = a.n_tok;
    const int bg = b * G + g;
    const uint32_t leader = rank & ~1u;
    const uint16_t pair_mask = (uint16_t)(3u << leader);

    const int32_t* cnt = S.counters + bg * 4;
    const int c_pos = cnt[0], c_bank = cnt[1], c_pend = cnt[2];
    if ((c_pos < 0 || c_bank < 0 || c_bank > S.A || c_pend < 0 || c_pend > S.P) && threadIdx.x == 0 && rank == 0 &&
        blockIdx.x == 0)
        atomicOr(S.status, (unsigned)RMA_STATUS_BAD_COUNTERS);   // a corrupted state: clamped below
    const int s = max(c_pos, 0);
    const int bank_fill = min(max(c_bank, 0), S.A);
    const int pend_fill = min(max(c_pend, 0), S.P);
    const int fill = min(s, S.R);

    // chunks (identical for both CTAs of a pair: tiles 2p and 2p+1 need block chunks 0..p)
    int n_ring = 0, n_blk = 0, n_bank = 0;
    if (phase == 0) {
        n_ring = (fill + kChunk - 1) / kChunk;
        n_blk = (kTileTok * (T | 1) + kTileTok - 1) / kChunk + 1;
    } else {
        n_bank = (bank_fill + kChunk - 1) / kChunk;
    }
    const int nchunks = n_ring + n_blk + n_bank;
    const bool has_work = nchunks > 0;        // uniform over the pair

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBar);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kNumBars + 1);
    int* tail_flag = reinterpret_cast<int*>(bars + kNumBars + 2);

    const int row = 32 * (warp & 3) + lane;   // softmax threads: row of this CTA
    const int wg = (warp >> 2) & 1;           // and which half of keys / columns
    const int tok = kTileTok * T + (row >> 2);
    const int head = g * kQPerGroup + (row & 3);
    float* xch = reinterpret_cast<float*>(smem + kSmemXch);
    float l = 0.f;
    uint32_t tmem = 0;

    if (tid == 0) {
        ptx::mbar_init(&bars[kQReady], 16);
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(&bars[kFull + i], 1);
            ptx::mbar_init(&bars[kEmpty + i], 1);
            ptx::mbar_init(&bars[kPeer + i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&bars[kSFull + i], 1);
            ptx::mbar_init(&bars[kPFull + i], 8);
            ptx::mbar_init(&bars[kSFree + i], 8);
        }
        ptx::mbar_init(&bars[kXfer], 1);
        ptx::mbar_init(&bars[kOFinal], 1);
        ptx::mbar_init(&bars[kDrain], 3);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (tid < kSoftmaxThreads)   // the gate weights of the group's heads, one float4 per thread
        reinterpret_cast<float4*>(smem + kSmemW)[tid] =
            __ldg(reinterpret_cast<const float4*>(a.w_g + (size_t)g * kQPerGroup * kHeadDim) + tid);
    if (has_work && warp == kWarpQK) {
        ptx::tmem_alloc2(tmem_holder, kTmemCols);
        ptx::tmem_relinquish2();
    }
    ptx::tc_fence_before();
    ptx::cluster_sync();   // barriers of all four CTAs initialised, tensor memory allocated
    ptx::tc_fence_after();
    if (has_work) tmem = *tmem_holder;

    // number of valid keys of chunk j (rows past it may hold stale bytes)
    auto chunk_valid = [&](int j) -> int {
        if (j < n_ring) return fill - kChunk * j;
        if (j < n_ring + n_blk) return n - kChunk * (j - n_ring);
        return bank_fill - kChunk * (j - n_ring - n_blk);
    };
    // clear V rows [nvalid, 64) of this CTA's half in stage st so that P = 0 times V stays 0
    auto clear_stale_v = [&](int j, int st) {
        const int nvalid = chunk_valid(j);
        if (nvalid < kChunk) {
            uint8_t* vst = smem + st * kStageBytes + kKHalfBytes;
            const int nz = (kChunk - nvalid) * 8;   // 16-byte pieces per slab
            for (int e = lane; e < 2 * nz; e += 32) {
                const int slab = e / nz, piece = e % nz;
                reinterpret_cast<uint4*>(vst + slab * kSlabV + nvalid * 128)[piece] = make_uint4(0, 0, 0, 0);
            }
            ptx::fence_proxy_async_smem();
        }
        __syncwarp();
    };

    if (has_work) {
        if (warp == kWarpTma) {
            // ---------------- TMA producer: this CTA's half of every chunk ----------------
            const int zreg = b * G + g;
            int issued = 0;
            for (int j = 0; j < nchunks; ++j) {
                const int st = j % kStages;
                if (j >= kStages &&
                    !ptx::mbar_wait_warp(&bars[kEmpty + st], ((j / kStages) - 1) & 1, abort_flag, S.status))
                    break;
                issued = j + 1;
                if (lane == 0) {
                    const CUtensorMap* mk;
                    const CUtensorMap* mv;
                    int yk, zk, yv, zv;
                    if (j < n_ring) {
                        mk = &tm.ring_k; mv = &tm.ring_v;
                        yk = kChunk * j + kHalfKeys * pr; zk = zreg; yv = kChunk * j; zv = zreg;
                    } else if (j < n_ring + n_blk) {
                        const int t0 = b * n + kChunk * (j - n_ring);
                        mk = &tm.k; mv = &tm.v;
                        yk = g; zk = t0 + kHalfKeys * pr; yv = g; zv = t0;
                    } else {
                        const int a0 = kChunk * (j - n_ring - n_blk);
                        mk = &tm.bank_k; mv = &tm.bank_v;
                        yk = a0 + kHalfKeys * pr; zk = zreg; yv = a0; zv = zreg;
                    }
                    uint8_t* stage = smem + st * kStageBytes;
                    ptx::mbar_arrive_expect_tx(&bars[kFull + st], kStageBytes);
                    for (int slab = 0; slab < 4; ++slab)
                        ptx::tma_load_3d(stage + slab * kSlabK, mk, &bars[kFull + st], 64 * slab, yk, zk);
                    for (int slab = 0; slab < 2; ++slab)
                        ptx::tma_load_3d(stage + kKHalfBytes + slab * kSlabV, mv, &bars[kFull + st],
                                         128 * pr + 64 * slab, yv, zv);
                }
                __syncwarp();
            }
            // Drain, normal or abandoned: this CTA's loads of the last stages have landed (earlier
            // stages were consumed before their reuse), and every MMA of the pair has completed.
            for (int jj = max(0, issued - kStages); jj < issued; ++jj)
                ptx::mbar_wait_drain(&bars[kFull + jj % kStages], (jj / kStages) & 1, S.status);
            ptx::mbar_wait_drain(&bars[kDrain], 0, S.status);
            __syncwarp();
        } else if (warp == kWarpQK && pr == 1) {
            // ---------------- odd CTA: check its half landed, clear stale rows, tell the even CTA ----------------
            for (int j = 0; j < nchunks; ++j) {
                const int st = j % kStages;
                if (!ptx::mbar_wait_warp(&bars[kFull + st], (j / kStages) & 1, abort_flag, S.status)) break;
                clear_stale_v(j, st);
                if (lane == 0) ptx::mbar_arrive_at(&bars[kPeer + st], leader, rank);
                __syncwarp();
            }
            for (int jj = max(0, nchunks - kStages); jj < nchunks; ++jj)
                if (!ptx::mbar_wait_warp(&bars[kEmpty + jj % kStages], (jj / kStages) & 1, abort_flag, S.status))
                    break;
        } else if (warp == kWarpQK || (warp == kWarpQK2 && pr == 0)) {
            // ---------------- even CTA: Q K^T issuers (warp 9: even chunks, warp 11: odd) ----------------
            // S of chunk j lives in columns kColS0 / kColS1 by j & 1 and P in shared memory, so
            // Q K^T of chunk j + 2 may start as soon as the softmax group has read S of chunk j.
            constexpr uint32_t idesc_qk = ptx::idesc_bf16_f32(2 * kRows, kChunk, false, false);
            bool ok = ptx::mbar_wait_warp(&bars[kQReady], 0, abort_flag, S.status);
            ptx::tc_fence_after();
            for (int j = warp == kWarpQK ? 0 : 1; ok && j < nchunks; j += 2) {
                if (j >= 2) {
                    ok = ptx::mbar_wait_warp(&bars[kSFree + (j & 1)], ((j - 2) >> 1) & 1, abort_flag, S.status);
                    if (!ok) break;
                }
                const int st = j % kStages;
                ok = ptx::mbar_wait_warp(&bars[kFull + st], (j / kStages) & 1, abort_flag, S.status);
                if (!ok) break;
                ok = ptx::mbar_wait_warp(&bars[kPeer + st], (j / kStages) & 1, abort_flag, S.status);
                if (!ok) break;
                clear_stale_v(j, st);
                ptx::tc_fence_after();
                if (lane == 0) {
                    const uint32_t k_base = ptx::smem_u32(smem + st * kStageBytes);
                    const uint32_t d = tmem + ((j & 1) ? kColS1 : kColS0);
                    for (int ks = 0; ks < kHeadDim / 16; ++ks) {
                        // 16 dims = 32 bytes inside the 128-byte swizzle atom of slab ks / 4
                        const uint64_t bd = ptx::smem_desc(k_base + (ks >> 2) * kSlabK + (ks & 3) * 32, 16, 1024,
                                                           ptx::kSwizzle128B);
                        ptx::mma_ts2(d, tmem + kColQ + 8 * ks, bd, idesc_qk, ks > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit2_mc(&bars[kSFull + (j & 1)], pair_mask);
                }
                __syncwarp();
            }
            if (lane == 0) ptx::mma_commit2_mc(&bars[kDrain], pair_mask);   // after this warp's last MMA
            __syncwarp();
        } else if (warp == kWarpPV && pr == 0) {
            // ---------------- even CTA: P V issuer ----------------
            // P V of chunk j needs P (which the softmax writes only after reading S of chunk j,
            // so Q K^T of chunk j has completed) and V (landed before Q K^T of chunk j was issued).
            constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(2 * kRows, kHeadDim, false, true);
            bool ok = true;
            for (int j = 0; ok && j < nchunks; ++j) {
                const int st = j % kStages;
                ok = ptx::mbar_wait_warp(&bars[kPFull + (j & 1)], (j >> 1) & 1, abort_flag, S.status);
                if (!ok) break;
                ptx::tc_fence_after();
                if (lane == 0) {
                    const uint32_t v_base = ptx::smem_u32(smem + st * kStageBytes + kKHalfBytes);
                    const uint32_t p_base = ptx::smem_u32(smem + kSmemP + (j & 1) * kPBytes);
                    for (int ks = 0; ks < kChunk / 16; ++ks) {
                        const uint64_t ad = ptx::smem_desc(p_base + ks * 32, 16, 1024, ptx::kSwizzle128B);
                        const uint64_t bd = ptx::smem_desc(v_base + ks * 16 * 128, kSlabV, 1024, ptx::kSwizzle128B);
                        ptx::mma_ss2(tmem + kColO, ad, bd, idesc_pv, (j > 0 || ks > 0) ? 1u : 0u);
                    }
                    ptx::mma_commit2_mc(&bars[kEmpty + st], pair_mask);
                }
                __syncwarp();
            }
            if (ok && lane == 0) ptx::mma_commit2_mc(&bars[kOFinal], pair_mask);
            __syncwarp();
            // consume the last stages' empty phases (the producer never waits on them) so that no
            // commit is still pending when the CTA moves on
            for (int jj = max(0, nchunks - kStages); ok && jj < nchunks; ++jj)
                if (!ptx::mbar_wait_warp(&bars[kEmpty + jj % kStages], (jj / kStages) & 1, abort_flag, S.status))
                    break;
            if (lane == 0) ptx::mma_commit2_mc(&bars[kDrain], pair_mask);   // after this warp's last MMA
            __syncwarp();
        } else if (warp < 8) {
            // ---------------- softmax: thread = (row, half) ----------------
            const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
            {
                // this half of the Q row -> tensor memory columns [384 + 64 wg, +64) as packed BF16
                // (rows past the block's last token repeat its query; their results are not stored)
                const uint4* qrow =
                    reinterpret_cast<const uint4*>(a.q + ((size_t)(b * n + min(tok, n - 1)) * HQ + head) * kHeadDim) +
                    16 * wg;
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
                if (lane == 0) ptx::mbar_arrive_at(&bars[kQReady], leader, rank);
                // this half's part of q . w_g for the gate (the Q row is read again, from L1),
                // while the first Q K^T runs
                const float4* wrow = reinterpret_cast<const float4*>(smem + kSmemW) + ((row & 3) * kHeadDim + 128 * wg) / 4;
                float gd = 0.f;
#pragma unroll 2
                for (int e = 0; e < 16; ++e) {
                    const uint4 u = __ldg(qrow + e);
                    const float4 w0 = wrow[2 * e], w1 = wrow[2 * e + 1];
                    gd += __uint_as_float(u.x << 16) * w0.x + __uint_as_float(u.x & 0xffff0000u) * w0.y +
                          __uint_as_float(u.y << 16) * w0.z + __uint_as_float(u.y & 0xffff0000u) * w0.w +
                          __uint_as_float(u.z << 16) * w1.x + __uint_as_float(u.z & 0xffff0000u) * w1.y +
                          __uint_as_float(u.w << 16) * w1.z + __uint_as_float(u.w & 0xffff0000u) * w1.w;
                }
                xch[kXchGate + wg * 128 + row] = gd;
                ptx::named_bar_sync(1, kSoftmaxThreads);
                if (wg == 0) {
                    const float gsum = xch[kXchGate + row] + xch[kXchGate + 128 + row];
                    xch[kXchGate + row] = tanhf(gsum + a.b_g[head]);
                }
            }
            const int pq = s + tok;                    // query position
            const int w = (s - 1) % S.R;               // slot of position s - 1 (s >= 1)
            const int base_pos = s - 1 - w;
            const float qs = a.qscale;
            // which of keys [32 h, 32 h + 32) of chunk j this row sees, one bit per key
            auto vis32 = [&](int j, int h) -> uint32_t {
                if (j < n_ring) {
                    const int slot0 = kChunk * j + 32 * h;
                    if (slot0 >= fill) return 0u;
                    const bool all_valid = slot0 + 31 < fill;
                    const bool wraps = (slot0 <= w) && (w < slot0 + 31) && (fill == S.R);
                    const int first = wraps ? w + 1 : slot0;   // the oldest slot of the range
                    const int pk_min = base_pos + first - (first > w ? S.R : 0);
                    if (all_valid && pk_min >= pq - S.R) return 0xffffffffu;
                    uint32_t v = 0;
#pragma unroll 4
                    for (int i = 0; i < 32; ++i) {
                        const int slot = slot0 + i;
                        const int pk = base_pos + slot - (slot > w ? S.R : 0);
                        v |= (uint32_t)((slot < fill) && (pk >= pq - S.R)) << i;
                    }
                    return v;
                }
                if (j < n_ring + n_blk) {
                    const int t0 = kChunk * (j - n_ring) + 32 * h;
                    if (t0 > tok || t0 >= n) return 0u;
                    const int last = min(tok, n - 1) - t0;     // keys t0 .. t0 + last are visible
                    return last >= 31 ? 0xffffffffu : ((2u << last) - 1u);
                }
                const int a0 = kChunk * (j - n_ring - n_blk) + 32 * h;
                if (a0 >= bank_fill) return 0u;
                return (bank_fill - a0 >= 32) ? 0xffffffffu : ((1u << (bank_fill - a0)) - 1u);
            };
            // The two warpgroups take alternate chunks (this one: j = wg, wg + 2, ...), each a whole
            // row of 64 keys. The reference max is handed from chunk to chunk through shared memory
            // (named barrier 2 + wg: this group's value is ready); each group keeps its own row sum
            // against the reference of its latest chunk.
            const uint32_t scol = wg ? kColS1 : kColS0;
            float m_w = -CUDART_INF_F;
            bool ok = true;
            for (int j = wg; j < nchunks; j += 2) {
                const uint32_t vlo = vis32(j, 0), vhi = vis32(j, 1);
                if (ok) ok = ptx::mbar_wait_warp(&bars[kSFull + wg], (j >> 1) & 1, abort_flag, S.status);
                ok = __all_sync(0xffffffffu, ok);
                uint32_t sa[32], sb[32];   // keys [0, 32) and [32, 64)
                if (ok) {
                    ptx::tc_fence_after();
                    ptx::tmem_ld32(lane_addr + scol, sa);
                    ptx::tmem_ld32(lane_addr + scol + 32, sb);
                    ptx::tmem_wait_ld();
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive_at(&bars[kSFree + wg], leader, rank);   // S may be overwritten
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) sa[i] = sb[i] = 0u;
                }
#define SR(i) __uint_as_float((i) < 32 ? sa[(i) & 31] : sb[(i) & 31])
                const bool full = (vlo & vhi) == 0xffffffffu;
                // the chunk's row max (raw scores; the scale is positive)
                float m4[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
                if (full) {
#pragma unroll
                    for (int i = 0; i < 64; ++i) m4[i & 3] = fmaxf(m4[i & 3], SR(i));
                } else {
#pragma unroll
                    for (int i = 0; i < 64; ++i) {
                        const uint32_t bit = ((i < 32 ? vlo : vhi) >> (i & 31)) & 1u;
                        m4[i & 3] = fmaxf(m4[i & 3], bit ? SR(i) : -CUDART_INF_F);
                    }
                }
                const float mloc = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * qs;
                float m_prev = -CUDART_INF_F;          // the reference O holds after chunk j - 1
                if (j >= 1) {
                    ptx::named_bar_sync(2 + (wg ^ 1), kSoftmaxThreads);
                    m_prev = xch[row];
                }
                float m_new = m_prev;
                bool resc = false;
                if (mloc > m_prev + 8.f) {
                    resc = (m_prev != -CUDART_INF_F);
                    m_new = mloc;
                }
                if (j + 1 < nchunks) {
                    xch[row] = m_new;
                    ptx::named_bar_arrive(2 + wg, kSoftmaxThreads);
                }
                const float mref = (m_new == -CUDART_INF_F) ? 0.f : m_new;
                const float fac_l = (m_w == m_new) ? 1.f : (m_w == -CUDART_INF_F ? 0.f : fast_ex2(m_w - m_new));
                m_w = m_new;
                float s4[4] = {0.f, 0.f, 0.f, 0.f};
                uint32_t pa[16], pb[16];
                if (full) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float e0 = fast_ex2(fmaf(SR(2 * i), qs, -mref));
                        const float e1 = fast_ex2(fmaf(SR(2 * i + 1), qs, -mref));
                        s4[i & 3] += e0 + e1;
                        (i < 16 ? pa[i & 15] : pb[i & 15]) = pack_bf16(e0, e1);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const uint32_t bits = ((i < 16 ? vlo : vhi) >> ((2 * i) & 31)) & 3u;
                        float e0 = fast_ex2(fmaf(SR(2 * i), qs, -mref));
                        float e1 = fast_ex2(fmaf(SR(2 * i + 1), qs, -mref));
                        e0 = (bits & 1u) ? e0 : 0.f;
                        e1 = (bits & 2u) ? e1 : 0.f;
                        s4[i & 3] += e0 + e1;
                        (i < 16 ? pa[i & 15] : pb[i & 15]) = pack_bf16(e0, e1);
                    }
                }
                l = l * fac_l + ((s4[0] + s4[1]) + (s4[2] + s4[3]));
                // O may be rescaled only once P V of chunk j - 1 (the other group's) has completed,
                // and this group's P buffer is free once P V of chunk j - 2 has; both are the
                // stage barriers of those chunks.  P V runs in chunk order and this group saw
                // P V of chunk j - 4 complete, so each barrier is at most one phase behind.
                const bool rescale_warp = __any_sync(0xffffffffu, resc);
                if (ok && rescale_warp)
                    ok = ptx::mbar_wait_warp(&bars[kEmpty + (j - 1) % kStages], ((j - 1) / kStages) & 1, abort_flag,
                                             S.status);
                if (ok && j >= 2)
                    ok = ptx::mbar_wait_warp(&bars[kEmpty + (j - 2) % kStages], ((j - 2) / kStages) & 1, abort_flag,
                                             S.status);
                if (!ok) continue;
                if (rescale_warp) {
                    ptx::tc_fence_after();
                    const float fac = resc ? fast_ex2(m_prev - m_new) : 1.f;
#pragma unroll 1
                    for (int c = 0; c < 8; ++c) {
                        uint32_t o[32];
                        const uint32_t col = kColO + 32 * c;
                        ptx::tmem_ld32(lane_addr + col, o);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * fac);
                        ptx::tmem_st32(lane_addr + col, o);
                    }
                    ptx::tmem_wait_st();
                }
#undef SR
                // P row: 64 keys as BF16 = 128 bytes, 16-byte pieces swizzled by the row within its 8-row atom
                uint8_t* prow = smem + kSmemP + wg * kPBytes + row * 128;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) << 4)) =
                        make_uint4(pa[4 * c], pa[4 * c + 1], pa[4 * c + 2], pa[4 * c + 3]);
                    *reinterpret_cast<uint4*>(prow + (((c + 4) ^ (row & 7)) << 4)) =
                        make_uint4(pb[4 * c], pb[4 * c + 1], pb[4 * c + 2], pb[4 * c + 3]);
                }
                ptx::fence_proxy_async_smem();   // P is read by the tensor cores
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive_at(&bars[kPFull + wg], leader, rank);
            }
            // the row sum over both groups, on the last chunk's reference (references only grow)
            xch[kXchEndL + wg * 128 + row] = l;
            xch[kXchEndM + wg * 128 + row] = m_w;
            ptx::named_bar_sync(1, kSoftmaxThreads);
            {
                const float lo = xch[kXchEndL + (wg ^ 1) * 128 + row];
                const float mo = xch[kXchEndM + (wg ^ 1) * 128 + row];
                const float mf = fmaxf(m_w, mo);
                float lt = 0.f;
                if (m_w != -CUDART_INF_F) lt += l * fast_ex2(m_w - mf);
                if (mo != -CUDART_INF_F) lt += lo * fast_ex2(mo - mf);
                l = lt;
            }
            const bool done = ok && ptx::mbar_wait_warp(&bars[kOFinal], 0, abort_flag, S.status);
            // every MMA of the pair has completed (or the CTA gave up): the K/V stages are free
            ptx::named_bar_sync(1, kSoftmaxThreads);
            if (done) ptx::tc_fence_after();
            const float inv = (done && l > 0.f) ? 1.f / l : 0.f;
            uint8_t* rrow = smem + (size_t)row * 1024;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                if (done) {
                    ptx::tmem_ld32(lane_addr + kColO + 128 * wg + 32 * c, o);
                    ptx::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0u;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int piece = 32 * wg + 8 * c + i;
                    *reinterpret_cast<float4*>(rrow + ((piece ^ (row & 7)) << 4)) =
                        make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                    __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
                }
            }
            ptx::fence_proxy_async_smem();   // the rows leave through a bulk copy
        }
    } else if (warp < 8) {
        // nothing to read (empty bank): this CTA's rows are zero (and so is the anchor's gate term)
        for (int c = 0; c < 32; ++c)
            *reinterpret_cast<float4*>(smem + (size_t)row * 1024 + ((32 * wg + c) << 4)) = make_float4(0.f, 0.f, 0.f, 0.f);
        if (wg == 0) xch[kXchGate + row] = 0.f;
        ptx::fence_proxy_async_smem();
    }

    // ---------------- tail ----------------
    // The local CTA of this tile combines rows [0, 64), the anchor CTA rows [64, 128): each first
    // pushes the 64 rows the other one needs into that CTA's free stage area [128 KiB, 192 KiB).
    // The cluster barrier below follows the producer warp's drain: this CTA's loads have landed and
    // every tensor-core operation of its pair has completed, also after a wait ran out and the CTA
    // abandoned its tile, so tensor memory may be freed and the stage area reused.
    __syncwarp();
    ptx::tc_fence_before();
    ptx::cluster_sync();   // all four CTAs have their rows in shared memory; all tensor memory reads done
    if (has_work && warp == kWarpQK) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc2(tmem, kTmemCols);
    }
    const uint32_t peer = rank ^ 2u;
    if (tid == 0) {
        ptx::mbar_arrive_expect_tx(&bars[kXfer], 64 * 1024);
        const uint32_t src = ptx::smem_u32(smem) + (uint32_t)(64 * (1 - phase)) * 1024u;
        const uint32_t dst = ptx::cluster_map(ptx::smem_u32(smem) + 128u * 1024u, peer);
        const uint32_t rbar = ptx::cluster_map(ptx::smem_u32(&bars[kXfer]), peer);
        ptx::bulk_copy_to_peer(dst, src, 64 * 1024, rbar);
        ptx::bulk_commit();
    }
    if (warp < 8) {
        // one row per warp at a time: lane L makes output dims [8 L, 8 L + 8) (16 contiguous bytes)
        // the partner's copy always comes: wait for it even after an abort, so that it has landed
        // before this CTA exits
        const bool got = ptx::mbar_wait_drain(&bars[kXfer], 0, S.status);
#pragma unroll 2
        for (int rr = 0; rr < 8; ++rr) {
            const int lrow = 8 * warp + rr, crow = 64 * phase + lrow;
            const int ctok = kTileTok * T + (crow >> 2), chead = g * kQPerGroup + (crow & 3);
            const float gate = xch[kXchGate + crow];
            const uint32_t off0 = (uint32_t)(((2 * lane) ^ (crow & 7)) << 4);
            const uint32_t off1 = (uint32_t)(((2 * lane + 1) ^ (crow & 7)) << 4);
            const uint8_t* mrow = smem + (size_t)crow * 1024;
            const uint8_t* prow = smem + 128 * 1024 + (size_t)lrow * 1024;
            const float4 m0 = *reinterpret_cast<const float4*>(mrow + off0);
            const float4 m1 = *reinterpret_cast<const float4*>(mrow + off1);
            float4 t0 = make_float4(0.f, 0.f, 0.f, 0.f), t1 = t0;
            if (got) {
                t0 = *reinterpret_cast<const float4*>(prow + off0);
                t1 = *reinterpret_cast<const float4*>(prow + off1);
            }
            const float4 l0 = phase == 0 ? m0 : t0, l1 = phase == 0 ? m1 : t1;
            const float4 c0 = phase == 0 ? t0 : m0, c1 = phase == 0 ? t1 : m1;
            uint4 r;
            r.x = pack_bf16(l0.x + gate * c0.x, l0.y + gate * c0.y);
            r.y = pack_bf16(l0.z + gate * c0.z, l0.w + gate * c0.w);
            r.z = pack_bf16(l1.x + gate * c1.x, l1.y + gate * c1.y);
            r.w = pack_bf16(l1.z + gate * c1.z, l1.w + gate * c1.w);
            if (ctok < n) reinterpret_cast<uint4*>(a.out + ((size_t)(b * n + ctok) * HQ + chead) * kHeadDim)[lane] = r;
        }
    }
    if (tid == 0) ptx::bulk_wait_read_all();   // the outgoing copy has read this CTA's rows

    // Ring write.  The slot of block token i holds position s + i - R, which queries up to token i
    // still read, so the rows of tile T (tokens [32 T, 32 T + 32)) may be written once tiles 0..T
    // have finished reading the ring; both CTAs of a local pair are done here (the cluster barrier
    // above follows every MMA of the pair).  Each local CTA marks its tile in bits 8.. of the
    // group's ticket word and writes the rows of every tile its mark completes the prefix for (the
    // count of finished CTAs is in bits 0..7).
    if (phase == 0) {
        int* range = tail_flag + 1;
        if (tid == 0) {
            __threadfence();
            const unsigned bit = 1u << (8 + T);
            const unsigned old = atomicOr(S.tickets + bg, bit) >> 8;
            __threadfence();
            range[0] = __ffs(~old) - 1;            // tiles done in a row before this mark
            range[1] = __ffs(~(old | (bit >> 8))) - 1;   // and after it
        }
        __syncthreads();
        const int t0 = min(n, kTileTok * range[0]), t1 = min(n, kTileTok * range[1]);
        copy_pieces<kThreads, 8>((t1 - t0) * 2 * kRowBytes / 16, [&](int e, const uint4*& from_p, uint4*& to_p) {
            constexpr int kP = kRowBytes / 16;
            const int i = t0 + e / (2 * kP), c = e % (2 * kP);
            const size_t src = ((size_t)(b * n + i) * G + g) * kHeadDim;
            const size_t dst = ((size_t)bg * S.R + (s + i) % S.R) * kHeadDim;
            if (c < kP) {
                from_p = reinterpret_cast<const uint4*>(a.k + src) + c;
                to_p = reinterpret_cast<uint4*>(S.ring_k + dst) + c;
            } else {
                from_p = reinterpret_cast<const uint4*>(a.v + src) + (c - kP);
                to_p = reinterpret_cast<uint4*>(S.ring_v + dst) + (c - kP);
            }
        });
    }

    // This CTA's share of the candidates goes to pending now (nothing in this launch reads those
    // slots before the last CTA's admit).
    const bool fits = pend_fill + n <= S.P;
    constexpr int kPieces = kRowBytes / 16;   // 32 per row
    const int nct = gridDim.x, share = (n + nct - 1) / nct;
    const int i0 = min(n, (int)blockIdx.x * share), i1 = min(n, i0 + share);
    if (fits) {
        copy_pieces<kThreads, 4>((i1 - i0) * 2 * kPieces, [&](int e, const uint4*& from_p, uint4*& to_p) {
            const int i = i0 + e / (2 * kPieces), c = e % (2 * kPieces);
            const size_t src = ((size_t)(b * n + i) * G + g) * kHeadDim;
            const size_t pd = ((size_t)bg * S.P + pend_fill + i) * kHeadDim;
            if (c < kPieces) {
                from_p = reinterpret_cast<const uint4*>(a.cand_k + src) + c;
                to_p = reinterpret_cast<uint4*>(S.pend_k + pd) + c;
            } else {
                from_p = reinterpret_cast<const uint4*>(a.cand_v + src) + (c - kPieces);
                to_p = reinterpret_cast<uint4*>(S.pend_v + pd) + (c - kPieces);
            }
        });
        for (int i = i0 + tid; i < i1; i += kThreads)
            S.pend_score[(size_t)bg * S.P + pend_fill + i] = a.cand_score[(size_t)(b * n + i) * G + g];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned old = atomicAdd(S.tickets + bg, 1u);
        *tail_flag = (int)(old & 0xFFu) == 2 * ntiles - 1;
    }
    __syncthreads();
    if (*tail_flag == 0) return;

    // ---------------- last CTA of (b, g): the forced admit ----------------
    __threadfence();
    const int np = fits ? pend_fill + n : pend_fill;
    __syncthreads();
    if (tid == 0) {
        int32_t* c = S.counters + bg * 4;
        c[0] = s + n;
        c[2] = np;
        if (!fits) atomicOr(S.status, (unsigned)RMA_STATUS_PREFILL_PENDING_OVERFLOW);
    }
    if (np > 0) admit_group<kThreads, 16>(S, bg, bank_fill, np, smem);
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
    // the tile CTAs exchange their rows through distributed shared memory: no device scratch
    (void)cfg;
    (void)n_tok;
    return 256;
}

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream) {
    const LayerView& s = a.s;
    const int B = s.B, G = s.G, n = a.n_tok;
    // tiles come in pairs (64 tokens, the last one possibly ragged); the ticket counts 2 * ntiles
    // arrivals in 8 bits and marks one bit per tile in bits 8..15
    if (n < 1 || n > kMaxPrefillTokens || n > s.R) return cudaErrorNotSupported;
    const int ntiles = kTilesPerCluster * ((n + kTilesPerCluster * kTileTok - 1) / (kTilesPerCluster * kTileTok));
    Tmaps tm;
    const uint64_t row = (uint64_t)kHeadDim * 2;
    bool ok = make_map(&tm.k, a.k, G, (uint64_t)B * n, row, row * G, 1, kHalfKeys) &&
              make_map(&tm.v, a.v, G, (uint64_t)B * n, row, row * G, 1, kChunk) &&
              make_map(&tm.ring_k, s.ring_k, s.R, (uint64_t)B * G, row, row * s.R, kHalfKeys, 1) &&
              make_map(&tm.ring_v, s.ring_v, s.R, (uint64_t)B * G, row, row * s.R, kChunk, 1) &&
              make_map(&tm.bank_k, s.bank_k, s.A, (uint64_t)B * G, row, row * s.A, kHalfKeys, 1) &&
              make_map(&tm.bank_v, s.bank_v, s.A, (uint64_t)B * G, row, row * s.A, kChunk, 1);
    if (!ok) return cudaErrorInvalidValue;
    static SmemLimit limit(reinterpret_cast<const void*>(prefill_kernel));
    const cudaError_t e = limit.ensure(kSmemBytes);
    if (e != cudaSuccess) return e;
    // grid x: clusters of 4 CTAs, one per pair of tiles; ranks (local, local, anchor, anchor)
    prefill_kernel<<<dim3(2 * ntiles, G, B), kThreads, kSmemBytes, stream>>>(tm, a, ntiles);
    return cudaGetLastError();
}

}  // namespace rma
