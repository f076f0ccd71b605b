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
// Three launches.
//
// 1. prefill_attn_kernel, persistent: clusters of 2 CTAs, one CTA per SM, as
//    few as keep the most items per cluster at its minimum (the SMs left over
//    run the commit of finished groups), each looping over work items.  An
//    item is one (sequence, group, pair of tiles, phase): a tile is 32 tokens
//    x the group's 4 query heads =
//    128 query rows, the two tiles of a pair are the two CTAs of a tcgen05
//    cta_group::2 MMA pair (M = 256; both read exactly the same keys, so each
//    CTA loads only half of every 64-key K/V chunk), and the phase is the local
//    window (ring + block, causal) or the bank.  Items run in (sequence,
//    group)-major order, a group's local items before its anchor items.  Per
//    CTA and item:
//      * tensor memory (512 columns, allocated once): O [0,256) FP32, S double
//        buffer [256,320) / [320,384), Q [384,512) packed BF16 (Q K^T takes A
//        from tensor memory); shared memory holds a five-stage ring of K/V
//        half-chunks (128-byte swizzle) and one BF16 P buffer per softmax group;
//      * warp 8 loads this CTA's half of each chunk with TMA; in the even CTA
//        warps 9 and 11 issue S = Q K^T for even and odd chunks and warp 10
//        issues O += P V (the tensor pipe queues few instructions, so three
//        issuers keep it fed); warp 9 of the odd CTA checks its half landed,
//        clears stale V rows and signals the even CTA;
//      * warps 0-7 are the softmax: two groups taking alternate chunks, each
//        thread a whole 64-key row, the reference max handed from chunk to chunk
//        through shared memory (moved only when a chunk's max exceeds it by more
//        than 2^8, O rescaled then).  At the end of the item they write the
//        normalised rows (FP32) to the workspace, 32 columns at a time through
//        their P buffer and a TMA store per warp (its 32 rows), and go on to the
//        next item, whose first K/V chunks are already loaded and whose query
//        rows the TMA warp has asked L2 for; the P V issuer starts that item's
//        P V once both CTAs have read O.
//    Every barrier phase follows a chunk counter (or a counter of the items
//    that have chunks) running on across items.  A group's counters are
//    constant while any of its items runs: the second launch writes them only
//    after every item of the group has finished.
// 2. prefill_commit_kernel, launched with programmatic stream serialisation
//    so that its CTAs are scheduled as soon as SMs free up: per (sequence,
//    group), slice CTAs append their tokens' candidates to pending and compute
//    the gate tanh(q . w_g + b_g) of their rows at once (neither is read by the
//    first launch), wait until every item of their group has stored its rows
//    (each softmax warp counts its rows of an item in the high half of the
//    group's ticket word once its TMA stores have completed; items run in
//    group-major order, so most groups are done well before the last), then
//    combine out = local +
//    gate * anchor in FP32, rounded once to BF16, and write the block's K/V into
//    the ring (every read of the group's ring is done); one CTA runs the forced
//    admit's competition (scores only, no wait) and leaves the list of admitted
//    candidates and their bank slots in the workspace; the last CTA of the group
//    to arrive writes the counters.
// 3. prefill_admit_copy_kernel, launched the same way after the commit, which
//    it waits for with griddepcontrol.wait (and so for every item of every
//    group): the admitted rows (pending rows, or the block's own candidates from
//    the inputs) into their bank slots.
// No load is multicast: every CTA reads its own data.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <algorithm>
#include <atomic>
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
// group's final reference max [2][128] at 128 and row sum [2][128] at 512
constexpr int kSmemXch = kSmemBar + 512;
constexpr int kSmemBytes = kSmemXch + 4096 + 1024;    // + 1 KiB for alignment
constexpr int kXchEndM = 128, kXchEndL = 512;
constexpr int kSoftmaxThreads = 256;                  // warps 0-7
constexpr int kWarpTma = 8, kWarpQK = 9, kWarpPV = 10, kWarpQK2 = 11;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS0 = 256, kColS1 = 320, kColQ = 384;
constexpr int kCommitThreads = 256;
constexpr int kCommitSlices = 32;                     // slice CTAs per (sequence, group) in the commit
constexpr int kCommitUnroll = 4;                      // combine tokens a thread loads before it stores
constexpr int kCommitMaxTok = 8;                      // tokens of one slice: 256 / kCommitSlices
static_assert(kMaxPrefillTokens <= kCommitSlices * kCommitMaxTok, "a slice holds at most kCommitMaxTok tokens");

static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");

struct Tmaps {
    CUtensorMap k, v, ring_k, ring_v, bank_k, bank_v;   // K maps: 32-row boxes; V maps: 64-row boxes
    CUtensorMap ws;   // FP32 [phase][b][t][head][256], boxes of 32 dims x 4 heads x 8 tokens (one warp's rows)
};

enum Bar {
    kQReady = 0,      // even CTA, per item with chunks: 16 arrivals (8 softmax warps x 2 CTAs): Q in TMEM
    kFull = 1,        // [5] both: this CTA's own loads of the stage landed (tx bytes)
    kEmpty = 6,       // [5] both: MMA commit after P V of the chunk in that stage
    kSFull = 11,      // [2] both: MMA commit after Q K^T into S buffer jg & 1
    kPFull = 13,      // [2] even CTA: P of chunk jg in shared memory, 8 arrivals (4 warps x 2 CTAs)
    kSFree = 15,      // [2] even CTA: S of chunk jg read, 8 arrivals
    kOFinal = 17,     // both, per item with chunks: MMA commit after the item's last P V
    kODrained = 18,   // even CTA, per item with chunks: O read by the 8 softmax warps of both CTAs (16)
    kPeer = 19,       // [5] even CTA: the odd CTA's half of the stage landed, stale V rows cleared
    kDrain = 24,      // both: one commit from each of the even CTA's three MMA-issuing warps after its last MMA
    kNumBars = 25
};

// The workspace: normalised local rows and anchor rows, each [B][n][HQ][256] FP32.
__host__ __device__ __forceinline__ size_t ws_rows_floats(int B, int n, int HQ) {
    return (size_t)B * n * HQ * kHeadDim;
}
// After the rows: per (sequence, group) the admit's list, [n_adm, pend_fill, -, -, src[P], dest[P]]
// (ints): admitted candidate t (pending slot t if t < pend_fill, else block token t - pend_fill)
// goes to bank slot dest, in ascending t.
__host__ __device__ __forceinline__ size_t admit_list_ints(int P) { return 4 + 2 * (size_t)P; }
__device__ __forceinline__ int* admit_list(float* ws, int B, int n, int HQ, int P, int bg) {
    return reinterpret_cast<int*>(ws + 2 * ws_rows_floats(B, n, HQ)) + (size_t)bg * admit_list_ints(P);
}

// One work item: tiles 2p and 2p+1 of (sequence b, group g) in one phase (0 local, 1 bank).
struct Item {
    int b, g, bg, p, phase;
    int s, bank_fill, pend_fill, fill;
    int n_ring, n_blk, n_bank, nchunks;
};

// Items in (sequence, group)-major order, the local items of a group before its anchor items, so
// that groups complete one after another and their commits can start before the launch ends.
__device__ __forceinline__ Item make_item(const LayerView& S, int it, int npairs) {
    Item x;
    x.bg = it / (2 * npairs);
    const int r = it % (2 * npairs);
    x.phase = r / npairs;
    x.p = r % npairs;
    x.g = x.bg % S.G;
    x.b = x.bg / S.G;
    const int32_t* cnt = S.counters + x.bg * 4;
    x.s = max(cnt[0], 0);
    x.bank_fill = min(max(cnt[1], 0), S.A);
    x.pend_fill = min(max(cnt[2], 0), S.P);
    x.fill = min(x.s, S.R);
    x.n_ring = x.n_blk = x.n_bank = 0;
    if (x.phase == 0) {
        x.n_ring = (x.fill + kChunk - 1) / kChunk;
        x.n_blk = x.p + 1;                       // tiles 2p and 2p+1 reach block chunk p
    } else {
        x.n_bank = (x.bank_fill + kChunk - 1) / kChunk;
    }
    x.nchunks = x.n_ring + x.n_blk + x.n_bank;
    return x;
}

// The items of cluster c out of n, nc clusters: at step k, item k nc + (c + 2 k) mod nc, a
// permutation of each wave of nc items (so that a cluster's items do not all sit at the same
// offset of their groups, which would give some clusters only the longest local items); a step
// whose item lies past the last is skipped.
struct ItemSeq {
    int c, nc, n;
    __device__ __forceinline__ int at(int k) const { return k * nc + (c + 2 * k) % nc; }
    // the first step >= k that has an item, or -1
    __device__ __forceinline__ int next(int k) const {
        for (; (long long)k * nc < n; ++k)
            if (at(k) < n) return k;
        return -1;
    }
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

// TMA store of one box of the FP32 workspace from shared memory (bulk-group completion)
__device__ __forceinline__ void tma_store_5d(const CUtensorMap* map, const void* src, int c0, int c1, int c2, int c3,
                                             int c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.global.shared::cta.bulk_group [%0, {%1, %2, %3, %4, %5}], [%6];\n" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(ptx::smem_u32(src))
        : "memory");
}
// Wait until every bulk store this thread committed has completed (its writes performed).
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory"); }
// Ask for `bytes` (a multiple of 16) at a 16-byte aligned global address to be brought into L2.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(reinterpret_cast<uint64_t>(p)), "r"(bytes)
                 : "memory");
}

// Wait (bounded) until the high half of the group's ticket word reaches `need`; on timeout the
// status word gets RMA_STATUS_TIMEOUT and the caller goes on (its results are then undefined).
__device__ __forceinline__ void wait_rows(const LayerView& S, int bg, unsigned need) {
    if (threadIdx.x == 0) {
        const long long t0 = clock64();
        unsigned v;
        while (true) {
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(S.tickets + bg) : "memory");
            if ((v >> 16) >= need) break;
            if (clock64() - t0 > ptx::kWaitLimitCycles) {
                atomicOr(S.status, (unsigned)RMA_STATUS_TIMEOUT);
                break;
            }
            __nanosleep(256);
        }
    }
    __syncthreads();
    __threadfence();
}

__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// number of valid keys of chunk j of item x (rows past it may hold stale bytes)
__device__ __forceinline__ int chunk_valid(const Item& x, int j, int n) {
    if (j < x.n_ring) return x.fill - kChunk * j;
    if (j < x.n_ring + x.n_blk) return n - kChunk * (j - x.n_ring);
    return x.bank_fill - kChunk * (j - x.n_ring - x.n_blk);
}

// clear V rows [nvalid, 64) of this CTA's half in stage st so that P = 0 times V stays 0 (one warp)
__device__ __forceinline__ void clear_stale_v(uint8_t* smem, int nvalid, int st, int lane) {
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
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    prefill_attn_kernel(const __grid_constant__ Tmaps tm, const __grid_constant__ PrefillArgs a, int npairs,
                        int n_items) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const LayerView& S = a.s;
    const uint32_t rank = ptx::cluster_ctarank();
    const int pr = rank & 1;                     // 0: the pair's MMA-issuing CTA
    const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
    const ItemSeq seq{cluster, n_clusters, n_items};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = S.G, HQ = G * kQPerGroup, n = a.n_tok;
    const uint16_t pair_mask = 3u;
    const uint32_t leader = 0;

    // the commit launch may be scheduled now: it waits for this grid's completion before it reads
    grid_dep_launch();

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBar);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kNumBars + 1);
    float* xch = reinterpret_cast<float*>(smem + kSmemXch);

    if (tid == 0) {
        if (cluster == 0 && rank == 0) {
            // a corrupted state is clamped for indexing (make_item); flag it once
            for (int bg = 0; bg < S.B * G; ++bg) {
                const int32_t* c = S.counters + bg * 4;
                if (c[0] < 0 || c[1] < 0 || c[1] > S.A || c[2] < 0 || c[2] > S.P) {
                    atomicOr(S.status, (unsigned)RMA_STATUS_BAD_COUNTERS);
                    break;
                }
            }
        }
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
        ptx::mbar_init(&bars[kOFinal], 1);
        ptx::mbar_init(&bars[kODrained], 16);
        ptx::mbar_init(&bars[kDrain], 3);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kWarpQK) {
        ptx::tmem_alloc2(tmem_holder, kTmemCols);
        ptx::tmem_relinquish2();
    }
    ptx::tc_fence_before();
    ptx::cluster_sync();   // barriers of both CTAs initialised, tensor memory allocated
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == kWarpTma) {
        // ---------------- TMA producer: this CTA's half of every chunk of every item ----------------
        int jg = 0, issued = 0;
        bool ok = true;
        for (int k = seq.next(0); ok && k >= 0; k = seq.next(k + 1)) {
            const Item x = make_item(S, seq.at(k), npairs);
            if (seq.next(k + 1) >= 0) {
                // the next item's query rows of this CTA into L2 (one token's 4 heads per lane): its
                // softmax threads load them when that item starts
                const Item y = make_item(S, seq.at(seq.next(k + 1)), npairs);
                const int t = kTileTok * (2 * y.p + pr) + lane;
                if (t < n) prefetch_l2(a.q + ((size_t)(y.b * n + t) * HQ + y.g * kQPerGroup) * kHeadDim, kQPerGroup * kRowBytes);
            }
            for (int j = 0; j < x.nchunks; ++j, ++jg) {
                const int st = jg % kStages;
                if (jg >= kStages &&
                    !ptx::mbar_wait_warp(&bars[kEmpty + st], ((jg / kStages) - 1) & 1, abort_flag, S.status)) {
                    ok = false;
                    break;
                }
                issued = jg + 1;
                if (lane == 0) {
                    const CUtensorMap* mk;
                    const CUtensorMap* mv;
                    int yk, zk, yv, zv;
                    if (j < x.n_ring) {
                        mk = &tm.ring_k; mv = &tm.ring_v;
                        yk = kChunk * j + kHalfKeys * pr; zk = x.bg; yv = kChunk * j; zv = x.bg;
                    } else if (j < x.n_ring + x.n_blk) {
                        const int t0 = x.b * n + kChunk * (j - x.n_ring);
                        mk = &tm.k; mv = &tm.v;
                        yk = x.g; zk = t0 + kHalfKeys * pr; yv = x.g; zv = t0;
                    } else {
                        const int a0 = kChunk * (j - x.n_ring - x.n_blk);
                        mk = &tm.bank_k; mv = &tm.bank_v;
                        yk = a0 + kHalfKeys * pr; zk = x.bg; yv = a0; zv = x.bg;
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
        }
        // Drain, normal or abandoned: this CTA's loads of the last stages have landed (earlier
        // stages were consumed before their reuse), and every MMA of the pair has completed.
        for (int jj = max(0, issued - kStages); jj < issued; ++jj)
            ptx::mbar_wait_drain(&bars[kFull + jj % kStages], (jj / kStages) & 1, S.status);
        ptx::mbar_wait_drain(&bars[kDrain], 0, S.status);
        __syncwarp();
    } else if (warp == kWarpQK && pr == 1) {
        // ---------------- odd CTA: check its half landed, clear stale rows, tell the even CTA ----------------
        int jg = 0;
        bool ok = true;
        for (int k = seq.next(0); ok && k >= 0; k = seq.next(k + 1)) {
            const Item x = make_item(S, seq.at(k), npairs);
            for (int j = 0; j < x.nchunks; ++j, ++jg) {
                const int st = jg % kStages;
                if (!ptx::mbar_wait_warp(&bars[kFull + st], (jg / kStages) & 1, abort_flag, S.status)) {
                    ok = false;
                    break;
                }
                clear_stale_v(smem, chunk_valid(x, j, n), st, lane);
                if (lane == 0) ptx::mbar_arrive_at(&bars[kPeer + st], leader, rank);
                __syncwarp();
            }
        }
        // consume the last stages' empty phases (commits into this CTA's barriers)
        for (int jj = max(0, jg - kStages); ok && jj < jg; ++jj)
            if (!ptx::mbar_wait_warp(&bars[kEmpty + jj % kStages], (jj / kStages) & 1, abort_flag, S.status)) break;
    } else if (warp == kWarpQK || (warp == kWarpQK2 && pr == 0)) {
        // ---------------- even CTA: Q K^T issuers (warp 9: even global chunks, warp 11: odd) ----------------
        constexpr uint32_t idesc_qk = ptx::idesc_bf16_f32(2 * kRows, kChunk, false, false);
        const int mine = warp == kWarpQK ? 0 : 1;
        int jg = 0, kw = 0;
        bool ok = true;
        for (int k = seq.next(0); ok && k >= 0; k = seq.next(k + 1)) {
            const Item x = make_item(S, seq.at(k), npairs);
            if (x.nchunks == 0) continue;        // an empty bank: no Q K^T, and its Q is not loaded
            // Q of this item is in tensor memory (phase kw of kQReady).  Both issuers wait for every
            // phase, in order, even in an item where one of them has no chunk: a parity wait on a
            // barrier two phases ahead would pass at once.
            ok = ptx::mbar_wait_warp(&bars[kQReady], kw & 1, abort_flag, S.status);
            ++kw;
            ptx::tc_fence_after();
            for (int j = 0; ok && j < x.nchunks; ++j, ++jg) {
                if ((jg & 1) != mine) continue;
                if (jg >= 2) {
                    ok = ptx::mbar_wait_warp(&bars[kSFree + (jg & 1)], ((jg - 2) >> 1) & 1, abort_flag, S.status);
                    if (!ok) break;
                }
                const int st = jg % kStages;
                ok = ptx::mbar_wait_warp(&bars[kFull + st], (jg / kStages) & 1, abort_flag, S.status);
                if (!ok) break;
                ok = ptx::mbar_wait_warp(&bars[kPeer + st], (jg / kStages) & 1, abort_flag, S.status);
                if (!ok) break;
                clear_stale_v(smem, chunk_valid(x, j, n), st, lane);
                ptx::tc_fence_after();
                if (lane == 0) {
                    const uint32_t k_base = ptx::smem_u32(smem + st * kStageBytes);
                    const uint32_t d = tmem + ((jg & 1) ? kColS1 : kColS0);
                    for (int ks = 0; ks < kHeadDim / 16; ++ks) {
                        // 16 dims = 32 bytes inside the 128-byte swizzle atom of slab ks / 4
                        const uint64_t bd = ptx::smem_desc(k_base + (ks >> 2) * kSlabK + (ks & 3) * 32, 16, 1024,
                                                           ptx::kSwizzle128B);
                        ptx::mma_ts2(d, tmem + kColQ + 8 * ks, bd, idesc_qk, ks > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit2_mc(&bars[kSFull + (jg & 1)], pair_mask);
                }
                __syncwarp();
            }
        }
        if (lane == 0) ptx::mma_commit2_mc(&bars[kDrain], pair_mask);   // after this warp's last MMA
        __syncwarp();
    } else if (warp == kWarpPV && pr == 0) {
        // ---------------- even CTA: P V issuer ----------------
        constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(2 * kRows, kHeadDim, false, true);
        // kQReady, kOFinal and kODrained count only the items that have chunks (kw of them so far)
        int jg = 0, kw = 0;
        bool ok = true;
        for (int k = seq.next(0); ok && k >= 0; k = seq.next(k + 1)) {
            const Item x = make_item(S, seq.at(k), npairs);
            if (x.nchunks == 0) continue;
            // the previous item's O has been read by both CTAs before this item's first P V
            if (kw >= 1) ok = ptx::mbar_wait_warp(&bars[kODrained], (kw - 1) & 1, abort_flag, S.status);
            ++kw;
            for (int j = 0; ok && j < x.nchunks; ++j, ++jg) {
                const int st = jg % kStages;
                ok = ptx::mbar_wait_warp(&bars[kPFull + (jg & 1)], (jg >> 1) & 1, abort_flag, S.status);
                if (!ok) break;
                ptx::tc_fence_after();
                if (lane == 0) {
                    const uint32_t v_base = ptx::smem_u32(smem + st * kStageBytes + kKHalfBytes);
                    const uint32_t p_base = ptx::smem_u32(smem + kSmemP + (jg & 1) * kPBytes);
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
        }
        for (int jj = max(0, jg - kStages); ok && jj < jg; ++jj)
            if (!ptx::mbar_wait_warp(&bars[kEmpty + jj % kStages], (jj / kStages) & 1, abort_flag, S.status)) break;
        if (lane == 0) ptx::mma_commit2_mc(&bars[kDrain], pair_mask);   // after this warp's last MMA
        __syncwarp();
    } else if (warp < 8) {
        // ---------------- softmax: thread = (row, half); then the item's rows to the workspace ----------------
        const int row = 32 * (warp & 3) + lane;   // row of this CTA (lane of tensor memory)
        const int wg = (warp >> 2) & 1;           // which half of keys / columns
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        const float qs = a.qscale;
        // this thread's half of the Q row of item y -> tensor memory columns [384 + 64 wg, +64) as
        // packed BF16 (the caller makes sure every Q K^T that read the columns has completed)
        auto load_q = [&](const Item& y) {
            const int ty = kTileTok * (2 * y.p + pr) + (row >> 2);
            const uint4* qrow = reinterpret_cast<const uint4*>(
                                    a.q + ((size_t)(y.b * n + min(ty, n - 1)) * HQ + y.g * kQPerGroup + (row & 3)) *
                                              kHeadDim) +
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
        };
        int jg = 0, kw = 0;
        bool ok = true;
        if (seq.next(0) >= 0) {
            const Item y = make_item(S, seq.at(seq.next(0)), npairs);
            if (y.nchunks > 0) load_q(y);
        }
        for (int k = seq.next(0); k >= 0; k = seq.next(k + 1)) {
            const Item x = make_item(S, seq.at(k), npairs);
            const int T = 2 * x.p + pr;
            const int tok = kTileTok * T + (row >> 2);
            const int pq = x.s + tok;                  // query position
            const int w = (x.s - 1) % S.R;             // slot of position s - 1 (s >= 1)
            const int base_pos = x.s - 1 - w;
            // which of keys [32 h, 32 h + 32) of the item's chunk j this row sees, one bit per key
            auto vis32 = [&](int j, int h) -> uint32_t {
                if (j < x.n_ring) {
                    const int slot0 = kChunk * j + 32 * h;
                    if (slot0 >= x.fill) return 0u;
                    const bool all_valid = slot0 + 31 < x.fill;
                    const bool wraps = (slot0 <= w) && (w < slot0 + 31) && (x.fill == S.R);
                    const int first = wraps ? w + 1 : slot0;   // the oldest slot of the range
                    const int pk_min = base_pos + first - (first > w ? S.R : 0);
                    if (all_valid && pk_min >= pq - S.R) return 0xffffffffu;
                    uint32_t v = 0;
#pragma unroll 4
                    for (int i = 0; i < 32; ++i) {
                        const int slot = slot0 + i;
                        const int pk = base_pos + slot - (slot > w ? S.R : 0);
                        v |= (uint32_t)((slot < x.fill) && (pk >= pq - S.R)) << i;
                    }
                    return v;
                }
                if (j < x.n_ring + x.n_blk) {
                    const int t0 = kChunk * (j - x.n_ring) + 32 * h;
                    if (t0 > tok || t0 >= n) return 0u;
                    const int last = min(tok, n - 1) - t0;     // keys t0 .. t0 + last are visible
                    return last >= 31 ? 0xffffffffu : ((2u << last) - 1u);
                }
                const int a0 = kChunk * (j - x.n_ring - x.n_blk) + 32 * h;
                if (a0 >= x.bank_fill) return 0u;
                return (x.bank_fill - a0 >= 32) ? 0xffffffffu : ((1u << (x.bank_fill - a0)) - 1u);
            };
            // chunk loop: this group takes the item's chunks whose global index has parity wg
            const uint32_t scol = wg ? kColS1 : kColS0;
            float m_w = -CUDART_INF_F, l = 0.f;
            const int jbase = jg;
            for (int j = (wg - jbase) & 1; j < x.nchunks; j += 2) {
                const int jj = jbase + j;               // global chunk index
                const uint32_t vlo = vis32(j, 0), vhi = vis32(j, 1);
                if (ok) ok = ptx::mbar_wait_warp(&bars[kSFull + wg], (jj >> 1) & 1, abort_flag, S.status);
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
                if (j + 1 < x.nchunks) {
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
#undef SR
                l = l * fac_l + ((s4[0] + s4[1]) + (s4[2] + s4[3]));
                // O may be rescaled once P V of the previous chunk has completed; this group's P buffer
                // is free once P V of global chunk jj - 2 has (possibly in the previous item: done then)
                const bool rescale_warp = __any_sync(0xffffffffu, resc);
                if (ok && rescale_warp)
                    ok = ptx::mbar_wait_warp(&bars[kEmpty + (jj - 1) % kStages], ((jj - 1) / kStages) & 1,
                                             abort_flag, S.status);
                if (ok && jj >= 2)
                    ok = ptx::mbar_wait_warp(&bars[kEmpty + (jj - 2) % kStages], ((jj - 2) / kStages) & 1,
                                             abort_flag, S.status);
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
            jg = jbase + x.nchunks;
            // the row sum over both groups, on the later reference (references only grow)
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
            ptx::named_bar_sync(1, kSoftmaxThreads);   // both groups have read the exchange of this item
            const bool have_o =
                ok && x.nchunks > 0 && ptx::mbar_wait_warp(&bars[kOFinal], kw & 1, abort_flag, S.status);
            if (have_o) ptx::tc_fence_after();
            // The next item's Q, so that its first Q K^T run during this drain: every Q K^T of this
            // item has completed (O final), or it had none.
            if (seq.next(k + 1) >= 0) {
                const Item y = make_item(S, seq.at(seq.next(k + 1)), npairs);
                if (y.nchunks > 0) load_q(y);
            }
            const float inv = (have_o && l > 0.f) ? 1.f / l : 0.f;
            // This group's half of the rows, normalised (zeros for an empty bank), to the workspace in
            // four steps of 32 columns: each thread writes its row into the group's P buffer (free:
            // every P V of the item has completed) in the 128-byte swizzled layout, then one thread
            // stores the [32 tokens][4 heads][32 dims] box with TMA (rows past the block are clipped);
            // the next 32 columns are read from tensor memory while the box leaves the buffer.
            // each warp stores its own 32 rows (8 tokens x 4 heads) from its 4 KB of the group's P buffer
            uint8_t* stg = smem + kSmemP + wg * kPBytes + (warp & 3) * 4096;
            uint8_t* srow = stg + lane * 128;
            uint32_t o[32];
            auto read_o = [&](int c) {
                if (have_o) {
                    ptx::tmem_ld32(lane_addr + kColO + 128 * wg + 32 * c, o);
                    ptx::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0u;
                }
            };
            read_o(0);
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                if (c > 0) {
                    if (lane == 0) ptx::bulk_wait_read_all();   // the previous box has left the buffer
                    __syncwarp();
                }
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    *reinterpret_cast<float4*>(srow + ((k ^ (lane & 7)) << 4)) =
                        make_float4(__uint_as_float(o[4 * k]) * inv, __uint_as_float(o[4 * k + 1]) * inv,
                                    __uint_as_float(o[4 * k + 2]) * inv, __uint_as_float(o[4 * k + 3]) * inv);
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && kTileTok * T + 8 * (warp & 3) < n) {   // rows past the block are not stored
                    tma_store_5d(&tm.ws, stg, 128 * wg + 32 * c, x.g * kQPerGroup, kTileTok * T + 8 * (warp & 3),
                                 x.b, x.phase);
                    ptx::bulk_commit();
                }
                if (c < 3) read_o(c + 1);
            }
            if (lane == 0) {
                // every box of this warp is written (and its rows of the P buffer are free): count
                // them as done for the commit of (sequence, group), which waits for all 16 warps of
                // the pair per item (high half of the group's ticket word)
                bulk_wait_all();
                asm volatile("fence.proxy.async.global;\n" ::: "memory");
                __threadfence();
                atomicAdd(S.tickets + x.bg, 1u << 16);
            }
            __syncwarp();
            if (x.nchunks > 0) {
                // O has been read by this warp: the pair's next item with chunks may overwrite it
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive_at(&bars[kODrained], leader, rank);
                ++kw;
            }
        }
    }
    // every CTA of the cluster is done with its roles, and (the producer's drain) no load into it
    // and no tensor-core operation of the pair is in flight; the softmax groups' workspace stores
    // have completed
    if (warp < 8 && (warp & 3) == 0 && lane == 0) bulk_wait_all();
    __syncwarp();
    ptx::tc_fence_before();
    ptx::cluster_sync();
    if (warp == kWarpQK) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc2(tmem, kTmemCols);
    }
}

// ---- the commit: gate and combine, ring write, pending append, forced admit ----
// (three CTAs per SM)
__global__ void __launch_bounds__(kCommitThreads, 4) prefill_commit_kernel(const __grid_constant__ PrefillArgs a) {
    extern __shared__ __align__(16) uint8_t csmem[];
    const LayerView& S = a.s;
    // CTAs [0, B G) run the admits (first, so that they are scheduled first), then kCommitSlices
    // slice CTAs per (sequence, group)
    const int G = S.G, HQ = G * kQPerGroup, n = a.n_tok;
    const int n_bg = S.B * G;
    const int ci = blockIdx.x < n_bg ? (int)blockIdx.x : (int)blockIdx.x - n_bg;
    const int bg = blockIdx.x < n_bg ? ci : ci / kCommitSlices;
    const int slice = blockIdx.x < n_bg ? kCommitSlices : ci % kCommitSlices;
    const int g = bg % G, b = bg / G;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int kP = kRowBytes / 16;           // 16-byte pieces per row
    __shared__ int s_last;

    // The counters as they were before this block; none is written before every CTA of the
    // group has arrived (the last one writes them all).
    const int32_t* cnt = S.counters + bg * 4;
    const int s = max(cnt[0], 0);
    const int bank_fill = min(max(cnt[1], 0), S.A);
    const int pend_fill = min(max(cnt[2], 0), S.P);
    const bool fits = pend_fill + n <= S.P;
    const int np = fits ? pend_fill + n : pend_fill;
    if (slice < kCommitSlices) {
        const int per = (n + kCommitSlices - 1) / kCommitSlices;
        const int t0 = min(n, slice * per), t1 = min(n, t0 + per);
        // The slice's candidates to pending slots pend_fill + i: no kernel of this call reads them
        // (the admit takes the block's candidates from the inputs), so this precedes the wait.
        if (fits) {
            copy_pieces<kCommitThreads, 4>((t1 - t0) * 2 * kP, [&](int e, const uint4*& from_p, uint4*& to_p) {
                const int i = t0 + e / (2 * kP), c = e % (2 * kP);
                const size_t src = ((size_t)(b * n + i) * G + g) * kHeadDim;
                const size_t pd = ((size_t)bg * S.P + pend_fill + i) * kHeadDim;
                if (c < kP) {
                    from_p = reinterpret_cast<const uint4*>(a.cand_k + src) + c;
                    to_p = reinterpret_cast<uint4*>(S.pend_k + pd) + c;
                } else {
                    from_p = reinterpret_cast<const uint4*>(a.cand_v + src) + (c - kP);
                    to_p = reinterpret_cast<uint4*>(S.pend_v + pd) + (c - kP);
                }
            });
            for (int i = t0 + tid; i < t1; i += kCommitThreads)
                S.pend_score[(size_t)bg * S.P + pend_fill + i] = a.cand_score[(size_t)(b * n + i) * G + g];
        }
        // The gate of the slice's rows, tanh(q . w_g + b_g) with the unscaled query: the group's 4
        // w_g rows staged in shared memory, then each warp takes rows warp, warp + 8, ... with
        // every query load issued before the first dot product (a lane holds 8 dims of a row).
        float* gate = reinterpret_cast<float*>(csmem);                     // [rows]
        float* wsh = reinterpret_cast<float*>(csmem) + 4 * kCommitMaxTok;    // [4][256]
        const int rows = (t1 - t0) * kQPerGroup;
        reinterpret_cast<float4*>(wsh)[tid] =
            __ldg(reinterpret_cast<const float4*>(a.w_g + (size_t)g * kQPerGroup * kHeadDim) + tid);
        __syncthreads();
        {
            constexpr int kRowsPerWarp = 4 * kCommitMaxTok / (kCommitThreads / 32);
            uint4 qv[kRowsPerWarp];
#pragma unroll
            for (int u = 0; u < kRowsPerWarp; ++u) {
                const int r = warp + 8 * u;
                const int t = t0 + min(r, rows - 1) / kQPerGroup, head = g * kQPerGroup + min(r, rows - 1) % kQPerGroup;
                qv[u] = rows > 0 ? __ldg(reinterpret_cast<const uint4*>(a.q + ((size_t)(b * n + t) * HQ + head) * kHeadDim) + lane)
                                 : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kRowsPerWarp; ++u) {
                const int r = warp + 8 * u;
                const int h = r % kQPerGroup;
                const float4 w0 = reinterpret_cast<const float4*>(wsh + h * kHeadDim)[2 * lane];
                const float4 w1 = reinterpret_cast<const float4*>(wsh + h * kHeadDim)[2 * lane + 1];
                const uint4 q4 = qv[u];
                float d = __uint_as_float(q4.x << 16) * w0.x + __uint_as_float(q4.x & 0xffff0000u) * w0.y +
                          __uint_as_float(q4.y << 16) * w0.z + __uint_as_float(q4.y & 0xffff0000u) * w0.w +
                          __uint_as_float(q4.z << 16) * w1.x + __uint_as_float(q4.z & 0xffff0000u) * w1.y +
                          __uint_as_float(q4.w << 16) * w1.z + __uint_as_float(q4.w & 0xffff0000u) * w1.w;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
                if (lane == 0 && r < rows) gate[r] = tanhf(d + a.b_g[g * kQPerGroup + h]);
            }
        }
        __syncthreads();
        // every row of this (sequence, group) is in the workspace after this: 16 arrivals (2 CTAs x
        // 8 softmax warps) per item, 2 npairs items
        wait_rows(S, bg, 32 * ((n + 2 * kTileTok - 1) / (2 * kTileTok)));
        // out = local + gate * anchor: thread (head r0, dims 4 d4 .. 4 d4 + 3) over the slice's
        // tokens, kCommitUnroll tokens' loads in flight before it combines and stores them
        {
            const int r0 = tid >> 6, d4 = tid & 63;
            const size_t row0 = (size_t)(b * n + t0) * HQ + g * kQPerGroup + r0;
            const size_t step = (size_t)HQ * (kHeadDim / 4);   // float4 (and 4-value output) pieces per token
            const float4* lb = reinterpret_cast<const float4*>(a.ws + row0 * kHeadDim) + d4;
            const float4* ab = reinterpret_cast<const float4*>(a.ws + ws_rows_floats(S.B, n, HQ) + row0 * kHeadDim) + d4;
            uint2* ob = reinterpret_cast<uint2*>(a.out + row0 * kHeadDim) + d4;
            const int ntok = t1 - t0;
            for (int k0 = 0; k0 < ntok; k0 += kCommitUnroll) {
                float4 lc[kCommitUnroll], an[kCommitUnroll];
#pragma unroll
                for (int u = 0; u < kCommitUnroll; ++u) {
                    const int k = min(k0 + u, ntok - 1);
                    lc[u] = __ldcg(lb + k * step);
                    an[u] = __ldcg(ab + k * step);
                }
#pragma unroll
                for (int u = 0; u < kCommitUnroll; ++u) {
                    if (k0 + u < ntok) {
                        const float gt = gate[(k0 + u) * kQPerGroup + r0];
                        uint2 o;
                        o.x = pack_bf16(lc[u].x + gt * an[u].x, lc[u].y + gt * an[u].y);
                        o.y = pack_bf16(lc[u].z + gt * an[u].z, lc[u].w + gt * an[u].w);
                        ob[(k0 + u) * step] = o;
                    }
                }
            }
        }
        // the block's K / V into ring slots (s + i) mod R (every read of the block is done)
        copy_pieces<kCommitThreads, 4>((t1 - t0) * 2 * kP, [&](int e, const uint4*& from_p, uint4*& to_p) {
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
    } else {
        // The forced admit over the committed bank and the pending buffer, the block's candidates
        // included when they fit.  The competition reads scores only, and neither the attention
        // launch nor the slices touch the bank's scores or the scores it reads, so this CTA does not
        // wait: it writes the kept candidates' scores and leaves the list of (source, bank slot)
        // pairs in the workspace for the copy launch, which moves the rows once the attention
        // launch has read the bank.
        const float* pscore = S.pend_score + (size_t)bg * S.P;
        auto score_of = [&](int t) {
            return t < pend_fill ? pscore[t] : a.cand_score[(size_t)(b * n + t - pend_fill) * G + g];
        };
        int n_adm = 0;
        if (np > 0) n_adm = admit_select<kCommitThreads>(S, bg, bank_fill, np, csmem, score_of);
        int* list = admit_list(a.ws, S.B, n, HQ, S.P, bg);
        if (tid == 0) {
            list[0] = n_adm;
            list[1] = pend_fill;
        }
        if (n_adm > 0) {
            const int* src = admit_src(csmem, S.A, S.P);
            const int* dest = admit_dest(csmem, S.A, S.P);
            for (int j = tid; j < n_adm; j += kCommitThreads) {
                list[4 + j] = src[j];
                list[4 + S.P + j] = dest[j];
                S.bank_score[(size_t)bg * S.A + dest[j]] = score_of(src[j]);
            }
        }
        if (tid == 0 && !fits) atomicOr(S.status, (unsigned)RMA_STATUS_PREFILL_PENDING_OVERFLOW);
    }
    // The last CTA of (b, g) to finish writes the counters (every CTA of the group read them
    // before it arrived): pos advances by the block, the admit kept min(A, bank + candidates)
    // records, and pending is empty.
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned old = atomicAdd(S.tickets + bg, 1u);
        s_last = (old & 0xffffu) == (unsigned)kCommitSlices;
    }
    __syncthreads();
    if (s_last && tid == 0) {
        __threadfence();
        int32_t* c = S.counters + bg * 4;
        c[0] = s + n;
        c[1] = min(S.A, bank_fill + np);
        c[2] = 0;
        S.tickets[bg] = 0u;
    }
}

// ---- the admitted rows into the bank, once the attention launch has read it ----
// kCopyParts CTAs per (sequence, group), each moving a share of the admit's list.
constexpr int kCopyParts = 8;
constexpr int kCopyThreads = 256;
__global__ void __launch_bounds__(kCopyThreads) prefill_admit_copy_kernel(const __grid_constant__ PrefillArgs a) {
    const LayerView& S = a.s;
    const int G = S.G, HQ = G * kQPerGroup, n = a.n_tok;
    const int bg = blockIdx.x / kCopyParts, part = blockIdx.x % kCopyParts;
    const int g = bg % G, b = bg / G;
    constexpr int kP = kRowBytes / 16;
    // the commit launch (the lists) and, before it, the attention launch (every read of the bank)
    // have completed
    grid_dep_wait();
    const int* list = admit_list(a.ws, S.B, n, HQ, S.P, bg);
    const int n_adm = min(max(list[0], 0), S.P), pend_fill = list[1];
    const int per = (n_adm + kCopyParts - 1) / kCopyParts;
    const int j0 = min(n_adm, part * per), j1 = min(n_adm, j0 + per);
    const int* src = list + 4;
    const int* dest = list + 4 + S.P;
    copy_pieces<kCopyThreads, 8>((j1 - j0) * 2 * kP, [&](int e, const uint4*& from_p, uint4*& to_p) {
        const int j = j0 + e / (2 * kP), c = e % (2 * kP);
        const bool kpart = c < kP;
        const int piece = kpart ? c : c - kP;
        const int t = src[j];
        const uint16_t* from_row =
            t < pend_fill ? (kpart ? S.pend_k : S.pend_v) + ((size_t)bg * S.P + t) * kHeadDim
                          : (kpart ? a.cand_k : a.cand_v) + ((size_t)(b * n + t - pend_fill) * G + g) * kHeadDim;
        from_p = reinterpret_cast<const uint4*>(from_row) + piece;
        to_p = reinterpret_cast<uint4*>((kpart ? S.bank_k : S.bank_v) + ((size_t)bg * S.A + dest[j]) * kHeadDim) + piece;
    });
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

// The FP32 workspace [phase 2][b B][t n][head HQ][256] for TMA stores: boxes of 32 dims x 4 heads
// x 8 tokens (one softmax warp's 32 rows), 128-byte swizzle (the rows' 16-byte pieces permuted by
// row within 8-row groups).
bool make_ws_map(CUtensorMap* m, void* ws, int HQ, int n, int B) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const uint64_t row = (uint64_t)kHeadDim * 4;
    const cuuint64_t dims[5] = {(cuuint64_t)kHeadDim, (cuuint64_t)HQ, (cuuint64_t)n, (cuuint64_t)B, 2};
    const cuuint64_t strides[4] = {row, row * HQ, row * HQ * n, row * HQ * n * B};
    const cuuint32_t box[5] = {32, (cuuint32_t)kQPerGroup, (cuuint32_t)(kTileTok / 4), 1, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 5, ws, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Clusters of 2 attention CTAs that can be resident at once on the current device (cached per
// device; half the SM count if the occupancy query fails).
int resident_clusters() {
    constexpr int kTracked = 64;
    static std::atomic<int> cached[kTracked] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    if (dev >= 0 && dev < kTracked) {
        const int c = cached[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    if (cudaOccupancyMaxActiveClusters(&n, prefill_attn_kernel, &cfg) != cudaSuccess || n < 1) {
        (void)cudaGetLastError();
        int sms = 0;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        n = sms / 2 > 0 ? sms / 2 : 1;
    }
    if (dev >= 0 && dev < kTracked) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

}  // namespace

size_t prefill_workspace_bytes(const rma_config& cfg, int n_tok) {
    // normalised local and anchor rows (FP32) of every (token, head) of the block
    const int HQ = cfg.n_groups * cfg.q_per_group;
    const size_t bytes = 2 * ws_rows_floats(cfg.batch, n_tok, HQ) * 4 +
                         (size_t)cfg.batch * cfg.n_groups * admit_list_ints(cfg.pend_slots) * 4;
    return (bytes + 255) / 256 * 256;
}

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream) {
    const LayerView& s = a.s;
    const int B = s.B, G = s.G, n = a.n_tok;
    if (n < 1 || n > kMaxPrefillTokens || n > s.R) return cudaErrorNotSupported;
    const int npairs = (n + 2 * kTileTok - 1) / (2 * kTileTok);
    const long long n_items = 2LL * B * G * npairs;
    if (n_items > (1 << 30)) return cudaErrorNotSupported;
    Tmaps tm;
    const uint64_t row = (uint64_t)kHeadDim * 2;
    bool ok = make_map(&tm.k, a.k, G, (uint64_t)B * n, row, row * G, 1, kHalfKeys) &&
              make_map(&tm.v, a.v, G, (uint64_t)B * n, row, row * G, 1, kChunk) &&
              make_map(&tm.ring_k, s.ring_k, s.R, (uint64_t)B * G, row, row * s.R, kHalfKeys, 1) &&
              make_map(&tm.ring_v, s.ring_v, s.R, (uint64_t)B * G, row, row * s.R, kChunk, 1) &&
              make_map(&tm.bank_k, s.bank_k, s.A, (uint64_t)B * G, row, row * s.A, kHalfKeys, 1) &&
              make_map(&tm.bank_v, s.bank_v, s.A, (uint64_t)B * G, row, row * s.A, kChunk, 1) &&
              make_ws_map(&tm.ws, a.ws, G * kQPerGroup, n, B);
    if (!ok) return cudaErrorInvalidValue;
    static SmemLimit limit(reinterpret_cast<const void*>(prefill_attn_kernel));
    cudaError_t e = limit.ensure(kSmemBytes);
    if (e != cudaSuccess) return e;
    // one cluster of 2 per co-resident slot, each looping over its items
    // As many clusters as keep the most items per cluster at its minimum: the SMs left over run the
    // commit of the groups that are done while the last items run.
    const long long per_cluster = (n_items + resident_clusters() - 1) / resident_clusters();
    const int n_clusters = (int)((n_items + per_cluster - 1) / per_cluster);
    prefill_attn_kernel<<<dim3(2 * n_clusters, 1, 1), kThreads, kSmemBytes, stream>>>(tm, a, npairs, (int)n_items);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // the commit, launched so that its CTAs may be scheduled while the attention launch finishes
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((kCommitSlices + 1) * B * G), 1, 1);
    cfg.blockDim = dim3(kCommitThreads, 1, 1);
    // the admit's scratch, or the slices' gate and w_g rows if a small state makes that larger
    cfg.dynamicSmemBytes = std::max(admit_scratch_bytes(s.A, s.P), (size_t)(4 * kCommitMaxTok + 4 * kHeadDim) * 4);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    static SmemLimit climit(reinterpret_cast<const void*>(prefill_commit_kernel));
    e = climit.ensure(cfg.dynamicSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, prefill_commit_kernel, a);
    if (e != cudaSuccess) return e;
    // the copy of the admitted rows, launched the same way after the commit
    cudaLaunchConfig_t ccfg = cfg;
    ccfg.gridDim = dim3((unsigned)(kCopyParts * B * G), 1, 1);
    ccfg.blockDim = dim3(kCopyThreads, 1, 1);
    ccfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&ccfg, prefill_admit_copy_kernel, a);
}

}  // namespace rma
