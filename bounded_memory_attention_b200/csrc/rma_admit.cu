// rma_admit: committed anchors and pending candidates compete; the top
// min(A, bank_fill + pend_fill) are kept per (sequence, layer, KV group).
//
// ("EdgeRock-4B holds KV cache at 72 MiB ..." (tpsreport.news), "How it
// works": after every 256 candidates they are compared with the existing
// anchors and the top 1,024 are kept, independently in each of four KV
// groups; ai-primer story, operations list, item 2 "Admit"; "EdgeRock" model
// card: retained records remain separate and unchanged.)
//
// One CTA per (b, g).  The order (higher score, then committed before
// candidate, then lower slot) is encoded in one 64-bit key per record:
//   bits 63..32  the FP32 score mapped to an unsigned integer that orders
//                like the float (sign bit flipped for >= 0, all bits flipped
//                for < 0; -0.0 first canonicalised to +0.0; NaN -> 0, below
//                the image of -inf)
//   bit  31      1 for a committed anchor, 0 for a candidate
//   bits 30..0   0x7FFFFFFF - slot
// Keys are unique, so "kept" = the k largest keys, found with a bitonic sort
// in shared memory.  Compaction: vacated bank slots (evicted anchors and
// empty slots) are listed in ascending order and the admitted candidates in
// ascending pending slot; the j-th candidate is copied to the j-th vacated
// slot.  Byte copies only: bit-exact by construction.
#include <math_constants.h>

#include "rma_internal.cuh"

namespace rma {
namespace {

constexpr int kThreads = 512;
constexpr int kWarpsA = kThreads / 32;

__device__ __forceinline__ uint32_t order_bits(float s) {
    if (isnan(s)) return 0u;
    if (s == 0.0f) s = 0.0f;   // -0.0 -> +0.0
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t make_key(float score, bool committed, int slot) {
    const uint32_t lo = (committed ? 0x80000000u : 0u) | (0x7FFFFFFFu - (uint32_t)slot);
    return ((uint64_t)order_bits(score) << 32) | lo;
}

// Exclusive prefix sum of one int per thread over the whole block; *total
// (shared memory) receives the sum over all threads.
__device__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int t = lane < kWarpsA ? warp_tot[lane] : 0;
        int wi = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += u;
        }
        if (lane < kWarpsA) warp_tot[lane] = wi - t;
        if (lane == kWarpsA - 1) *total = wi;
    }
    __syncthreads();
    const int r = incl - v + warp_tot[warp];
    __syncthreads();   // warp_tot is reused by the next scan
    return r;
}

// prefill_n > 0: first account for a prefill block of prefill_n tokens whose
// K/V and candidates were already written (pos += n; pend_fill += n if the
// candidates fit, else RMA_STATUS_PREFILL_PENDING_OVERFLOW).
__global__ void __launch_bounds__(kThreads) admit_kernel(const __grid_constant__ LayerView s, int force,
                                                         int prefill_n) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int g = blockIdx.x, b = blockIdx.y;
    const int bg = b * s.G + g;
    const int tid = threadIdx.x;
    int32_t* cnt = s.counters + bg * 4;
    int nb = cnt[1], np = cnt[2];
    if (nb < 0 || nb > s.A || np < 0 || np > s.P) {
        // a corrupted state: never index outside the buffers
        if (threadIdx.x == 0) atomicOr(s.status, (unsigned)RMA_STATUS_BAD_COUNTERS);
        nb = min(max(nb, 0), s.A);
        np = min(max(np, 0), s.P);
    }
    if (prefill_n > 0) {
        const bool fits = np + prefill_n <= s.P;
        __syncthreads();   // every thread has read the counters
        if (tid == 0) {
            cnt[0] = max(cnt[0], 0) + prefill_n;
            if (fits) cnt[2] = np + prefill_n;
            else atomicOr(s.status, (unsigned)RMA_STATUS_PREFILL_PENDING_OVERFLOW);
        }
        if (fits) np += prefill_n;
    }
    if (!(np == s.P || (force && np > 0))) return;

    const int A = s.A, P = s.P;
    const int n = nb + np;
    const int k = min(A, n);
    int n2 = 2;
    while (n2 < n) n2 <<= 1;

    // shared memory: keys[n2max] | flags_bank[A] | flags_pend[P] | dest[P] | src[P] | warp_tot[32]
    uint64_t* keys = reinterpret_cast<uint64_t*>(smem);
    int n2max = 2;
    while (n2max < A + P) n2max <<= 1;
    uint8_t* kept_bank = reinterpret_cast<uint8_t*>(keys + n2max);
    uint8_t* kept_pend = kept_bank + A;
    int* dest = reinterpret_cast<int*>(smem + (((size_t)n2max * 8 + A + P + 15) & ~(size_t)15));
    int* src = dest + P;
    int* warp_tot = src + P;
    __shared__ int s_nan;

    const float* bscore = s.bank_score + (size_t)bg * A;
    const float* pscore = s.pend_score + (size_t)bg * P;
    if (tid == 0) s_nan = 0;
    __syncthreads();
    bool nan_seen = false;
    for (int i = tid; i < n2; i += kThreads) {
        uint64_t key = 0;
        if (i < nb) {
            const float sc = bscore[i];
            nan_seen |= isnan(sc);
            key = make_key(sc, true, i);
        } else if (i < n) {
            const float sc = pscore[i - nb];
            nan_seen |= isnan(sc);
            key = make_key(sc, false, i - nb);
        }
        keys[i] = key;
    }
    for (int i = tid; i < A + P; i += kThreads) kept_bank[i] = 0;   // kept_pend follows kept_bank
    if (nan_seen) s_nan = 1;
    __syncthreads();
    if (tid == 0 && s_nan) atomicOr(s.status, (unsigned)RMA_STATUS_NAN_SCORE);

    // bitonic sort, descending
    for (int size = 2; size <= n2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = tid; i < (n2 >> 1); i += kThreads) {
                const int lo = ((i & ~(stride - 1)) << 1) | (i & (stride - 1));
                const int hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const uint64_t x = keys[lo], y = keys[hi];
                if ((x < y) == desc) {
                    keys[lo] = y;
                    keys[hi] = x;
                }
            }
            __syncthreads();
        }
    }

    // mark the kept records
    for (int i = tid; i < k; i += kThreads) {
        const uint32_t lo = (uint32_t)keys[i];
        const int slot = (int)(0x7FFFFFFFu - (lo & 0x7FFFFFFFu));
        if (lo & 0x80000000u) kept_bank[slot] = 1;
        else kept_pend[slot] = 1;
    }
    __syncthreads();

    // admitted candidates in ascending pending slot -> src[j]
    __shared__ int s_total;
    int n_adm;
    {
        const int seg = (P + kThreads - 1) / kThreads;
        const int t0 = tid * seg, t1 = min(P, t0 + seg);
        int c = 0;
        for (int t = t0; t < t1; ++t) c += (t < np) && kept_pend[t];
        int idx = block_exclusive_scan(c, warp_tot, &s_total);
        for (int t = t0; t < t1; ++t)
            if ((t < np) && kept_pend[t]) src[idx++] = t;
        n_adm = s_total;
    }
    // vacated bank slots (evicted anchors and empty slots), ascending -> dest[j]; only the first
    // n_adm (<= P) are needed
    {
        const int seg = (A + kThreads - 1) / kThreads;
        const int s0 = tid * seg, s1 = min(A, s0 + seg);
        int c = 0;
        for (int sl = s0; sl < s1; ++sl) c += (sl >= nb) || !kept_bank[sl];
        int idx = block_exclusive_scan(c, warp_tot, &s_total);
        for (int sl = s0; sl < s1; ++sl) {
            if ((sl >= nb) || !kept_bank[sl]) {
                if (idx < n_adm) dest[idx] = sl;
                ++idx;
            }
        }
    }
    __syncthreads();

    // copy admitted candidates: K and V rows (16-byte chunks) and scores
    const uint4* pk = reinterpret_cast<const uint4*>(s.pend_k + (size_t)bg * P * kHeadDim);
    const uint4* pv = reinterpret_cast<const uint4*>(s.pend_v + (size_t)bg * P * kHeadDim);
    uint4* bk = reinterpret_cast<uint4*>(s.bank_k + (size_t)bg * A * kHeadDim);
    uint4* bv = reinterpret_cast<uint4*>(s.bank_v + (size_t)bg * A * kHeadDim);
    constexpr int kChunks = kRowBytes / 16;   // 32 per row
    for (int e = tid; e < n_adm * 2 * kChunks; e += kThreads) {
        const int j = e / (2 * kChunks);
        const int c = e % (2 * kChunks);
        const int from = src[j], to = dest[j];
        if (c < kChunks) bk[(size_t)to * kChunks + c] = pk[(size_t)from * kChunks + c];
        else bv[(size_t)to * kChunks + (c - kChunks)] = pv[(size_t)from * kChunks + (c - kChunks)];
    }
    for (int j = tid; j < n_adm; j += kThreads)
        s.bank_score[(size_t)bg * A + dest[j]] = pscore[src[j]];
    if (tid == 0) {
        cnt[1] = k;
        cnt[2] = 0;
    }
}

}  // namespace

size_t admit_smem_bytes(int A, int P) {
    int n2max = 2;
    while (n2max < A + P) n2max <<= 1;
    size_t off = ((size_t)n2max * 8 + A + P + 15) & ~(size_t)15;
    return off + (size_t)(2 * P + 32) * 4;
}

cudaError_t launch_admit(const LayerView& s, int force, int prefill_n, cudaStream_t stream) {
    const size_t smem = admit_smem_bytes(s.A, s.P);
    static size_t configured = 0;
    if (smem > 48 * 1024 && smem > configured) {
        cudaError_t e = cudaFuncSetAttribute(admit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured = smem;
    }
    dim3 grid(s.G, s.B);
    admit_kernel<<<grid, kThreads, smem, stream>>>(s, force, prefill_n);
    return cudaGetLastError();
}

}  // namespace rma
