// The admit of one (sequence, layer, KV group), as a device function that a
// whole CTA calls: the standalone admit kernel, the decode kernel's merge tail
// and the prefill kernel's last CTA all use it.
//
// ("EdgeRock-4B holds KV cache at 72 MiB ..." (tpsreport.news), "How it
// works": the candidates are compared with the existing anchors and the top
// 1,024 are kept, per KV group; ai-primer story, operations list, item 2;
// "EdgeRock" model card: retained records remain separate and unchanged.)
//
// Order: higher score, then committed before candidate, then lower slot,
// encoded in one unique 64-bit key per record:
//   bits 63..32  the FP32 score mapped to an unsigned integer that orders like
//                the float (sign bit flipped for >= 0, all bits flipped for
//                < 0; -0.0 first made +0.0; NaN -> 0, below the image of -inf)
//   bit  31      1 for a committed anchor, 0 for a candidate
//   bits 30..0   0x7FFFFFFF - slot
// Selection: when n = bank_fill + pend_fill exceeds A, the k-th largest key
// (k = A) is found by a most-significant-digit-first radix select over 8-bit
// digits (a 256-bin shared-memory histogram per digit); kept = keys >= it.
// Compaction: the vacated bank slots (evicted anchors, then empty slots) in
// ascending order receive the admitted candidates in ascending pending slot.
// Byte copies only, so the result is bit-exact by construction.
#pragma once

#include "rma_internal.cuh"

namespace rma {

__device__ __forceinline__ uint32_t admit_order_bits(float s) {
    if (isnan(s)) return 0u;
    if (s == 0.0f) s = 0.0f;   // -0.0 -> +0.0
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t admit_key(float score, bool committed, int slot) {
    const uint32_t lo = (committed ? 0x80000000u : 0u) | (0x7FFFFFFFu - (uint32_t)slot);
    return ((uint64_t)admit_order_bits(score) << 32) | lo;
}

// Scratch (shared memory) the admit of one group needs.
__host__ __device__ constexpr size_t admit_scratch_bytes(int A, int P) {
    return ((size_t)(A + P) * 8 + (size_t)(A + P) + 15) / 16 * 16 + (size_t)(2 * P + 256 + 64) * 4;
}

// Copy `total` 16-byte pieces with the whole CTA (NT threads): piece e goes from src(e) to
// dst(e), given by where(e, src, dst).  Each thread issues U loads before the first of its
// stores so that U pieces per thread are in flight at once.  The loads go through L2 only
// (.cg): the source may have been written earlier in the same launch by another CTA.
template <int NT, int U, class Where>
__device__ __forceinline__ void copy_pieces(int total, Where where) {
    for (int e0 = threadIdx.x; e0 < total; e0 += NT * U) {
        uint4 v[U];
        uint4* d[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = e0 + u * NT;
            d[u] = nullptr;
            if (e < total) {
                const uint4* src;
                where(e, src, d[u]);
                v[u] = __ldcg(src);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (d[u]) *d[u] = v[u];
    }
}

// Exclusive prefix sum of one int per thread over NT threads; *total gets the sum.
template <int NT>
__device__ __forceinline__ int admit_block_scan(int v, int* warp_tot, int* total) {
    constexpr int kW = NT / 32;
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
        const int t = lane < kW ? warp_tot[lane] : 0;
        int wi = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += u;
        }
        if (lane < kW) warp_tot[lane] = wi - t;
        if (lane == kW - 1) *total = wi;
    }
    __syncthreads();
    const int r = incl - v + warp_tot[warp];
    __syncthreads();
    return r;
}

// The K and V rows of the admitted candidates: pending slot src[j] -> bank slot dest[j], for
// j < n_adm, with rows of kChunks 16-byte pieces (32 for BF16, 16 for FP8 codes).
template <int NT, int U, int kChunks>
__device__ __forceinline__ void admit_copy_rows(const LayerView& s, int bg, int n_adm, const int* src,
                                                const int* dest) {
    constexpr int kRow = kChunks * 16;
    const uint8_t* pk = reinterpret_cast<const uint8_t*>(s.pend_k) + (size_t)bg * s.P * kRow;
    const uint8_t* pv = reinterpret_cast<const uint8_t*>(s.pend_v) + (size_t)bg * s.P * kRow;
    uint8_t* bk = reinterpret_cast<uint8_t*>(s.bank_k) + (size_t)bg * s.A * kRow;
    uint8_t* bv = reinterpret_cast<uint8_t*>(s.bank_v) + (size_t)bg * s.A * kRow;
    copy_pieces<NT, U>(n_adm * 2 * kChunks, [&](int e, const uint4*& from_p, uint4*& to_p) {
        const int j = e / (2 * kChunks);
        const int c = e % (2 * kChunks);
        const int from = src[j], to = dest[j];
        if (c < kChunks) {
            from_p = reinterpret_cast<const uint4*>(pk + (size_t)from * kRow) + c;
            to_p = reinterpret_cast<uint4*>(bk + (size_t)to * kRow) + c;
        } else {
            from_p = reinterpret_cast<const uint4*>(pv + (size_t)from * kRow) + (c - kChunks);
            to_p = reinterpret_cast<uint4*>(bv + (size_t)to * kRow) + (c - kChunks);
        }
    });
}

// Where admit_select leaves its result in the scratch: the admitted candidates' pending slots
// src[j], ascending, and the bank slots they go to, dest[j], ascending, j < n_adm.
__device__ __forceinline__ int* admit_src(uint8_t* scratch, int A, int P) {
    return reinterpret_cast<int*>(scratch + ((size_t)(A + P) * 8 + (A + P) + 15) / 16 * 16);
}
__device__ __forceinline__ int* admit_dest(uint8_t* scratch, int A, int P) { return admit_src(scratch, A, P) + P; }

// The competition of group bg (nb committed records, np candidates, both validated): every
// thread of the CTA (NT of them) calls it.  pscore_of(t) is candidate t's score (t < np).
// Returns n_adm and leaves the lists in the scratch (admit_src / admit_dest); the kept count is
// min(A, nb + np).  Reads scores only; writes nothing outside the scratch but the status word.
template <int NT, class PScore>
__device__ int admit_select(const LayerView& s, int bg, int nb, int np, uint8_t* scratch, PScore pscore_of) {
    const int A = s.A, P = s.P;
    const int tid = threadIdx.x;
    const int n = nb + np;
    const int k = min(A, n);

    uint64_t* keys = reinterpret_cast<uint64_t*>(scratch);
    uint8_t* kept_bank = reinterpret_cast<uint8_t*>(keys + (A + P));
    uint8_t* kept_pend = kept_bank + A;
    int* ints = reinterpret_cast<int*>(scratch + ((size_t)(A + P) * 8 + (A + P) + 15) / 16 * 16);
    int* src = ints;              // [P]
    int* dest = src + P;          // [P]
    int* hist = dest + P;         // [256]
    int* misc = hist + 256;       // [64]: warp totals [0,32), then shared scalars
    int* s_total = misc + 32;
    int* s_digit = misc + 33;
    int* s_need = misc + 34;
    int* s_count = misc + 35;
    int* s_nan = misc + 36;
    unsigned long long* s_tau = reinterpret_cast<unsigned long long*>(misc + 38);   // 8-aligned

    const float* bscore = s.bank_score + (size_t)bg * A;
    if (tid == 0) *s_nan = 0;
    __syncthreads();
    bool nan_seen = false;
    for (int i = tid; i < n; i += NT) {
        const bool committed = i < nb;
        const float sc = committed ? bscore[i] : pscore_of(i - nb);
        nan_seen |= isnan(sc);
        keys[i] = admit_key(sc, committed, committed ? i : i - nb);
    }
    for (int i = tid; i < A + P; i += NT) kept_bank[i] = 0;   // kept_pend follows kept_bank
    if (nan_seen) *s_nan = 1;
    __syncthreads();
    if (tid == 0 && *s_nan) atomicOr(s.status, (unsigned)RMA_STATUS_NAN_SCORE);

    if (n <= A) {
        for (int i = tid; i < nb; i += NT) kept_bank[i] = 1;
        for (int i = tid; i < np; i += NT) kept_pend[i] = 1;
    } else {
        // radix select of the k-th largest key
        uint64_t prefix = 0, mask = 0;
        if (tid == 0) *s_need = k;
        bool found = false;
        for (int shift = 56; shift >= 0 && !found; shift -= 8) {
            for (int i = tid; i < 256; i += NT) hist[i] = 0;
            __syncthreads();
            for (int i = tid; i < n; i += NT) {
                const uint64_t key = keys[i];
                if ((key & mask) == prefix) atomicAdd(&hist[(int)((key >> shift) & 0xFF)], 1);
            }
            __syncthreads();
            if (tid < 32) {
                // lane L covers digits 255-8L .. 248-8L (from the top down)
                const int lane = tid;
                int c[8], sum = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    c[e] = hist[255 - 8 * lane - e];
                    sum += c[e];
                }
                int incl = sum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += t;
                }
                const int above = incl - sum;   // keys with a larger digit in earlier lanes
                const int need = *s_need;
                const unsigned hit = __ballot_sync(0xffffffffu, above < need && need <= incl);
                const int owner = __ffs(hit) - 1;
                if (lane == owner) {
                    int acc = above;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        if (acc < need && need <= acc + c[e]) {
                            *s_digit = 255 - 8 * lane - e;
                            *s_count = c[e];
                            *s_need = need - acc;
                            break;
                        }
                        acc += c[e];
                    }
                }
            }
            __syncthreads();
            prefix |= (uint64_t)(*s_digit) << shift;
            mask |= (uint64_t)0xFF << shift;
            found = (*s_count == 1);
            __syncthreads();
        }
        // the k-th largest key is the one key with this prefix (unique keys)
        for (int i = tid; i < n; i += NT)
            if ((keys[i] & mask) == prefix) *s_tau = keys[i];
        __syncthreads();
        const uint64_t tau = *s_tau;
        for (int i = tid; i < n; i += NT) {
            if (keys[i] >= tau) {
                if (i < nb) kept_bank[i] = 1;
                else kept_pend[i - nb] = 1;
            }
        }
    }
    __syncthreads();

    // admitted candidates in ascending pending slot -> src[j]
    int n_adm;
    {
        constexpr int kSegDiv = NT;
        const int seg = (P + kSegDiv - 1) / kSegDiv;
        const int t0 = tid * seg, t1 = min(P, t0 + seg);
        int c = 0;
        for (int t = t0; t < t1; ++t) c += (t < np) && kept_pend[t];
        int idx = admit_block_scan<NT>(c, misc, s_total);
        for (int t = t0; t < t1; ++t)
            if ((t < np) && kept_pend[t]) src[idx++] = t;
        n_adm = *s_total;
    }
    // vacated bank slots (evicted anchors and empty slots), ascending -> dest[j] (first n_adm only)
    {
        const int seg = (A + NT - 1) / NT;
        const int s0 = tid * seg, s1 = min(A, s0 + seg);
        int c = 0;
        for (int sl = s0; sl < s1; ++sl) c += (sl >= nb) || !kept_bank[sl];
        int idx = admit_block_scan<NT>(c, misc, s_total);
        for (int sl = s0; sl < s1; ++sl) {
            if ((sl >= nb) || !kept_bank[sl]) {
                if (idx < n_adm) dest[idx] = sl;
                ++idx;
            }
        }
    }
    __syncthreads();
    return n_adm;
}

// Admit group bg of layer view s with nb committed records and np candidates
// (both already validated).  Every thread of the CTA (NT of them) must call it; each
// thread keeps U 16-byte pieces of the row copies in flight;
// `scratch` is shared memory of admit_scratch_bytes(A, P) bytes, 16-aligned.
// Writes the bank rows, scores and the counters bank_fill and pend_fill.
template <int NT, int U = 8>
__device__ void admit_group(const LayerView& s, int bg, int nb, int np, uint8_t* scratch) {
    const int A = s.A, P = s.P;
    const int tid = threadIdx.x;
    const int k = min(A, nb + np);
    const float* pscore = s.pend_score + (size_t)bg * P;
    const int n_adm = admit_select<NT>(s, bg, nb, np, scratch, [&](int t) { return pscore[t]; });
    const int* src = admit_src(scratch, A, P);
    const int* dest = admit_dest(scratch, A, P);

    if (s.fp8) {
        admit_copy_rows<NT, U, kHeadDim / 16>(s, bg, n_adm, src, dest);
        for (int j = tid; j < n_adm; j += NT) {
            s.bank_ke[(size_t)bg * s.AE + dest[j]] = s.pend_ke[(size_t)bg * s.PE + src[j]];
            s.bank_ve[(size_t)bg * s.AE + dest[j]] = s.pend_ve[(size_t)bg * s.PE + src[j]];
        }
    } else {
        admit_copy_rows<NT, U, kRowBytes / 16>(s, bg, n_adm, src, dest);
    }
    for (int j = tid; j < n_adm; j += NT) s.bank_score[(size_t)bg * A + dest[j]] = pscore[src[j]];
    if (tid == 0) {
        int32_t* cnt = s.counters + bg * 4;
        cnt[1] = k;
        cnt[2] = 0;
    }
    __syncthreads();
}

}  // namespace rma
