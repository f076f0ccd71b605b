// Internal declarations shared by the librma translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "rma.h"

namespace rma {

// A kernel's dynamic shared-memory limit, raised past the default 48 KiB the first time a
// launch on a device needs more.  The attribute belongs to the kernel as loaded on each
// device, so the largest size set is tracked per device (devices past the first 64 set it
// on every launch).  Safe to call from several host threads.
class SmemLimit {
  public:
    explicit SmemLimit(const void* func) : func_(func) {}

    cudaError_t ensure(size_t bytes) {
        if (bytes <= 48 * 1024) return cudaSuccess;
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        const bool tracked = dev >= 0 && dev < kTracked;
        if (tracked && set_[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
        std::lock_guard<std::mutex> lock(mu_);
        // never lower a limit another thread raised for a larger launch on this device
        const size_t want = tracked ? std::max(bytes, set_[dev].load(std::memory_order_relaxed)) : bytes;
        e = cudaFuncSetAttribute(func_, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)want);
        if (e == cudaSuccess && tracked) set_[dev].store(want, std::memory_order_release);
        return e;
    }

  private:
    static constexpr int kTracked = 64;
    const void* func_;
    std::mutex mu_;
    std::atomic<size_t> set_[kTracked] = {};
};

constexpr int kHeadDim = 256;        // D: elements per K/V/Q row
constexpr int kQPerGroup = 4;        // H: query heads reading one KV group
constexpr int kRowBytes = kHeadDim * 2;

// Host-side state handle: the caller's device buffer plus its layout.
struct State {
    rma_config cfg;
    rma_layout lay;
    uint8_t* base;         // device
    int ring_splits_override;
    int bank_splits_override;
    int sm_count;
    int decode_overlap;    // rma_set_decode_overlap
};

// Per-call view of one layer of the state, with device pointers already
// offset to that layer.  All [.][.] shapes below are [batch][n_groups].
struct LayerView {
    uint16_t* ring_k;      // [B][G][R][D]
    uint16_t* ring_v;
    uint16_t* bank_k;      // [B][G][A][D]
    uint16_t* bank_v;
    float* bank_score;     // [B][G][A]
    uint16_t* pend_k;      // [B][G][P][D]
    uint16_t* pend_v;
    float* pend_score;     // [B][G][P]
    int32_t* counters;     // [B][G][4] = pos, bank_fill, pend_fill, 0
    uint32_t* tickets;     // [B][G]
    uint32_t* status;
    int B, G, R, A, P;
    // FP8 storage (fp8 != 0): the K/V pointers above hold u8 E4M3 codes with the same shapes
    // (reinterpret them as bytes), and each row's scale exponent lives in these arrays,
    // [B][G][RE] etc., RE / AE / PE = R / A / P rounded up to 16 (null in a BF16 state)
    int fp8;
    int8_t* ring_ke;
    int8_t* ring_ve;
    int8_t* bank_ke;
    int8_t* bank_ve;
    int8_t* pend_ke;
    int8_t* pend_ve;
    int RE, AE, PE;
};

// Bytes of one stored K or V row.
__host__ __device__ __forceinline__ int row_bytes(const LayerView& s) { return s.fp8 ? kHeadDim : kRowBytes; }

struct DecodeArgs {
    LayerView s;
    const uint16_t* q;          // [B][G*H][D]
    const uint16_t* k_cur;      // [B][G][D]
    const uint16_t* v_cur;
    const uint16_t* cand_k;
    const uint16_t* cand_v;
    const float* cand_score;    // [B][G]
    const float* w_g;           // [G*H][D]
    const float* b_g;           // [G*H]
    uint16_t* out;              // [B][G*H][D]
    float* ws;                  // partials [B][G][splits][kPartialFloats]
    int ring_splits, bank_splits;
    int ring_chunk, bank_chunk; // rows per split (multiples of 16)
    float qscale;               // softmax_scale * log2(e)
    int early;                  // 1: stream the ring and bank before waiting on the previous launch
};

struct PrefillArgs {
    LayerView s;
    const uint16_t* q;          // [B][n][G*H][D]
    const uint16_t* k;          // [B][n][G][D]
    const uint16_t* v;
    const uint16_t* cand_k;
    const uint16_t* cand_v;
    const float* cand_score;    // [B][n][G]
    const float* w_g;
    const float* b_g;
    uint16_t* out;              // [B][n][G*H][D]
    float* ws;
    int n_tok;
    float qscale;
};

// One split's partial softmax result for the 4 heads of a group:
// m[4] (running max, log2 domain), l[4] (sum of exponentials), acc[4][D].
constexpr int kPartialFloats = 4 + 4 + kQPerGroup * kHeadDim;

// Size of the library's own decode scratch (rma_decode_step_noalloc).
constexpr size_t kStaticDecodeScratchBytes = size_t(32) << 20;
// Device address of that scratch in the current context (looked up on every call).
cudaError_t static_decode_scratch(void** ptr);

// Launchers (each returns cudaGetLastError() of its launch).
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_admit(const LayerView& s, int force, cudaStream_t stream);
// Longest prefill block (tokens per sequence) one rma_prefill_block call takes.
constexpr int kMaxPrefillTokens = 256;
cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream);
// Quantise every row of `src` (BF16) into `dst` (FP8), one layer at a time; scores and counters copied.
cudaError_t launch_quantize_layer(const LayerView& dst, const LayerView& src, cudaStream_t stream);
size_t prefill_workspace_bytes(const rma_config& cfg, int n_tok);

}  // namespace rma
