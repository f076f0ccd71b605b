// rma_admit: committed anchors and pending candidates compete; the top
// min(A, bank_fill + pend_fill) are kept per (sequence, layer, KV group).
//
// ("EdgeRock-4B holds KV cache at 72 MiB ..." (tpsreport.news), "How it
// works": after every 256 candidates they are compared with the existing
// anchors and the top 1,024 are kept, independently in each of four KV
// groups; ai-primer story, operations list, item 2 "Admit"; "EdgeRock" model
// card: retained records remain separate and unchanged.)
//
// The standalone admit launch: one CTA per (b, g), exiting at once unless
// that group's pending buffer is full (or the admit is forced).  The work
// itself is admit_group() in rma_admit_impl.cuh, shared with the fused
// decode and prefill paths.
#include <math_constants.h>

#include "rma_admit_impl.cuh"
#include "rma_internal.cuh"

namespace rma {
namespace {

constexpr int kThreads = 256;

// One CTA per (b, g); four CTAs per SM (64 registers a thread) keep more groups in flight.
__global__ void __launch_bounds__(kThreads, 4) admit_kernel(const __grid_constant__ LayerView s, int force) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int g = blockIdx.x, b = blockIdx.y;
    const int bg = b * s.G + g;
    const int tid = threadIdx.x;
    int32_t* cnt = s.counters + bg * 4;
    int nb = cnt[1], np = cnt[2];
    if (nb < 0 || nb > s.A || np < 0 || np > s.P) {
        // a corrupted state: never index outside the buffers
        if (tid == 0) atomicOr(s.status, (unsigned)RMA_STATUS_BAD_COUNTERS);
        nb = min(max(nb, 0), s.A);
        np = min(max(np, 0), s.P);
    }
    if (!(np == s.P || (force && np > 0))) return;
    admit_group<kThreads>(s, bg, nb, np, smem);
}

}  // namespace

cudaError_t launch_admit(const LayerView& s, int force, cudaStream_t stream) {
    const size_t smem = admit_scratch_bytes(s.A, s.P);
    static SmemLimit limit(reinterpret_cast<const void*>(admit_kernel));
    const cudaError_t e = limit.ensure(smem);
    if (e != cudaSuccess) return e;
    dim3 grid(s.G, s.B);
    admit_kernel<<<grid, kThreads, smem, stream>>>(s, force);
    return cudaGetLastError();
}

}  // namespace rma
