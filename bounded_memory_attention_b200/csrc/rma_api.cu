// librma host side: argument checks, state layout, split choice, launches.
// The C declarations and their documentation are in include/rma.h.
#include <cmath>
#include <cstdio>
#include <map>
#include <mutex>
#include <new>
#include <string>
#include <utility>

#include <nvtx3/nvToolsExt.h>

#include "rma_internal.cuh"

namespace rma {
namespace {

thread_local std::string g_last_error;

int fail(int code, const std::string& why) {
    g_last_error = why;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(RMA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// An NVTX range named after the API call around its host work and launches, so that a
// profiler's launch list shows which call issued each kernel (no cost without a profiler).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr uint64_t kAlign = 256;
constexpr int kMaxDecodeSplits = 64;   // must match the decode kernel's kMaxSplits

uint64_t round_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_config(const rma_config* c) {
    if (!c) return fail(RMA_ERR_INVALID_ARG, "config is NULL");
    if (c->batch < 1 || c->n_layers < 1 || c->n_groups < 1)
        return fail(RMA_ERR_INVALID_ARG, "batch, n_layers and n_groups must be >= 1");
    if (c->ring_slots < 1 || c->bank_slots < 1 || c->pend_slots < 1)
        return fail(RMA_ERR_INVALID_ARG, "ring_slots, bank_slots and pend_slots must be >= 1");
    if (!(std::isfinite(c->softmax_scale) && c->softmax_scale > 0.f))
        return fail(RMA_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
    if (c->q_per_group != kQPerGroup || c->head_dim != kHeadDim)
        return fail(RMA_ERR_UNSUPPORTED, "the library implements q_per_group == 4 and head_dim == 256");
    if (c->ring_slots > (1 << 20)) return fail(RMA_ERR_UNSUPPORTED, "ring_slots > 2^20");
    if (c->bank_slots + c->pend_slots > 4096) return fail(RMA_ERR_UNSUPPORTED, "bank_slots + pend_slots > 4096");
    if (c->batch > 65535 || c->n_groups > 65535) return fail(RMA_ERR_UNSUPPORTED, "batch or n_groups > 65535");
    if ((int64_t)c->batch * c->n_groups > (1 << 24)) return fail(RMA_ERR_UNSUPPORTED, "batch * n_groups > 2^24");
    if (c->kv_format != RMA_KV_BF16 && c->kv_format != RMA_KV_FP8_E4M3)
        return fail(RMA_ERR_INVALID_ARG, "kv_format must be RMA_KV_BF16 or RMA_KV_FP8_E4M3");
    return RMA_OK;
}

// Slot count rounded up to 16: the stride of an FP8 state's exponent arrays, so that the
// exponents of 16 consecutive rows start on a 16-byte boundary.
uint64_t pad16(int n) { return round_up((uint64_t)n, 16); }

void compute_layout(const rma_config& c, rma_layout& L) {
    const uint64_t lbg = (uint64_t)c.n_layers * c.batch * c.n_groups;
    const bool fp8 = c.kv_format == RMA_KV_FP8_E4M3;
    const uint64_t row = (uint64_t)c.head_dim * (fp8 ? 1 : 2);
    uint64_t off = 0;
    auto take = [&](uint64_t bytes) {
        const uint64_t o = off;
        off = round_up(off + bytes, kAlign);
        return o;
    };
    L.ring_k = take(lbg * c.ring_slots * row);
    L.ring_v = take(lbg * c.ring_slots * row);
    L.bank_k = take(lbg * c.bank_slots * row);
    L.bank_v = take(lbg * c.bank_slots * row);
    L.bank_score = take(lbg * c.bank_slots * 4);
    L.pend_k = take(lbg * c.pend_slots * row);
    L.pend_v = take(lbg * c.pend_slots * row);
    L.pend_score = take(lbg * c.pend_slots * 4);
    L.counters = take(lbg * 16);
    L.tickets = take(lbg * 4);
    L.status = take(4);
    L.ring_k_exp = L.ring_v_exp = L.bank_k_exp = L.bank_v_exp = L.pend_k_exp = L.pend_v_exp = 0;
    if (fp8) {
        L.ring_k_exp = take(lbg * pad16(c.ring_slots));
        L.ring_v_exp = take(lbg * pad16(c.ring_slots));
        L.bank_k_exp = take(lbg * pad16(c.bank_slots));
        L.bank_v_exp = take(lbg * pad16(c.bank_slots));
        L.pend_k_exp = take(lbg * pad16(c.pend_slots));
        L.pend_v_exp = take(lbg * pad16(c.pend_slots));
    }
    L.total_bytes = off;
}

LayerView layer_view(const State& s, int layer) {
    const rma_config& c = s.cfg;
    const uint64_t bg = (uint64_t)c.batch * c.n_groups;
    const uint64_t l = (uint64_t)layer;
    const bool fp8 = c.kv_format == RMA_KV_FP8_E4M3;
    const uint64_t rowb = (uint64_t)c.head_dim * (fp8 ? 1 : 2);
    auto rows = [&](uint64_t off, int slots) {   // layer `layer` of a K/V array (bytes, as uint16_t*)
        return reinterpret_cast<uint16_t*>(s.base + off + l * bg * slots * rowb);
    };
    LayerView v;
    v.ring_k = rows(s.lay.ring_k, c.ring_slots);
    v.ring_v = rows(s.lay.ring_v, c.ring_slots);
    v.bank_k = rows(s.lay.bank_k, c.bank_slots);
    v.bank_v = rows(s.lay.bank_v, c.bank_slots);
    v.bank_score = reinterpret_cast<float*>(s.base + s.lay.bank_score) + l * bg * c.bank_slots;
    v.pend_k = rows(s.lay.pend_k, c.pend_slots);
    v.pend_v = rows(s.lay.pend_v, c.pend_slots);
    v.pend_score = reinterpret_cast<float*>(s.base + s.lay.pend_score) + l * bg * c.pend_slots;
    v.counters = reinterpret_cast<int32_t*>(s.base + s.lay.counters) + l * bg * 4;
    v.tickets = reinterpret_cast<uint32_t*>(s.base + s.lay.tickets) + l * bg;
    v.status = reinterpret_cast<uint32_t*>(s.base + s.lay.status);
    v.B = c.batch;
    v.G = c.n_groups;
    v.R = c.ring_slots;
    v.A = c.bank_slots;
    v.P = c.pend_slots;
    v.fp8 = fp8 ? 1 : 0;
    v.RE = (int)pad16(c.ring_slots);
    v.AE = (int)pad16(c.bank_slots);
    v.PE = (int)pad16(c.pend_slots);
    auto exps = [&](uint64_t off, int stride) {
        return fp8 ? reinterpret_cast<int8_t*>(s.base + off) + l * bg * stride : nullptr;
    };
    v.ring_ke = exps(s.lay.ring_k_exp, v.RE);
    v.ring_ve = exps(s.lay.ring_v_exp, v.RE);
    v.bank_ke = exps(s.lay.bank_k_exp, v.AE);
    v.bank_ve = exps(s.lay.bank_v_exp, v.AE);
    v.pend_ke = exps(s.lay.pend_k_exp, v.PE);
    v.pend_ve = exps(s.lay.pend_v_exp, v.PE);
    return v;
}

struct Splits {
    int ring_splits, bank_splits, ring_chunk, bank_chunk;
};

// Cut `rows` into at most `want` contiguous ranges of a multiple of 16 rows (the decode
// kernel's tensor-core tile).
void cut(int rows, int want, int& n, int& chunk) {
    want = want < 1 ? 1 : want;
    chunk = (rows + want - 1) / want;
    chunk = (chunk + 15) / 16 * 16;
    if (chunk < 16) chunk = 16;
    n = (rows + chunk - 1) / chunk;
}

Splits decode_splits(const State& s) {
    const rma_config& c = s.cfg;
    int want_r = s.ring_splits_override, want_b = s.bank_splits_override;
    if (want_r <= 0 || want_b <= 0) {
        // One CTA per SM at a time.  From 16 (sequence, group) units up, about half a wave of CTAs:
        // the tensor-core kernel streams a split fast enough that fewer, longer splits (less merging)
        // win; a batch of 1 or 2 is latency bound and takes the most splits (8 + 8, 128 rows each
        // for the pages' ring and bank).
        const long units = (long)c.batch * c.n_groups;
        const long target = (long)s.sm_count / 2;
        long per_unit = units <= 8 ? 16 : (target + units - 1) / units;
        if (per_unit < 2) per_unit = 2;
        if (per_unit > 16) per_unit = 16;
        want_r = (int)(per_unit / 2);
        want_b = (int)(per_unit - per_unit / 2);
    }
    Splits sp;
    cut(c.ring_slots, want_r, sp.ring_splits, sp.ring_chunk);
    cut(c.bank_slots, want_b, sp.bank_splits, sp.bank_chunk);
    return sp;
}

// The kernel this library launched last on each stream (a stream being captured counts as a
// separate stream per capture), for the decode overlap rule: a decode launch may request its ring
// and bank before the previous kernel finishes only when that kernel is a decode of another layer
// (or another state).
struct LastLaunch {
    bool decode = false;
    const void* state = nullptr;
    int layer = -1;
};
std::mutex g_launch_mu;
std::map<std::pair<uintptr_t, unsigned long long>, LastLaunch> g_last_launch;

std::pair<uintptr_t, unsigned long long> launch_key(cudaStream_t stream) {
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    unsigned long long id = 0;
    if (cudaStreamGetCaptureInfo(stream, &st, &id) != cudaSuccess) {
        (void)cudaGetLastError();
        id = ~0ull;
    } else if (st != cudaStreamCaptureStatusActive) {
        id = 0;
    }
    return {reinterpret_cast<uintptr_t>(stream), id};
}

// Record a launch of this library on `stream` (call with g_launch_mu held).
void record_launch(const std::pair<uintptr_t, unsigned long long>& key, const LastLaunch& l) {
    if (g_last_launch.size() > 4096) g_last_launch.clear();   // captures that ended long ago
    g_last_launch[key] = l;
}

// A non-decode launch of this library on `stream`.
void note_other_launch(cudaStream_t stream) {
    std::lock_guard<std::mutex> lock(g_launch_mu);
    record_launch(launch_key(stream), LastLaunch{});
}

State* as_state(rma_state* p) { return reinterpret_cast<State*>(p); }
const State* as_state(const rma_state* p) { return reinterpret_cast<const State*>(p); }

int check_layer(const State* s, int layer) {
    if (!s) return fail(RMA_ERR_INVALID_ARG, "state is NULL");
    if (layer < 0 || layer >= s->cfg.n_layers) return fail(RMA_ERR_INVALID_ARG, "layer index out of range");
    return RMA_OK;
}

}  // namespace
}  // namespace rma

using namespace rma;

extern "C" {

size_t rma_state_bytes(const rma_config* cfg) {
    if (check_config(cfg) != RMA_OK) return 0;
    rma_layout L;
    compute_layout(*cfg, L);
    return (size_t)L.total_bytes;
}

int rma_state_alloc(const rma_config* cfg, void* dev_buf, size_t dev_bytes, void* stream, rma_state** out) {
    int rc = check_config(cfg);
    if (rc != RMA_OK) return rc;
    if (!dev_buf || !out) return fail(RMA_ERR_INVALID_ARG, "dev_buf and out must be non-NULL");
    if (!aligned(dev_buf, kAlign)) return fail(RMA_ERR_MISALIGNED, "dev_buf must be 256-byte aligned");
    rma_layout L;
    compute_layout(*cfg, L);
    if (dev_bytes < L.total_bytes)
        return fail(RMA_ERR_BUFFER_TOO_SMALL, "state buffer smaller than rma_state_bytes()");
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "querying the device");
    State* s = new (std::nothrow) State;
    if (!s) return fail(RMA_ERR_INVALID_ARG, "host allocation of the handle failed");
    s->cfg = *cfg;
    s->lay = L;
    s->base = static_cast<uint8_t*>(dev_buf);
    s->ring_splits_override = 0;
    s->bank_splits_override = 0;
    s->sm_count = sms;
    s->decode_overlap = 0;
    e = cudaMemsetAsync(s->base + L.counters, 0, L.total_bytes - L.counters, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        delete s;
        return cuda_fail(e, "zeroing counters");
    }
    *out = reinterpret_cast<rma_state*>(s);
    return RMA_OK;
}

int rma_state_layout(const rma_state* st, rma_layout* out) {
    if (!st || !out) return fail(RMA_ERR_INVALID_ARG, "state and out must be non-NULL");
    *out = as_state(st)->lay;
    return RMA_OK;
}

void rma_state_free(rma_state* st) { delete as_state(st); }

int rma_workspace_bytes(const rma_state* st, int n_tok, size_t* out) {
    if (!st || !out) return fail(RMA_ERR_INVALID_ARG, "state and out must be non-NULL");
    const State* s = as_state(st);
    if (n_tok < 1) return fail(RMA_ERR_INVALID_ARG, "n_tok must be >= 1");
    if (n_tok > kMaxPrefillTokens) return fail(RMA_ERR_UNSUPPORTED, "n_tok > 256");
    size_t bytes = prefill_workspace_bytes(s->cfg, n_tok);
    if (n_tok == 1) {   // a decode step, or a one-token prefill block: enough for either
        const Splits sp = decode_splits(*s);
        const size_t dec = (size_t)s->cfg.batch * s->cfg.n_groups * (sp.ring_splits + sp.bank_splits) * kPartialFloats * 4;
        bytes = dec > bytes ? dec : bytes;
    }
    *out = bytes;
    return RMA_OK;
}

int rma_set_decode_splits(rma_state* st, int ring_splits, int bank_splits) {
    if (!st) return fail(RMA_ERR_INVALID_ARG, "state is NULL");
    if (ring_splits == 0 && bank_splits == 0) {
        as_state(st)->ring_splits_override = 0;
        as_state(st)->bank_splits_override = 0;
        return RMA_OK;
    }
    if (ring_splits < 1 || bank_splits < 1 || ring_splits + bank_splits > kMaxDecodeSplits)
        return fail(RMA_ERR_INVALID_ARG, "splits must be >= 1 each and <= 64 together (or both 0)");
    as_state(st)->ring_splits_override = ring_splits;
    as_state(st)->bank_splits_override = bank_splits;
    return RMA_OK;
}

int rma_decode_step(rma_state* st, int layer, const uint16_t* q, const uint16_t* k_cur, const uint16_t* v_cur,
                    const uint16_t* cand_k, const uint16_t* cand_v, const float* cand_score, const float* w_g,
                    const float* b_g, uint16_t* out, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange range("rma_decode_step");
    State* s = as_state(st);
    int rc = check_layer(s, layer);
    if (rc != RMA_OK) return rc;
    if (!q || !k_cur || !v_cur || !cand_k || !cand_v || !cand_score || !w_g || !b_g || !out || !ws)
        return fail(RMA_ERR_INVALID_ARG, "a tensor pointer is NULL");
    const void* a16[] = {q, k_cur, v_cur, cand_k, cand_v, w_g, out, ws};
    for (const void* p : a16)
        if (!aligned(p, 16)) return fail(RMA_ERR_MISALIGNED, "q, k_cur, v_cur, cand_k, cand_v, w_g, out, ws need 16-byte alignment");
    if (!aligned(cand_score, 4) || !aligned(b_g, 4)) return fail(RMA_ERR_MISALIGNED, "cand_score and b_g need 4-byte alignment");
    const Splits sp = decode_splits(*s);
    const size_t need = (size_t)s->cfg.batch * s->cfg.n_groups * (sp.ring_splits + sp.bank_splits) * kPartialFloats * 4;
    if (ws_bytes < need) return fail(RMA_ERR_BUFFER_TOO_SMALL, "workspace smaller than rma_workspace_bytes(st, 1)");
    if (sp.ring_splits + sp.bank_splits > kMaxDecodeSplits) return fail(RMA_ERR_UNSUPPORTED, "too many splits");
    DecodeArgs a;
    a.s = layer_view(*s, layer);
    a.q = q;
    a.k_cur = k_cur;
    a.v_cur = v_cur;
    a.cand_k = cand_k;
    a.cand_v = cand_v;
    a.cand_score = cand_score;
    a.w_g = w_g;
    a.b_g = b_g;
    a.out = out;
    a.ws = static_cast<float*>(ws);
    a.ring_splits = sp.ring_splits;
    a.bank_splits = sp.bank_splits;
    a.ring_chunk = sp.ring_chunk;
    a.bank_chunk = sp.bank_chunk;
    a.qscale = s->cfg.softmax_scale * 1.4426950408889634f;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    {
        std::lock_guard<std::mutex> lock(g_launch_mu);
        const auto key = launch_key(cs);
        a.early = 0;
        if (s->decode_overlap) {
            const auto it = g_last_launch.find(key);
            // the ring and bank of this layer may be read early when the previous kernel on the
            // stream is a decode of another layer (or another state): it writes nothing of them
            a.early = (it != g_last_launch.end() && it->second.decode &&
                       !(it->second.state == s->base && it->second.layer == layer)) ? 1 : 0;
        }
        e = launch_decode(a, cs);
        if (e == cudaSuccess) {
            LastLaunch l;
            l.decode = true;
            l.state = s->base;
            l.layer = layer;
            record_launch(key, l);
        }
    }
    if (e != cudaSuccess) return cuda_fail(e, "launching rma_decode");
    return RMA_OK;
}

int rma_set_decode_overlap(rma_state* st, int enable) {
    if (!st) return fail(RMA_ERR_INVALID_ARG, "state is NULL");
    if (enable != 0 && enable != 1) return fail(RMA_ERR_INVALID_ARG, "enable must be 0 or 1");
    as_state(st)->decode_overlap = enable;
    return RMA_OK;
}

int rma_decode_step_noalloc(rma_state* st, int layer, const uint16_t* q, const uint16_t* k_cur,
                            const uint16_t* v_cur, const uint16_t* cand_k, const uint16_t* cand_v,
                            const float* cand_score, const float* w_g, const float* b_g, uint16_t* out,
                            void* stream) {
    NvtxRange range("rma_decode_step_noalloc");
    State* s = as_state(st);
    int rc = check_layer(s, layer);
    if (rc != RMA_OK) return rc;
    const Splits sp = decode_splits(*s);
    const size_t need =
        (size_t)s->cfg.batch * s->cfg.n_groups * (sp.ring_splits + sp.bank_splits) * kPartialFloats * 4;
    if (need > kStaticDecodeScratchBytes)
        return fail(RMA_ERR_BUFFER_TOO_SMALL,
                    "rma_decode_step_noalloc: this batch and split shape need " + std::to_string(need) +
                        " bytes of scratch but the built-in scratch holds " +
                        std::to_string(kStaticDecodeScratchBytes) +
                        " (use fewer sequences per call, fewer splits, or rma_decode_step with a workspace)");
    void* scratch = nullptr;
    cudaError_t e = static_decode_scratch(&scratch);
    if (e != cudaSuccess) return cuda_fail(e, "looking up the built-in decode scratch");
    return rma_decode_step(st, layer, q, k_cur, v_cur, cand_k, cand_v, cand_score, w_g, b_g, out, scratch,
                           kStaticDecodeScratchBytes, stream);
}

int rma_admit(rma_state* st, int layer, int force, void* stream) {
    NvtxRange range("rma_admit");
    State* s = as_state(st);
    int rc = check_layer(s, layer);
    if (rc != RMA_OK) return rc;
    if (force != 0 && force != 1) return fail(RMA_ERR_INVALID_ARG, "force must be 0 or 1");
    cudaError_t e = launch_admit(layer_view(*s, layer), force, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "launching rma_admit");
    note_other_launch(static_cast<cudaStream_t>(stream));
    return RMA_OK;
}

int rma_prefill_block(rma_state* st, int layer, int n_tok, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      const uint16_t* cand_k, const uint16_t* cand_v, const float* cand_score, const float* w_g,
                      const float* b_g, uint16_t* out, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange range("rma_prefill_block");
    State* s = as_state(st);
    int rc = check_layer(s, layer);
    if (rc != RMA_OK) return rc;
    if (!q || !k || !v || !cand_k || !cand_v || !cand_score || !w_g || !b_g || !out || !ws)
        return fail(RMA_ERR_INVALID_ARG, "a tensor pointer is NULL");
    const void* a16[] = {q, k, v, cand_k, cand_v, w_g, out, ws};
    for (const void* p : a16)
        if (!aligned(p, 16)) return fail(RMA_ERR_MISALIGNED, "q, k, v, cand_k, cand_v, w_g, out, ws need 16-byte alignment");
    if (!aligned(cand_score, 4) || !aligned(b_g, 4)) return fail(RMA_ERR_MISALIGNED, "cand_score and b_g need 4-byte alignment");
    if (n_tok < 1) return fail(RMA_ERR_INVALID_ARG, "n_tok must be >= 1");
    if (s->cfg.kv_format != RMA_KV_BF16)
        return fail(RMA_ERR_UNSUPPORTED, "rma_prefill_block takes BF16 states (prefill in BF16, then rma_state_quantize)");
    if (n_tok > kMaxPrefillTokens || n_tok > s->cfg.ring_slots)
        return fail(RMA_ERR_UNSUPPORTED, "rma_prefill_block takes n_tok <= 256 and n_tok <= ring_slots");
    if (ws_bytes < prefill_workspace_bytes(s->cfg, n_tok))
        return fail(RMA_ERR_BUFFER_TOO_SMALL, "workspace smaller than rma_workspace_bytes(st, n_tok)");
    PrefillArgs a;
    a.s = layer_view(*s, layer);
    a.q = q;
    a.k = k;
    a.v = v;
    a.cand_k = cand_k;
    a.cand_v = cand_v;
    a.cand_score = cand_score;
    a.w_g = w_g;
    a.b_g = b_g;
    a.out = out;
    a.ws = static_cast<float*>(ws);
    a.n_tok = n_tok;
    a.qscale = s->cfg.softmax_scale * 1.4426950408889634f;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_prefill(a, cs);
    if (e == cudaErrorNotSupported) return fail(RMA_ERR_UNSUPPORTED, "this prefill block shape is not implemented");
    if (e != cudaSuccess) return cuda_fail(e, "launching rma_prefill_block");
    note_other_launch(cs);
    return RMA_OK;
}

int rma_state_quantize(rma_state* dst, const rma_state* src, void* stream) {
    NvtxRange range("rma_state_quantize");
    if (!dst || !src) return fail(RMA_ERR_INVALID_ARG, "dst and src must be non-NULL");
    State* d = as_state(dst);
    const State* s = as_state(src);
    if (d->cfg.kv_format != RMA_KV_FP8_E4M3 || s->cfg.kv_format != RMA_KV_BF16)
        return fail(RMA_ERR_INVALID_ARG, "rma_state_quantize takes an FP8 destination and a BF16 source");
    rma_config a = d->cfg, b = s->cfg;
    a.kv_format = b.kv_format = 0;
    if (a.batch != b.batch || a.n_layers != b.n_layers || a.n_groups != b.n_groups || a.ring_slots != b.ring_slots ||
        a.bank_slots != b.bank_slots || a.pend_slots != b.pend_slots)
        return fail(RMA_ERR_INVALID_ARG, "rma_state_quantize: the two states' dimensions differ");
    const uint8_t *d0 = d->base, *d1 = d->base + d->lay.total_bytes, *s0 = s->base, *s1 = s->base + s->lay.total_bytes;
    if (d0 < s1 && s0 < d1) return fail(RMA_ERR_INVALID_ARG, "rma_state_quantize: the two state buffers overlap");
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    for (int l = 0; l < d->cfg.n_layers; ++l) {
        const cudaError_t e = launch_quantize_layer(layer_view(*d, l), layer_view(*s, l), cs);
        if (e != cudaSuccess) return cuda_fail(e, "launching rma_state_quantize");
    }
    note_other_launch(cs);
    return RMA_OK;
}

int rma_get_status(rma_state* st, void* stream, uint32_t* flags) {
    if (!st || !flags) return fail(RMA_ERR_INVALID_ARG, "state and flags must be non-NULL");
    State* s = as_state(st);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    uint32_t h = 0;
    cudaError_t e = cudaMemcpyAsync(&h, s->base + s->lay.status, 4, cudaMemcpyDeviceToHost, cs);
    if (e == cudaSuccess) e = cudaMemsetAsync(s->base + s->lay.status, 0, 4, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
    *flags = h;
    return RMA_OK;
}

const char* rma_strerror(int code) {
    switch (code) {
        case RMA_OK: return "ok";
        case RMA_ERR_INVALID_ARG: return "invalid argument";
        case RMA_ERR_UNSUPPORTED: return "unsupported shape or option";
        case RMA_ERR_BUFFER_TOO_SMALL: return "buffer too small";
        case RMA_ERR_CUDA: return "CUDA error";
        case RMA_ERR_MISALIGNED: return "misaligned pointer";
        default: return "unknown error code";
    }
}

const char* rma_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
