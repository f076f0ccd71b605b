/*
 * librma: the Rock Memory Anchors (RMA) attention hot path on NVIDIA B200 (sm_100a).
 *
 * A C ABI over plain pointers and sizes.  Every device buffer is owned by the
 * caller; the library allocates no device memory, ever.  Calls are
 * asynchronous on the stream passed in (a cudaStream_t given as `void*`;
 * NULL is the legacy default stream) and return before the GPU work ends.
 *
 * Pages the operations come from (cited by title and section):
 *   [NEWS] "EdgeRock-4B holds KV cache at 72 MiB up to 256K context, with
 *          12,124 tokens/s on one 80GB GPU" (tpsreport.news)
 *   [PRIM] "EdgeRock-4B fixes its attention KV cache at 72 MiB" (ai-primer.com)
 *   [CARD] "EdgeRock" model card (modelscope.cn/models/rockmatrix/EdgeRock)
 *   [SITE] "Models / EdgeRock-4B" product page (rockmatrix.ai/models)
 *
 * State, per (sequence, RMA layer, KV group) ([CARD] "How Rock Memory Anchors
 * work", history-component table; [PRIM] persistent-history table):
 *   ring     R slots of (K, V)      the preceding positions of the local window
 *                                   (position p lives in slot p mod R); the
 *                                   decoder supplies the current token.
 *   bank     A records (K, V, score) committed anchors, valid prefix [0, bank_fill)
 *   pending  P records (K, V, score) candidates of the next admit, [0, pend_fill)
 *   counters pos, bank_fill, pend_fill
 * The pages fix R = 1023, A = 1024, P = 256, 4 KV groups, BF16 K/V; head_dim
 * 256 and 4 query heads per group follow from the source model's 32 KiB of KV
 * per token over 8 layers ([NEWS] "Throughput and memory").
 *
 * Numbers: K, V, Q and outputs are BF16, passed as their uint16_t bit
 * patterns; scores and gate parameters are FP32; all accumulation is FP32.
 *
 * Error behaviour: every call returns RMA_OK (0) or a negative RMA_ERR_* code.
 * Argument, shape, size and alignment errors are found on the host before
 * anything is launched; rma_last_error() then gives a one-line reason.
 * Conditions only the GPU can see never trap: they set bits in a device
 * status word (RMA_STATUS_*), read and cleared by rma_get_status().
 */
#ifndef RMA_H
#define RMA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RMA_API __attribute__((visibility("default")))
#else
#define RMA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes ---- */
#define RMA_OK                    0
#define RMA_ERR_INVALID_ARG      -1  /* null pointer, bad layer index, bad flag value */
#define RMA_ERR_UNSUPPORTED      -2  /* a shape the library does not implement */
#define RMA_ERR_BUFFER_TOO_SMALL -3  /* state buffer or workspace smaller than required */
#define RMA_ERR_CUDA             -4  /* a CUDA runtime call or kernel launch failed */
#define RMA_ERR_MISALIGNED       -5  /* a pointer lacks the alignment stated below */

/* ---- device status bits (rma_get_status) ---- */
/* A decode step found the pending buffer full (rma_admit was skipped): its
 * candidate was dropped; attention, ring write and pos advance still happened. */
#define RMA_STATUS_PENDING_OVERFLOW          1u
/* An admit met a NaN score; NaN ranks below every number (see rma_admit). */
#define RMA_STATUS_NAN_SCORE                 2u
/* A prefill block's candidates did not fit the pending buffer: they were
 * dropped; the rest of the block (attention, ring, forced admit) ran. */
#define RMA_STATUS_PREFILL_PENDING_OVERFLOW  4u
/* A kernel found counters outside their ranges (pos < 0, bank_fill not in
 * [0, bank_slots], pend_fill not in [0, pend_slots]), e.g. a corrupted restore:
 * it clamped them for its own indexing and went on. */
#define RMA_STATUS_BAD_COUNTERS              8u
/* A kernel gave up waiting on one of its own pipeline barriers, or a prefill
 * commit CTA on the attention launch's rows of its group (a bounded wait of
 * about two seconds ran out), and abandoned its work; its outputs are
 * not valid, and the state of the groups it served (slots, counters,
 * tickets) may be inconsistent: restore the state buffer from a copy or lay
 * it out afresh with rma_state_alloc before the next call on it.  Indicates
 * a fault in the library, never an input condition. */
#define RMA_STATUS_TIMEOUT                  16u

/* Storage of the ring, bank and pending K/V rows (rma_config.kv_format). */
#define RMA_KV_BF16      0   /* BF16 values, the pages' storage */
#define RMA_KV_FP8_E4M3  1   /* E4M3 codes with one power-of-two scale per stored row (see below) */

/* Dimensions.  The library implements q_per_group == 4 and head_dim == 256
 * (RMA_ERR_UNSUPPORTED otherwise), any n_groups >= 1, ring_slots in
 * [1, 1<<20], bank_slots >= 1, pend_slots >= 1, bank_slots + pend_slots <= 4096.
 *
 * kv_format RMA_KV_FP8_E4M3 halves the K/V bytes ([PRIM] packages paragraph
 * and [SITE] downloads list: FP8 packages validated for text inference; the
 * pages do not say how K/V would be stored in FP8, so this storage is the
 * library's own).  Each stored row (one position's K, or its V, for one KV
 * group) holds head_dim E4M3 codes (1 sign, 4 exponent bits with bias 7,
 * 3 mantissa bits, no infinities, S.1111.111 = NaN, max 448) and a signed
 * 8-bit exponent e: the row's values are code * 2^e, e the smallest integer
 * in [-127, 127] with max|x| <= 448 * 2^e (0 for an all-zero row), the codes
 * x * 2^-e rounded to nearest, ties to even.  Rows are quantised when written
 * (the ring write and candidate append of rma_decode_step, and
 * rma_state_quantize); the admit copies codes, exponents and scores
 * unchanged; attention reads the stored values, and the current token is
 * attended as passed in (BF16).  K/V inputs must be finite.  An FP8 state
 * takes rma_decode_step, rma_decode_step_noalloc, rma_admit and
 * rma_state_quantize; rma_prefill_block returns RMA_ERR_UNSUPPORTED on it
 * (prefill a BF16 state, then quantise it). */
typedef struct rma_config {
    int32_t batch;          /* independent sequences */
    int32_t n_layers;       /* RMA layers (8 in the pages' model) */
    int32_t n_groups;       /* KV groups (4) */
    int32_t q_per_group;    /* query heads per KV group (4) */
    int32_t head_dim;       /* D (256) */
    int32_t ring_slots;     /* R (1023) */
    int32_t bank_slots;     /* A (1024) */
    int32_t pend_slots;     /* P (256) */
    float   softmax_scale;  /* 1/sqrt(head_dim) = 1/16 */
    int32_t kv_format;      /* RMA_KV_BF16 (0) or RMA_KV_FP8_E4M3 (1) */
} rma_config;

/* Byte offsets, from the start of the caller's state buffer, of each array.
 * Every offset is a multiple of 256.  Shapes (row-major, innermost last):
 *   ring_k, ring_v        bf16  [n_layers][batch][n_groups][ring_slots][head_dim]
 *   bank_k, bank_v        bf16  [n_layers][batch][n_groups][bank_slots][head_dim]
 *   bank_score            f32   [n_layers][batch][n_groups][bank_slots]
 *   pend_k, pend_v        bf16  [n_layers][batch][n_groups][pend_slots][head_dim]
 *   pend_score            f32   [n_layers][batch][n_groups][pend_slots]
 *   counters              i32   [n_layers][batch][n_groups][4] = {pos, bank_fill, pend_fill, 0}
 *   tickets               u32   [n_layers][batch][n_groups]  (library-internal, zero between calls)
 *   status                u32   one word (RMA_STATUS_* bits)
 * In an RMA_KV_FP8_E4M3 state the six K/V arrays hold u8 E4M3 codes (same
 * shapes), and six more arrays hold the rows' scale exponents:
 *   ring_k_exp, ring_v_exp  i8  [n_layers][batch][n_groups][ring_slots rounded up to 16]
 *   bank_k_exp, bank_v_exp  i8  [n_layers][batch][n_groups][bank_slots rounded up to 16]
 *   pend_k_exp, pend_v_exp  i8  [n_layers][batch][n_groups][pend_slots rounded up to 16]
 * (entries past the slot count are padding); in a BF16 state their offsets are 0.
 * A caller may write the slot arrays and counters directly (to restore a
 * checkpoint or set up a test) while no call is in flight. */
typedef struct rma_layout {
    uint64_t total_bytes;
    uint64_t ring_k, ring_v, bank_k, bank_v, bank_score;
    uint64_t pend_k, pend_v, pend_score, counters, tickets, status;
    uint64_t ring_k_exp, ring_v_exp, bank_k_exp, bank_v_exp, pend_k_exp, pend_v_exp;
} rma_layout;

typedef struct rma_state rma_state;   /* opaque host handle; the device memory is the caller's */

/* Bytes of device memory the state needs for cfg, or 0 if cfg is invalid.
 * Independent of sequence length: the state has fixed capacity ([CARD]
 * "How Rock Memory Anchors work": O(1) persistent history). */
RMA_API size_t rma_state_bytes(const rma_config* cfg);

/* Lay the state out over dev_buf (device memory, 256-byte aligned, at least
 * rma_state_bytes(cfg) bytes, owned by the caller and kept alive until
 * rma_state_free) and zero its counters, tickets and status word on
 * `stream`.  Slot contents are left as they are.  Allocates no device memory.
 * On success *out receives a host handle. */
RMA_API int rma_state_alloc(const rma_config* cfg, void* dev_buf, size_t dev_bytes, void* stream, rma_state** out);

/* Copy the layout of st into *out. */
RMA_API int rma_state_layout(const rma_state* st, rma_layout* out);

/* Release the host handle (not the caller's device buffer).  NULL is a no-op. */
RMA_API void rma_state_free(rma_state* st);

/* Workspace (device scratch, 256-byte aligned) a call with n_tok tokens per
 * sequence needs: n_tok == 1 for rma_decode_step (the size also covers a
 * one-token prefill block), 1 <= n_tok <= 256 for rma_prefill_block.
 * RMA_ERR_INVALID_ARG for n_tok < 1, RMA_ERR_UNSUPPORTED above 256.  The
 * caller owns it; its contents need not be preserved between calls, but two
 * calls in flight at once need two workspaces. */
RMA_API int rma_workspace_bytes(const rma_state* st, int n_tok, size_t* out);

/* Decode split-K shape: the ring and the bank are each cut into this many
 * contiguous row ranges, one CTA per range.  0 for both restores the default
 * (chosen from batch size and SM count).  Affects speed only, not results
 * beyond FP32 summation order. */
RMA_API int rma_set_decode_splits(rma_state* st, int ring_splits, int bank_splits);

/* Let a decode call start loading its layer's ring and bank while the
 * previous kernel on the same stream is still finishing (0: off, the default;
 * 1: on).  Every decode launch may begin before the previous kernel in its
 * stream ends (programmatic dependent launch), but by default it touches no
 * global memory until that kernel has completed, which only hides the launch.
 * With overlap on, the counters are read and the first ring and bank tiles
 * requested before that point when the previous kernel is a decode call of
 * this library on another layer of this state (or on another state); the
 * library tracks this per stream (and per stream capture) and waits first
 * otherwise.  Inputs and the workspace are always read after the wait, and a
 * launch never overlaps more than the one before it.  The caller's side of
 * the contract: while overlap is on, no kernel other than this library's
 * writes the state between two decode calls on a stream (restoring a
 * checkpoint with cudaMemcpy is fine; with a kernel of one's own, synchronise
 * the stream first).  Affects speed only. */
RMA_API int rma_set_decode_overlap(rma_state* st, int enable);

/* One decode token for every sequence at RMA layer `layer`
 * ([PRIM] operations list, items 1-3; [CARD] "How Rock Memory Anchors work"):
 *   local_h  = softmax(scale q_h K^T) V over the window: ring slots holding
 *              positions [pos - min(pos, R), pos) plus the current token;
 *   anchor_h = the same over bank slots [0, bank_fill) (0 if bank_fill == 0);
 *   g_h      = tanh(q_h . w_g[h] + b_g[h]);   out_h = local_h + g_h anchor_h,
 * for every query head h, which reads KV group h / q_per_group.  Then, after
 * every read of the step: (k_cur, v_cur) go to ring slot pos mod R, pos += 1,
 * and (cand_k, cand_v, cand_score) are appended at pending slot pend_fill
 * (or dropped with RMA_STATUS_PENDING_OVERFLOW if pend_fill == P).
 * Pending records are never read.
 *   q          bf16 [batch][n_groups*q_per_group][head_dim]
 *   k_cur, v_cur, cand_k, cand_v   bf16 [batch][n_groups][head_dim]
 *   cand_score f32  [batch][n_groups]
 *   w_g        f32  [n_groups*q_per_group][head_dim]   (this layer's)
 *   b_g        f32  [n_groups*q_per_group]
 *   out        bf16 [batch][n_groups*q_per_group][head_dim]   (written)
 *   ws         workspace of rma_workspace_bytes(st, 1) bytes
 * When this step fills a group's pending buffer (pend_fill reaches P), the
 * admit of that (sequence, group) runs in the same launch, after every read
 * of the step, exactly as rma_admit would (so calling rma_admit afterwards
 * finds nothing to do); its records are visible from the next step on.
 * All pointers are device pointers; q, k_cur, v_cur, cand_k, cand_v, w_g and
 * out must be 16-byte aligned. */
RMA_API int rma_decode_step(rma_state* st, int layer,
                    const uint16_t* q, const uint16_t* k_cur, const uint16_t* v_cur,
                    const uint16_t* cand_k, const uint16_t* cand_v, const float* cand_score,
                    const float* w_g, const float* b_g, uint16_t* out,
                    void* ws, size_t ws_bytes, void* stream);

/* rma_decode_step without a caller-supplied workspace.  The pages have no
 * counterpart to this entry point; it exists for callers that cannot
 * allocate device memory when they call: for example a plug-in inside a host
 * framework that owns all device memory and hands out no scratch, a
 * real-time serving loop that forbids allocation after start-up, or an
 * embedded deployment that reserves its memory once.  Such a caller still
 * passes its inputs and outputs; the per-split partials go to a scratch
 * array built into the library (32 MiB per GPU, held on every GPU that loads
 * the library until the process exits).  The call allocates nothing.
 *   Limit: batch * n_groups * (ring_splits + bank_splits) * 4128 bytes must
 *   fit in 32 MiB (batch 512 with the default split shape needs 16.9 MB);
 *   larger calls return RMA_ERR_BUFFER_TOO_SMALL and launch nothing.
 *   Every call looks up the scratch's device address (cudaGetSymbolAddress)
 *   in the CUDA context current on the calling thread, so the address is
 *   never stale after a device reset or in a second context.  The first call
 *   on a device may load the library's device code there: make that first
 *   call before any stream capture.
 *   One scratch per GPU is shared by every call on it, and keeps whatever the
 *   last call left: calls that can overlap on the GPU (other streams, other
 *   states) race on it, so the caller must order them.  Nothing in it needs to
 *   start at zero: each partial is written before it is read.
 * Arguments, alignment and results are those of rma_decode_step. */
RMA_API int rma_decode_step_noalloc(rma_state* st, int layer,
                                    const uint16_t* q, const uint16_t* k_cur, const uint16_t* v_cur,
                                    const uint16_t* cand_k, const uint16_t* cand_v, const float* cand_score,
                                    const float* w_g, const float* b_g, uint16_t* out, void* stream);

/* Admit at RMA layer `layer` ([NEWS] "How it works": after every 256
 * candidates the existing anchors and the candidates compete and the top
 * 1,024 are kept, independently per KV group; [SITE] "Commit interval 256").
 * For each (sequence, group) with pend_fill == P (or, when force != 0, with
 * pend_fill > 0): the bank_fill committed records and pend_fill candidates
 * are ordered by score (higher first), then committed before candidate, then
 * lower slot (-0.0 equals +0.0; NaN below every number, and it sets
 * RMA_STATUS_NAN_SCORE); the first min(A, bank_fill + pend_fill) are kept.
 * Retained anchors stay in their slots, unchanged ([PRIM] item 3).  Admitted
 * candidates, in ascending pending slot, are copied (K, V and score,
 * bit-exact) into the vacated slots (evicted anchors' slots and empty slots)
 * in ascending order.  Then bank_fill = number kept, pend_fill = 0.
 * Other (sequence, group) pairs are untouched.  force must be 0 or 1. */
RMA_API int rma_admit(rma_state* st, int layer, int force, void* stream);

/* A prefill block of n_tok consecutive tokens per sequence at RMA layer
 * `layer` ([CARD] FAQ "How do Rock Memory Anchors preserve distant
 * information?": reads use the committed bank; updates take effect at the
 * next block).  With block start s = pos, query i (position s + i) attends
 * causally to positions [s + i - R, s + i] (ring slots for those below s, the
 * block's own k, v for the rest) and to bank slots [0, bank_fill) as
 * committed before the block; gate and output as in rma_decode_step.  Then,
 * after every read: ring slots (s + i) mod R take k, v of the block, pos +=
 * n_tok, the candidates are appended to pending (if pend_fill + n_tok <= P,
 * else dropped with RMA_STATUS_PREFILL_PENDING_OVERFLOW), and the admit runs
 * forced (as rma_admit with force = 1).
 *   q           bf16 [batch][n_tok][n_groups*q_per_group][head_dim]
 *   k, v, cand_k, cand_v   bf16 [batch][n_tok][n_groups][head_dim]
 *   cand_score  f32  [batch][n_tok][n_groups]
 *   w_g, b_g    as in rma_decode_step
 *   out         bf16 [batch][n_tok][n_groups*q_per_group][head_dim]  (written)
 *   ws          workspace of rma_workspace_bytes(st, n_tok) bytes
 * Three launches on the stream: the attention (persistent, over work items of
 * 64 tokens x one group x local window or bank), the commit (gate, combine,
 * ring write, pending append, the admit's competition) and the copy of the
 * admitted rows into the bank; the second and third may begin while the one
 * before them finishes, and touch nothing it still reads.  The workspace holds
 * the normalised local and anchor rows, 2 x batch x n_tok x n_groups x
 * q_per_group x head_dim FP32, and the admit's lists.
 * n_tok is any length from 1 (RMA_ERR_INVALID_ARG below) to 256 and at most
 * ring_slots (RMA_ERR_UNSUPPORTED above): a prompt whose length is not a
 * multiple of pend_slots ends in a shorter block, and a block may follow
 * decode steps (pend_fill != 0 at its start).  Alignment as in
 * rma_decode_step. */
RMA_API int rma_prefill_block(rma_state* st, int layer, int n_tok,
                      const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      const uint16_t* cand_k, const uint16_t* cand_v, const float* cand_score,
                      const float* w_g, const float* b_g, uint16_t* out,
                      void* ws, size_t ws_bytes, void* stream);

/* Quantise every row of the BF16 state `src` into the RMA_KV_FP8_E4M3 state
 * `dst` (same dimensions), as rma_config's kv_format describes, and copy the
 * scores and counters: the way to decode in FP8 after a BF16 prefill.  Every
 * slot is converted, filled or not.  Both states stay the caller's; they must
 * not overlap.  RMA_ERR_INVALID_ARG if the formats or dimensions do not match. */
RMA_API int rma_state_quantize(rma_state* dst, const rma_state* src, void* stream);

/* Wait for `stream`, then read the device status word into *flags and clear it. */
RMA_API int rma_get_status(rma_state* st, void* stream, uint32_t* flags);

/* Text for a return code. */
RMA_API const char* rma_strerror(int code);

/* One line describing the most recent error returned on this host thread ("" if none). */
RMA_API const char* rma_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* RMA_H */
