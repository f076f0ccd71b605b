"""CPU oracle for the Rock Memory Anchors (RMA) attention hot path.

TEST INFRASTRUCTURE.  This module exists to check the CUDA library.  Only the
test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference (``--impl reference``) legs may import it.  The product path (the C-ABI library and its
Python binding) never calls it and has no CPU fallback.

It is a plain, slow, step-by-step restatement of what the pages say the RMA
layer computes.  It shares no code with the CUDA path: its BF16 conversions,
softmax, gate and admit ordering are written here from the pages' statement
of the method.  Arithmetic is FP64 on values expanded exactly from their BF16
or FP32 storage; outputs are rounded once to BF16 (round to nearest even).

Pages cited (by title):
  [NEWS]  "EdgeRock-4B holds KV cache at 72 MiB up to 256K context, with 12,124
          tokens/s on one 80GB GPU" (tpsreport.news)
  [PRIM]  "EdgeRock-4B fixes its attention KV cache at 72 MiB" (ai-primer.com)
  [CARD]  "EdgeRock" model card (modelscope.cn/models/rockmatrix/EdgeRock)
  [SITE]  "Models / EdgeRock-4B" product page (rockmatrix.ai/models)

Per (sequence, layer, KV group) the state is three fixed-capacity stores
([CARD] "How Rock Memory Anchors work", history-component table;
[PRIM] persistent-history table):
  ring    R = 1023 slots of (K, V): the preceding positions of the local window;
          the decoder supplies the current token as the 1024th position.
  bank    A = 1024 committed anchor records (K, V, score).
  pending P = 256 candidate records (K, V, score) waiting for the next admit.
plus counters pos (tokens seen), bank_fill, pend_fill.

Readings taken where the pages are silent (each one is also listed in the
repository's design notes):
  * position p lives in ring slot p mod R;
  * query head h reads KV group h // H (consecutive heads share a group);
  * gate g_h = tanh(q_h . w_g[h] + b_g[h]); out_h = local_h + g_h * anchor_h;
  * an empty bank gives anchor = 0; pending records are never read;
  * admit order: higher score first, then committed before candidate, then
    lower slot; -0.0 equals +0.0; a NaN score ranks below every number and
    raises STATUS_NAN_SCORE;
  * admitted candidates, in ascending pending slot, fill the vacated bank slots
    (evicted committed slots and empty slots) in ascending order; retained
    records do not move;
  * a retained anchor keeps its stored score (no re-scoring);
  * a decode step that finds the pending buffer full drops its candidate and
    raises STATUS_PENDING_OVERFLOW; a prefill block whose candidates do not fit
    drops them and raises STATUS_PREFILL_PENDING_OVERFLOW;
  * a prefill block may hold any number n of tokens (the last block of a prompt
    whose length is not a multiple of 256 is shorter); it appends after the
    candidates still pending and always ends with the forced admit;
  * Q and K arrive already position-encoded (no RoPE inside the layer).

Parity pins: every function here is checked by ``tests/test_oracle_*.py``
against what the pages and the mathematics fix (printed byte counts, brute
force masked attention over the full history, closed forms, admit order
properties checked pair by pair, visibility).  No function is unpinned.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

# Device status bits (readings above; the CUDA library defines the same meanings).
STATUS_PENDING_OVERFLOW = 1
STATUS_NAN_SCORE = 2
STATUS_PREFILL_PENDING_OVERFLOW = 4


# ---------------------------------------------------------------------------
# BF16 storage <-> FP64 arithmetic
# ---------------------------------------------------------------------------

def bf16_to_f64(bits) -> np.ndarray:
    """Expand BF16 bit patterns (uint16) exactly: a BF16 value is the top half of an FP32."""
    b = np.asarray(bits, dtype=np.uint16)
    with np.errstate(invalid="ignore"):     # NaN patterns stay NaN
        return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f64_to_bf16(x) -> np.ndarray:
    """Round FP64 values to BF16 (8 significant bits), ties to even, in one step.

    x = m * 2**e with 0.5 <= |m| < 1; m * 256 is exact, np.round rounds half to
    even, so the result is the correctly rounded BF16 value.  Valid for the
    normal BF16 range, which is all this layer produces (values below 2**-126
    in magnitude are flushed to zero here).
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    r = np.ldexp(np.round(m * 256.0) / 256.0, e)
    r = np.where(np.abs(r) < 2.0 ** -126, 0.0 * r, r)
    return (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def f32_to_bf16(x) -> np.ndarray:
    """Round FP32 values to BF16 by the same rule (used to build inputs in tests)."""
    return f64_to_bf16(np.asarray(x, dtype=np.float32).astype(np.float64))


# ---------------------------------------------------------------------------
# Configuration and state
# ---------------------------------------------------------------------------

@dataclass
class Config:
    """Dimensions of the RMA state.

    Defaults are the ones the pages fix: 4 KV groups, a 1,023 + 1 position
    window, 1,024 anchors per group, 256 pending candidates ([CARD] history
    table; [SITE] "02 / Architecture" spec list), and head_dim 256 with 4 query
    heads per group (the per-token KV size of the source model, [NEWS]
    "Throughput and memory": 32 KiB per token over 8 layers and 4 KV heads).
    Tests use smaller R, A, P to reach many wrap-arounds and admits quickly.
    """
    batch: int = 1
    n_layers: int = 1
    n_groups: int = 4
    q_per_group: int = 4
    head_dim: int = 256
    ring_slots: int = 1023
    bank_slots: int = 1024
    pend_slots: int = 256
    softmax_scale: float = 1.0 / 16.0

    @property
    def n_q_heads(self) -> int:
        return self.n_groups * self.q_per_group


@dataclass
class State:
    cfg: Config
    ring_k: np.ndarray      # uint16 [L,B,G,R,D]
    ring_v: np.ndarray
    bank_k: np.ndarray      # uint16 [L,B,G,A,D]
    bank_v: np.ndarray
    bank_score: np.ndarray  # float32 [L,B,G,A]
    pend_k: np.ndarray      # uint16 [L,B,G,P,D]
    pend_v: np.ndarray
    pend_score: np.ndarray  # float32 [L,B,G,P]
    pos: np.ndarray         # int64 [L,B,G]
    bank_fill: np.ndarray   # int64 [L,B,G]
    pend_fill: np.ndarray   # int64 [L,B,G]
    status: int = 0


def new_state(cfg: Config) -> State:
    """An empty state: every slot zero, every counter zero."""
    L, B, G, D = cfg.n_layers, cfg.batch, cfg.n_groups, cfg.head_dim
    R, A, P = cfg.ring_slots, cfg.bank_slots, cfg.pend_slots
    z16 = lambda *s: np.zeros(s, dtype=np.uint16)
    return State(cfg=cfg,
                 ring_k=z16(L, B, G, R, D), ring_v=z16(L, B, G, R, D),
                 bank_k=z16(L, B, G, A, D), bank_v=z16(L, B, G, A, D),
                 bank_score=np.zeros((L, B, G, A), np.float32),
                 pend_k=z16(L, B, G, P, D), pend_v=z16(L, B, G, P, D),
                 pend_score=np.zeros((L, B, G, P), np.float32),
                 pos=np.zeros((L, B, G), np.int64),
                 bank_fill=np.zeros((L, B, G), np.int64),
                 pend_fill=np.zeros((L, B, G), np.int64))


def state_from_arrays(cfg: Config, arrays: dict, pos, bank_fill, pend_fill) -> State:
    """A state whose slot bytes are ``arrays`` (numpy, storage dtypes) and whose counters are given.

    ``pos``, ``bank_fill`` and ``pend_fill`` broadcast to [L, B, G].
    """
    st = new_state(cfg)
    for name in ("ring_k", "ring_v", "bank_k", "bank_v", "pend_k", "pend_v"):
        getattr(st, name)[...] = np.asarray(arrays[name]).view(np.uint16)
    st.bank_score[...] = np.asarray(arrays["bank_score"], dtype=np.float32)
    st.pend_score[...] = np.asarray(arrays["pend_score"], dtype=np.float32)
    shape = st.pos.shape
    st.pos[...] = np.broadcast_to(np.asarray(pos, dtype=np.int64), shape)
    st.bank_fill[...] = np.broadcast_to(np.asarray(bank_fill, dtype=np.int64), shape)
    st.pend_fill[...] = np.broadcast_to(np.asarray(pend_fill, dtype=np.int64), shape)
    return st


def copy_state(st: State) -> State:
    return State(cfg=st.cfg, **{k: getattr(st, k).copy() for k in (
        "ring_k", "ring_v", "bank_k", "bank_v", "bank_score", "pend_k", "pend_v",
        "pend_score", "pos", "bank_fill", "pend_fill")}, status=st.status)


# ---------------------------------------------------------------------------
# Memory accounting ([PRIM] persistent-history table; [CARD] "Constant history
# and GPU memory"; [SITE] "BF16 attention KV 72 MiB per sequence")
# ---------------------------------------------------------------------------

def attention_kv_bytes_per_sequence(n_layers=8, n_groups=4, head_dim=256, ring_slots=1023,
                                    bank_slots=1024, pend_slots=256, elem_bytes=2) -> dict:
    """Bytes of K/V storage per sequence, by component.

    One record is one K row plus one V row of head_dim elements; each
    component holds its slot count of records per (layer, KV group).
    """
    record = 2 * head_dim * elem_bytes
    per_group_layer = n_layers * n_groups * record
    return {
        "committed_anchors": bank_slots * per_group_layer,
        "pending_candidates": pend_slots * per_group_layer,
        "local_window": ring_slots * per_group_layer,
    }


def full_attention_kv_bytes_per_token(n_layers=8, n_kv_heads=4, head_dim=256, elem_bytes=2) -> int:
    """K and V of one token over every full-attention layer of the source model ([NEWS])."""
    return n_layers * n_kv_heads * head_dim * 2 * elem_bytes


# ---------------------------------------------------------------------------
# Retrieve: two softmax attentions and the signed gate ([PRIM] operations
# list, item 3 "Retrieve"; [CARD] "How Rock Memory Anchors work")
# ---------------------------------------------------------------------------

def _attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * K q)^T V for one query, in two passes: the maximum, then the exponentials."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    logits = scale * (K @ q)
    w = np.exp(logits - logits.max())
    return (w @ V) / w.sum()


def _gate(q: np.ndarray, w_g_row: np.ndarray, b_g: float) -> float:
    return math.tanh(float(q @ np.asarray(w_g_row, dtype=np.float64)) + float(b_g))


def decode_step(st: State, layer: int, q, k_cur, v_cur, cand_k, cand_v, cand_score,
                w_g, b_g, return_f64: bool = False):
    """One decode token for every sequence at one RMA layer.

    Inputs (storage dtypes): q [B, G*H, D] bf16 bits; k_cur, v_cur, cand_k,
    cand_v [B, G, D] bf16 bits; cand_score [B, G] f32; w_g [G*H, D] f32;
    b_g [G*H] f32.  Returns out [B, G*H, D] as bf16 bits (and the unrounded
    FP64 values when ``return_f64``).

    Reads first, writes after ([CARD] FAQ "How do Rock Memory Anchors preserve
    distant information?": reads use the committed bank):
      local  = attention over the window: ring positions [pos - min(pos, R), pos)
               plus the current token ([PRIM]: the ring stores the 1,023
               preceding positions and the decoder supplies the current token);
      anchor = attention over bank slots [0, bank_fill);
      out    = local + tanh(q . w_g + b_g) * anchor.
    Then the current token's K/V go to ring slot pos mod R, pos advances, and
    the candidate record is appended to pending ([PRIM] item 1 "Write").
    """
    cfg = st.cfg
    B, G, H, D, R, P = cfg.batch, cfg.n_groups, cfg.q_per_group, cfg.head_dim, cfg.ring_slots, cfg.pend_slots
    q = np.asarray(q).view(np.uint16)
    out = np.zeros((B, G * H, D), dtype=np.float64)
    for b in range(B):
        for g in range(G):
            pos = int(st.pos[layer, b, g])
            n_prev = min(pos, R)
            prev_positions = np.arange(pos - n_prev, pos)
            slots = prev_positions % R
            K_loc = np.concatenate([bf16_to_f64(st.ring_k[layer, b, g][slots]),
                                    bf16_to_f64(np.asarray(k_cur).view(np.uint16)[b, g])[None, :]])
            V_loc = np.concatenate([bf16_to_f64(st.ring_v[layer, b, g][slots]),
                                    bf16_to_f64(np.asarray(v_cur).view(np.uint16)[b, g])[None, :]])
            nb = int(st.bank_fill[layer, b, g])
            K_anc = bf16_to_f64(st.bank_k[layer, b, g, :nb])
            V_anc = bf16_to_f64(st.bank_v[layer, b, g, :nb])
            for h in range(H):
                head = g * H + h
                qh = bf16_to_f64(q[b, head])
                local = _attend(qh, K_loc, V_loc, cfg.softmax_scale)
                anchor = _attend(qh, K_anc, V_anc, cfg.softmax_scale)
                gate = _gate(qh, np.asarray(w_g)[head], np.asarray(b_g)[head])
                out[b, head] = local + gate * anchor
    # Writes, after every read of this step.
    for b in range(B):
        for g in range(G):
            pos = int(st.pos[layer, b, g])
            st.ring_k[layer, b, g, pos % R] = np.asarray(k_cur).view(np.uint16)[b, g]
            st.ring_v[layer, b, g, pos % R] = np.asarray(v_cur).view(np.uint16)[b, g]
            st.pos[layer, b, g] = pos + 1
            pf = int(st.pend_fill[layer, b, g])
            if pf < P:
                st.pend_k[layer, b, g, pf] = np.asarray(cand_k).view(np.uint16)[b, g]
                st.pend_v[layer, b, g, pf] = np.asarray(cand_v).view(np.uint16)[b, g]
                st.pend_score[layer, b, g, pf] = np.asarray(cand_score, dtype=np.float32)[b, g]
                st.pend_fill[layer, b, g] = pf + 1
            else:
                st.status |= STATUS_PENDING_OVERFLOW
    bits = f64_to_bf16(out)
    return (bits, out) if return_f64 else bits


# ---------------------------------------------------------------------------
# Admit ([NEWS] "How it works": after every 256 candidates, compare with the
# existing anchors and keep the top 1,024, independently per KV group;
# [PRIM] item 2 "Admit"; [SITE] "Commit interval 256 tokens")
# ---------------------------------------------------------------------------

def _rank_key(score: float, is_candidate: int, slot: int):
    """Sort key for the admit order: smaller key = kept first.

    NaN sorts after every number; -score makes higher scores come first
    (and -(+0.0) == -(-0.0) compares equal, so signed zeros tie); committed
    records (0) come before candidates (1); then the lower slot.
    """
    if math.isnan(score):
        return (1, 0.0, is_candidate, slot)
    return (0, -score, is_candidate, slot)


def admit_plan(bank_scores, pend_scores, A: int):
    """The competition of one (sequence, layer, KV group), on scores alone.

    bank_scores: the nb committed anchors' scores (slots 0 .. nb-1); pend_scores:
    the candidates' (pending slots 0 .. npend-1).  The top min(A, nb + npend)
    records by the admit order are kept.  Returns (kept count, moves, nan_seen):
    moves pairs each admitted candidate, in ascending pending slot, with a
    vacated bank slot (evicted committed slots and empty slots) in ascending
    order, as (bank slot, pending slot).
    """
    nb, npend = len(bank_scores), len(pend_scores)
    records = ([(float(bank_scores[s]), 0, s) for s in range(nb)] +
               [(float(pend_scores[t]), 1, t) for t in range(npend)])
    nan_seen = any(math.isnan(r[0]) for r in records)
    order = sorted(records, key=lambda r: _rank_key(*r))
    kept = order[:min(A, len(records))]
    kept_committed = {slot for (_, kind, slot) in kept if kind == 0}
    admitted = sorted(slot for (_, kind, slot) in kept if kind == 1)
    vacated = [s for s in range(nb) if s not in kept_committed] + list(range(nb, A))
    return len(kept), list(zip(vacated, admitted)), nan_seen


def admit(st: State, layer: int, force: bool = False) -> None:
    """Per (sequence, KV group): committed anchors compete with pending candidates.

    Runs when pend_fill == P, or when ``force`` and pend_fill > 0.  The top
    min(A, bank_fill + pend_fill) records by the admit order are kept.
    Retained anchors stay in their slots, unchanged ([PRIM] item 3; [CARD]
    "Retained records remain separate and unchanged").  The admitted
    candidates, in ascending pending slot, fill the vacated slots in ascending
    order (``admit_plan``).  Afterwards bank_fill = number kept and pend_fill = 0.
    """
    cfg = st.cfg
    A, P = cfg.bank_slots, cfg.pend_slots
    for b in range(cfg.batch):
        for g in range(cfg.n_groups):
            nb = int(st.bank_fill[layer, b, g])
            npend = int(st.pend_fill[layer, b, g])
            if not (npend == P or (force and npend > 0)):
                continue
            kept, moves, nan_seen = admit_plan(st.bank_score[layer, b, g, :nb], st.pend_score[layer, b, g, :npend], A)
            if nan_seen:
                st.status |= STATUS_NAN_SCORE
            for dst, src in moves:
                st.bank_k[layer, b, g, dst] = st.pend_k[layer, b, g, src]
                st.bank_v[layer, b, g, dst] = st.pend_v[layer, b, g, src]
                st.bank_score[layer, b, g, dst] = st.pend_score[layer, b, g, src]
            st.bank_fill[layer, b, g] = kept
            st.pend_fill[layer, b, g] = 0


# ---------------------------------------------------------------------------
# Block prefill ([CARD] FAQ: "reads use the committed bank; updates take effect
# at the next block")
# ---------------------------------------------------------------------------

def prefill_block(st: State, layer: int, q, k, v, cand_k, cand_v, cand_score, w_g, b_g,
                  return_f64: bool = False):
    """A block of n consecutive tokens for every sequence at one RMA layer.

    Inputs: q [B, n, G*H, D]; k, v, cand_k, cand_v [B, n, G, D] bf16 bits;
    cand_score [B, n, G] f32; w_g [G*H, D]; b_g [G*H].  Returns out
    [B, n, G*H, D] bf16 bits.

    Block start s = pos.  Query i (position s+i) attends causally to positions
    [s+i-R, s+i]: those below s come from the ring, the rest are the block's
    own keys.  Every query reads the bank as committed before the block.
    After all reads: ring writes of the n positions, pos += n, the block's
    candidates are appended to pending (if they fit), and admit runs forced.
    """
    cfg = st.cfg
    B, G, H, D, R, P = cfg.batch, cfg.n_groups, cfg.q_per_group, cfg.head_dim, cfg.ring_slots, cfg.pend_slots
    q = np.asarray(q).view(np.uint16)
    k = np.asarray(k).view(np.uint16)
    v = np.asarray(v).view(np.uint16)
    n = q.shape[1]
    out = np.zeros((B, n, G * H, D), dtype=np.float64)
    for b in range(B):
        for g in range(G):
            s = int(st.pos[layer, b, g])
            n_prev = min(s, R)
            hist_pos = np.arange(s - n_prev, s + n)
            ring_slots = hist_pos[:n_prev] % R
            K_hist = np.concatenate([bf16_to_f64(st.ring_k[layer, b, g][ring_slots]), bf16_to_f64(k[b, :, g])])
            V_hist = np.concatenate([bf16_to_f64(st.ring_v[layer, b, g][ring_slots]), bf16_to_f64(v[b, :, g])])
            qpos = s + np.arange(n)
            visible = (hist_pos[None, :] <= qpos[:, None]) & (hist_pos[None, :] >= qpos[:, None] - R)
            nb = int(st.bank_fill[layer, b, g])
            K_anc = bf16_to_f64(st.bank_k[layer, b, g, :nb])
            V_anc = bf16_to_f64(st.bank_v[layer, b, g, :nb])
            for h in range(H):
                head = g * H + h
                Qh = bf16_to_f64(q[b, :, head])                       # [n, D]
                logits = np.where(visible, cfg.softmax_scale * (Qh @ K_hist.T), -np.inf)
                w = np.exp(logits - logits.max(axis=1, keepdims=True))
                local = (w @ V_hist) / w.sum(axis=1, keepdims=True)
                if nb > 0:
                    la = cfg.softmax_scale * (Qh @ K_anc.T)
                    wa = np.exp(la - la.max(axis=1, keepdims=True))
                    anchor = (wa @ V_anc) / wa.sum(axis=1, keepdims=True)
                else:
                    anchor = np.zeros((n, D))
                gate = np.tanh(Qh @ np.asarray(w_g, dtype=np.float64)[head] + float(np.asarray(b_g)[head]))
                out[b, :, head] = local + gate[:, None] * anchor
    for b in range(B):
        for g in range(G):
            s = int(st.pos[layer, b, g])
            for i in range(n):
                st.ring_k[layer, b, g, (s + i) % R] = k[b, i, g]
                st.ring_v[layer, b, g, (s + i) % R] = v[b, i, g]
            st.pos[layer, b, g] = s + n
            pf = int(st.pend_fill[layer, b, g])
            if pf + n <= P:
                st.pend_k[layer, b, g, pf:pf + n] = np.asarray(cand_k).view(np.uint16)[b, :, g]
                st.pend_v[layer, b, g, pf:pf + n] = np.asarray(cand_v).view(np.uint16)[b, :, g]
                st.pend_score[layer, b, g, pf:pf + n] = np.asarray(cand_score, dtype=np.float32)[b, :, g]
                st.pend_fill[layer, b, g] = pf + n
            else:
                st.status |= STATUS_PREFILL_PENDING_OVERFLOW
    admit(st, layer, force=True)
    bits = f64_to_bf16(out)
    return (bits, out) if return_f64 else bits
