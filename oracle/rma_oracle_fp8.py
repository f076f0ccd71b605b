"""CPU oracle for RMA state stored in FP8: ring, bank and pending K/V as E4M3 codes.

TEST INFRASTRUCTURE, like ``rma_oracle``: only the test suite, ``__graft_entry__``
and ``bench.py``'s CPU legs may import it; the CUDA library never calls it.

The pages list FP8 and INT8 packages of the model, validated for text inference
("EdgeRock-4B fixes its attention KV cache at 72 MiB" (ai-primer.com), packages
paragraph; "Models / EdgeRock-4B" (rockmatrix.ai), downloads list).  They do
not say how K/V would be stored in FP8, so this module takes the plainest
storage that keeps every copy exact:

  * every stored row (one position's K, or its V, for one KV group: head_dim
    values) is kept as head_dim E4M3 codes plus one power-of-two scale 2**e,
    e a signed 8-bit integer;
  * e is the smallest integer in [-127, 127] with amax(|row|) <= 448 * 2**e
    (0 for an all-zero row), so row * 2**-e is exact in FP32 and lies in
    [-448, 448]; the only rounding is the E4M3 one (to nearest, ties to even),
    and a stored value is code * 2**e;
  * rows are quantised when written (the ring write of the current token, the
    candidate append, and the conversion of a BF16 state); the admit copies
    codes, scale exponents and scores unchanged;
  * attention reads the dequantised rows; the current token is attended at the
    precision it arrives in (BF16) and stored quantised afterwards, and Q stays
    BF16.  Everything else is ``rma_oracle``'s decode step and admit.

E4M3 here is the variant without infinities: 1 sign bit, 4 exponent bits
(bias 7), 3 mantissa bits; exponent field 0 holds the subnormals m * 2**-9;
S.1111.111 is NaN; the largest finite value is 448 = 1.75 * 2**8.

Pins: ``tests/test_oracle_fp8.py`` checks the code table and the rounding
against torch's float8_e4m3fn conversion (all 256 codes; every BF16 value in
range and every tie between neighbouring codes), the scale's minimality, the
round-trip bound, a decode step against brute-force attention over the
dequantised history, and the equality of the FP8 and BF16 oracles on rows that
E4M3 represents exactly.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

from .rma_oracle import (Config, STATUS_NAN_SCORE, STATUS_PENDING_OVERFLOW, State, _attend, _gate, admit_plan,
                         bf16_to_f64, f64_to_bf16)

E4M3_MAX = 448.0


def e4m3_to_f64(codes) -> np.ndarray:
    """Decode E4M3 codes (uint8) from the format's definition."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = np.ldexp(m / 8.0, -6)
    v = np.where(e == 0, sub, normal)
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return sign * v


def _e4m3_grid() -> np.ndarray:
    """The non-negative finite E4M3 values in increasing order, with their codes."""
    codes = np.arange(0, 0x7F, dtype=np.uint8)          # 0x00 .. 0x7E
    return e4m3_to_f64(codes), codes


def f32_to_e4m3(x) -> np.ndarray:
    """Round values (FP32, |x| <= 448) to the nearest E4M3 code, ties to the even code.

    The grid of non-negative finite values is enumerated from the definition;
    the two neighbours of |x| are found and the nearer is taken (on a tie, the
    one whose mantissa is even, i.e. whose code is even).  -0.0 and negative
    values that round to zero keep their sign bit.  NaN maps to 0x7F.
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    if np.any(np.abs(x[~np.isnan(x)]) > E4M3_MAX):
        raise ValueError("f32_to_e4m3 takes |x| <= 448 (rows are scaled into range first)")
    vals, codes = _e4m3_grid()
    a = np.abs(x)
    hi = np.searchsorted(vals, np.nan_to_num(a), side="left")       # first grid value >= a
    hi = np.clip(hi, 0, len(vals) - 1)
    lo = np.clip(hi - 1, 0, len(vals) - 1)
    d_hi = vals[hi] - a
    d_lo = a - vals[lo]
    take_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (codes[lo] % 2 == 0))
    take_lo &= vals[lo] <= a
    mag = np.where(take_lo, codes[lo], codes[hi]).astype(np.uint8)
    signbit = np.signbit(x)
    out = np.where(signbit, mag | np.uint8(0x80), mag).astype(np.uint8)
    return np.where(np.isnan(x), np.uint8(0x7F), out).astype(np.uint8)


def row_exponent(amax) -> np.ndarray:
    """Smallest e in [-127, 127] with amax <= 448 * 2**e, per element (0 where amax == 0).

    Write amax = m * 2**x with 0.5 <= m < 1 (exact, frexp) and 448 = 0.875 * 2**9:
    amax <= 448 * 2**e  <=>  m * 2**x <= 0.875 * 2**(9 + e), which holds for
    e >= x - 9 when m <= 0.875 and for e >= x - 8 otherwise.
    """
    a = np.asarray(amax, dtype=np.float64)
    m, x = np.frexp(a)
    e = x.astype(np.int64) - 9 + (m > 0.875)
    e = np.clip(e, -127, 127)
    return np.where(a == 0.0, 0, e).astype(np.int64)


def quantize_rows(rows_bf16):
    """Quantise BF16 rows (uint16 bits, [..., D]) to (codes uint8 [..., D], exponents int8 [...])."""
    x = bf16_to_f64(np.asarray(rows_bf16).view(np.uint16))
    e = row_exponent(np.max(np.abs(x), axis=-1)) if x.shape[-1] else np.zeros(x.shape[:-1], np.int64)
    # x * 2**-e: a power-of-two scaling, exact in FP32 (values of a BF16 row never leave its range)
    scaled = (x.astype(np.float32) * np.ldexp(np.float32(1.0), (-e)[..., None]).astype(np.float32)).astype(np.float32)
    return f32_to_e4m3(scaled), e.astype(np.int8)


def dequantize_rows(codes, exps) -> np.ndarray:
    """code * 2**e for every element (FP64, exact)."""
    c = e4m3_to_f64(codes)
    return c * np.ldexp(1.0, np.asarray(exps, dtype=np.int64))[..., None]


# ---------------------------------------------------------------------------
# State and the decode step / admit on FP8 storage
# ---------------------------------------------------------------------------

_ROWS = ("ring_k", "ring_v", "bank_k", "bank_v", "pend_k", "pend_v")


@dataclass
class Fp8State:
    cfg: Config
    ring_k: np.ndarray      # uint8 [L,B,G,R,D] E4M3 codes
    ring_v: np.ndarray
    bank_k: np.ndarray      # uint8 [L,B,G,A,D]
    bank_v: np.ndarray
    pend_k: np.ndarray      # uint8 [L,B,G,P,D]
    pend_v: np.ndarray
    ring_k_exp: np.ndarray  # int8 [L,B,G,R] scale exponents
    ring_v_exp: np.ndarray
    bank_k_exp: np.ndarray  # int8 [L,B,G,A]
    bank_v_exp: np.ndarray
    pend_k_exp: np.ndarray  # int8 [L,B,G,P]
    pend_v_exp: np.ndarray
    bank_score: np.ndarray  # float32 [L,B,G,A]
    pend_score: np.ndarray  # float32 [L,B,G,P]
    pos: np.ndarray         # int64 [L,B,G]
    bank_fill: np.ndarray
    pend_fill: np.ndarray
    status: int = 0


def quantize_state(st: State) -> Fp8State:
    """The FP8 state holding every row of a BF16 state quantised (scores and counters copied)."""
    kw = {}
    for name in _ROWS:
        codes, exps = quantize_rows(getattr(st, name))
        kw[name], kw[name + "_exp"] = codes, exps
    return Fp8State(cfg=st.cfg, bank_score=st.bank_score.copy(), pend_score=st.pend_score.copy(),
                    pos=st.pos.copy(), bank_fill=st.bank_fill.copy(), pend_fill=st.pend_fill.copy(),
                    status=st.status, **kw)


def fp8_state_from_arrays(cfg: Config, arrays: dict, pos, bank_fill, pend_fill) -> Fp8State:
    """An FP8 state whose codes, exponents and scores are ``arrays``; counters broadcast to [L, B, G]."""
    kw = {}
    for name in _ROWS:
        kw[name] = np.array(arrays[name], dtype=np.uint8)
        kw[name + "_exp"] = np.array(arrays[name + "_exp"], dtype=np.int8)
    shape = kw["ring_k_exp"].shape[:3]
    return Fp8State(cfg=cfg, bank_score=np.array(arrays["bank_score"], dtype=np.float32),
                    pend_score=np.array(arrays["pend_score"], dtype=np.float32),
                    pos=np.broadcast_to(np.asarray(pos, dtype=np.int64), shape).copy(),
                    bank_fill=np.broadcast_to(np.asarray(bank_fill, dtype=np.int64), shape).copy(),
                    pend_fill=np.broadcast_to(np.asarray(pend_fill, dtype=np.int64), shape).copy(), **kw)


def decode_step_fp8(st: Fp8State, layer: int, q, k_cur, v_cur, cand_k, cand_v, cand_score, w_g, b_g,
                    return_f64: bool = False):
    """``rma_oracle.decode_step`` on FP8 storage: the window's and the bank's rows are read
    dequantised, the current token as given; then k_cur / v_cur are quantised into ring slot
    pos mod R and the candidate is quantised into pending."""
    cfg = st.cfg
    B, G, H, D, R, P = cfg.batch, cfg.n_groups, cfg.q_per_group, cfg.head_dim, cfg.ring_slots, cfg.pend_slots
    q = np.asarray(q).view(np.uint16)
    kc = np.asarray(k_cur).view(np.uint16)
    vc = np.asarray(v_cur).view(np.uint16)
    out = np.zeros((B, G * H, D), dtype=np.float64)
    for b in range(B):
        for g in range(G):
            pos = int(st.pos[layer, b, g])
            n_prev = min(pos, R)
            slots = np.arange(pos - n_prev, pos) % R
            K_loc = np.concatenate([dequantize_rows(st.ring_k[layer, b, g][slots], st.ring_k_exp[layer, b, g][slots]),
                                    bf16_to_f64(kc[b, g])[None, :]])
            V_loc = np.concatenate([dequantize_rows(st.ring_v[layer, b, g][slots], st.ring_v_exp[layer, b, g][slots]),
                                    bf16_to_f64(vc[b, g])[None, :]])
            nb = int(st.bank_fill[layer, b, g])
            K_anc = dequantize_rows(st.bank_k[layer, b, g, :nb], st.bank_k_exp[layer, b, g, :nb])
            V_anc = dequantize_rows(st.bank_v[layer, b, g, :nb], st.bank_v_exp[layer, b, g, :nb])
            for h in range(H):
                head = g * H + h
                qh = bf16_to_f64(q[b, head])
                local = _attend(qh, K_loc, V_loc, cfg.softmax_scale)
                anchor = _attend(qh, K_anc, V_anc, cfg.softmax_scale)
                gate = _gate(qh, np.asarray(w_g)[head], np.asarray(b_g)[head])
                out[b, head] = local + gate * anchor
    # writes, after every read of the step
    kq, ke = quantize_rows(kc)
    vq, ve = quantize_rows(vc)
    ckq, cke = quantize_rows(np.asarray(cand_k).view(np.uint16))
    cvq, cve = quantize_rows(np.asarray(cand_v).view(np.uint16))
    for b in range(B):
        for g in range(G):
            pos = int(st.pos[layer, b, g])
            st.ring_k[layer, b, g, pos % R], st.ring_k_exp[layer, b, g, pos % R] = kq[b, g], ke[b, g]
            st.ring_v[layer, b, g, pos % R], st.ring_v_exp[layer, b, g, pos % R] = vq[b, g], ve[b, g]
            st.pos[layer, b, g] = pos + 1
            pf = int(st.pend_fill[layer, b, g])
            if pf < P:
                st.pend_k[layer, b, g, pf], st.pend_k_exp[layer, b, g, pf] = ckq[b, g], cke[b, g]
                st.pend_v[layer, b, g, pf], st.pend_v_exp[layer, b, g, pf] = cvq[b, g], cve[b, g]
                st.pend_score[layer, b, g, pf] = np.asarray(cand_score, dtype=np.float32)[b, g]
                st.pend_fill[layer, b, g] = pf + 1
            else:
                st.status |= STATUS_PENDING_OVERFLOW
    bits = f64_to_bf16(out)
    return (bits, out) if return_f64 else bits


def admit_fp8(st: Fp8State, layer: int, force: bool = False) -> None:
    """``rma_oracle.admit`` on FP8 storage: the same competition (scores only); the admitted
    candidates' codes, scale exponents and scores are copied into the vacated bank slots."""
    cfg = st.cfg
    for b in range(cfg.batch):
        for g in range(cfg.n_groups):
            nb = int(st.bank_fill[layer, b, g])
            npend = int(st.pend_fill[layer, b, g])
            if not (npend == cfg.pend_slots or (force and npend > 0)):
                continue
            kept, moves, nan_seen = admit_plan(st.bank_score[layer, b, g, :nb], st.pend_score[layer, b, g, :npend],
                                               cfg.bank_slots)
            if nan_seen:
                st.status |= STATUS_NAN_SCORE
            for dst, src in moves:
                for name in ("k", "v"):
                    getattr(st, f"bank_{name}")[layer, b, g, dst] = getattr(st, f"pend_{name}")[layer, b, g, src]
                    getattr(st, f"bank_{name}_exp")[layer, b, g, dst] = getattr(st, f"pend_{name}_exp")[layer, b, g, src]
                st.bank_score[layer, b, g, dst] = st.pend_score[layer, b, g, src]
            st.bank_fill[layer, b, g] = kept
            st.pend_fill[layer, b, g] = 0
