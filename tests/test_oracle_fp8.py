"""Pins for the FP8 oracle (E4M3 ring / bank / pending storage with per-row power-of-two scales).

Each function of ``oracle/rma_oracle_fp8.py`` is checked against something other
than itself: torch's float8_e4m3fn conversion (a library routine) for the code
table and the rounding, the defining inequality for the scale exponent, the
rounding bound for the round trip, brute-force attention over the dequantised
history for the decode step, and the BF16 oracle on rows that E4M3 holds exactly.
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import softmax

import oracle
import synth_inputs as si
from _util import to_np


def _torch_e4m3_codes(x_f32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x_f32, dtype=np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def test_code_table_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6   # max, min subnormal, min normal


def test_rounding_matches_torch_on_every_bf16_value_in_range():
    bits = np.arange(1 << 16, dtype=np.uint32)
    x = (bits << 16).view(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) <= 448.0)]
    assert np.array_equal(oracle.f32_to_e4m3(x), _torch_e4m3_codes(x))


def test_rounding_matches_torch_on_ties_and_their_neighbours():
    vals = oracle.e4m3_to_f64(np.arange(0x7F, dtype=np.uint8))       # 0 .. 448, increasing
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)            # exact in FP32
    assert np.array_equal(mids.astype(np.float64), (vals[:-1] + vals[1:]) / 2)
    up = np.nextafter(mids, np.float32(np.inf))
    dn = np.nextafter(mids, np.float32(0))
    x = np.concatenate([mids, up, dn, -mids, -up, -dn, np.float32([0.0, -0.0])]).astype(np.float32)
    x = x[np.abs(x) <= 448.0]
    assert np.array_equal(oracle.f32_to_e4m3(x), _torch_e4m3_codes(x))
    # a tie goes to the even code: the midpoint of codes 1 and 2 gives 2, of 2 and 3 gives 2
    assert oracle.f32_to_e4m3(np.float32([1.5 * 2 ** -9, 2.5 * 2 ** -9])).tolist() == [2, 2]


def test_row_exponent_is_the_smallest_that_fits():
    rng = np.random.default_rng(0)
    a = np.exp(rng.uniform(-80, 80, 20000))
    edges = np.array([448.0 * 2.0 ** k for k in range(-40, 40)])
    a = np.concatenate([a, edges, np.nextafter(edges, np.inf), np.nextafter(edges, 0)])
    e = oracle.row_exponent(a)
    for amax, ee in zip(a, e):
        assert amax <= math.ldexp(448.0, int(ee))
        assert ee == -127 or amax > math.ldexp(448.0, int(ee) - 1)
    assert oracle.row_exponent(0.0) == 0
    assert oracle.row_exponent(1e-300) == -127 and oracle.row_exponent(3.3e38) == 120


def test_quantized_row_round_trip():
    rng = np.random.default_rng(1)
    rows = oracle.f32_to_bf16(rng.standard_normal((64, 256)) * np.exp(rng.uniform(-20, 20, (64, 1))))
    rows[3] = 0                                     # an all-zero row: exponent 0, codes 0
    codes, exps = oracle.quantize_rows(rows)
    x = oracle.bf16_to_f64(rows)
    deq = oracle.dequantize_rows(codes, exps)
    # the same rounding, done by the library on the scaled values
    scaled = (x * np.ldexp(1.0, -exps.astype(np.int64))[:, None]).astype(np.float32)
    lib_deq = torch.from_numpy(scaled).to(torch.float8_e4m3fn).to(torch.float64).numpy() * \
        np.ldexp(1.0, exps.astype(np.int64))[:, None]
    assert np.array_equal(deq, lib_deq)
    # E4M3 keeps 4 significant bits: |error| <= 2**-4 |x| for scaled magnitudes in the normal range,
    # and <= 2**-10 * 2**e below it (half the subnormal spacing)
    scale = np.ldexp(1.0, exps.astype(np.int64))[:, None]
    bound = np.maximum(np.abs(x) / 16.0, scale * 2.0 ** -10)
    assert np.all(np.abs(deq - x) <= bound)
    assert exps[3] == 0 and not codes[3].any()
    assert np.all(np.max(np.abs(codes.astype(np.int64) & 0x7F), axis=1)[np.arange(64) != 3] >= 0x70)  # amax in [256, 448]


def _exact_rows(rng, shape, k):
    """BF16 rows that E4M3 holds exactly at scale 2**k: grid values times 2**k, each row reaching 448 * 2**k."""
    grid = oracle.e4m3_to_f64(rng.integers(0, 0x7F, size=shape, dtype=np.uint8) | (rng.integers(0, 2, size=shape,
                                                                                              dtype=np.uint8) << 7))
    grid[..., 0] = 448.0
    return oracle.f64_to_bf16(grid * 2.0 ** k)


def test_fp8_oracle_equals_bf16_oracle_on_exact_rows():
    """Rows that E4M3 represents exactly quantise losslessly: the FP8 decode step, admit and
    state then agree with the BF16 oracle's, value for value."""
    rng = np.random.default_rng(2)
    cfg = oracle.Config(batch=2, n_layers=1, ring_slots=9, bank_slots=6, pend_slots=3)
    L, B, G, D = 1, 2, 4, 256
    arrays = {n: _exact_rows(rng, (L, B, G, s, D), -6) for n, s in
              (("ring_k", 9), ("ring_v", 9), ("bank_k", 6), ("bank_v", 6), ("pend_k", 3), ("pend_v", 3))}
    arrays["bank_score"] = rng.standard_normal((L, B, G, 6)).astype(np.float32)
    arrays["pend_score"] = rng.standard_normal((L, B, G, 3)).astype(np.float32)
    st = oracle.state_from_arrays(cfg, arrays, pos=[[[12], [4]]], bank_fill=[[[6], [2]]], pend_fill=[[[1], [0]]])
    fst = oracle.quantize_state(st)
    w, b = si.gate_params(1, 16, 256, seed=2)
    for t in range(7):
        x = {k: to_np(v) for k, v in si.decode_inputs(B, G, 4, D, seed=100 + t).items()}
        for name in ("k_cur", "v_cur", "cand_k", "cand_v"):
            x[name] = _exact_rows(rng, (B, G, D), -5)
        o1 = oracle.decode_step(st, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"],
                                w[0].numpy(), b[0].numpy())
        o2 = oracle.decode_step_fp8(fst, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                                    x["cand_score"], w[0].numpy(), b[0].numpy())
        assert np.array_equal(o1, o2), f"step {t}"
        oracle.admit(st, 0)
        oracle.admit_fp8(fst, 0)
        q = oracle.quantize_state(st)
        for name in ("ring_k", "ring_v", "bank_k", "bank_v", "pend_k", "pend_v", "ring_k_exp", "bank_v_exp"):
            assert np.array_equal(getattr(q, name), getattr(fst, name)), f"step {t}: {name}"
        assert np.array_equal(q.bank_score.view(np.uint32), fst.bank_score.view(np.uint32))
        for name in ("pos", "bank_fill", "pend_fill"):
            assert np.array_equal(getattr(q, name), getattr(fst, name))
    assert int(fst.pend_fill.max()) < 3 and int(fst.bank_fill.min()) >= 2   # admits happened


def test_fp8_decode_matches_brute_force_over_the_dequantized_history():
    """g = 0: the output is softmax attention over the last R dequantised ring rows plus the current
    token (as given); the state afterwards holds the current token quantised in slot pos mod R."""
    rng = np.random.default_rng(3)
    R, D = 5, 256
    cfg = oracle.Config(batch=1, n_layers=1, ring_slots=R, bank_slots=4, pend_slots=4)
    st = oracle.quantize_state(oracle.new_state(cfg))
    w = np.zeros((16, D), np.float32)
    b = np.zeros(16, np.float32)
    hist_k, hist_v = [], []
    for t in range(13):                                      # wraps the ring twice
        x = {k: to_np(v) for k, v in si.decode_inputs(1, 4, 4, D, seed=300 + t).items()}
        out = oracle.decode_step_fp8(st, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                                     x["cand_score"], w, b, return_f64=True)[1]
        kq, ke = oracle.quantize_rows(x["k_cur"])
        vq, ve = oracle.quantize_rows(x["v_cur"])
        for g in range(4):
            Kh = np.array([r[g] for r in hist_k[-R:]] + [oracle.bf16_to_f64(x["k_cur"][0, g])]).reshape(-1, D)
            Vh = np.array([r[g] for r in hist_v[-R:]] + [oracle.bf16_to_f64(x["v_cur"][0, g])]).reshape(-1, D)
            for h in range(4):
                qh = oracle.bf16_to_f64(x["q"][0, 4 * g + h])
                p = softmax(Kh @ qh / 16.0)
                assert np.allclose(out[0, 4 * g + h], p @ Vh, rtol=1e-12, atol=1e-12), (t, g, h)
            slot = t % R
            assert np.array_equal(st.ring_k[0, 0, g, slot], kq[0, g]) and st.ring_k_exp[0, 0, g, slot] == ke[0, g]
            assert np.array_equal(st.ring_v[0, 0, g, slot], vq[0, g]) and st.ring_v_exp[0, 0, g, slot] == ve[0, g]
        hist_k.append(oracle.dequantize_rows(kq, ke)[0])
        hist_v.append(oracle.dequantize_rows(vq, ve)[0])


def test_fp8_admit_commutes_with_quantisation():
    """Admit copies rows unchanged, so quantising then admitting equals admitting then quantising."""
    rng = np.random.default_rng(4)
    cfg = oracle.Config(batch=3, n_layers=1, ring_slots=4, bank_slots=8, pend_slots=5)
    arrays = si.state_contents(1, 3, 4, 256, 4, 8, 5, seed=4, quantized_scores=True)
    arrays = {k: to_np(v) for k, v in arrays.items()}
    bank = rng.integers(0, 9, size=(1, 3, 4))
    st = oracle.state_from_arrays(cfg, arrays, pos=50, bank_fill=bank, pend_fill=5)
    fst = oracle.quantize_state(st)
    oracle.admit(st, 0)
    oracle.admit_fp8(fst, 0)
    q = oracle.quantize_state(st)
    for name in ("bank_k", "bank_v", "bank_k_exp", "bank_v_exp", "pend_k", "pend_v"):
        assert np.array_equal(getattr(q, name), getattr(fst, name)), name
    assert np.array_equal(q.bank_score.view(np.uint32), fst.bank_score.view(np.uint32))
    assert np.array_equal(q.bank_fill, fst.bank_fill) and not fst.pend_fill.any()
