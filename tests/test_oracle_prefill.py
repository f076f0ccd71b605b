"""Pin the oracle's block prefill.

  * g = 0: every query's output equals brute-force masked attention over the
    full history the test keeps by position (window [p - R, p], causal);
  * a block of n = P tokens starting with an empty pending buffer equals n
    decode steps (each followed by the admit rule): same outputs, same state
    bytes; this ties prefill to the brute-force-pinned decode;
  * a block of any n <= P tokens that starts with pend_fill != 0 (its
    candidates fit) equals n decode steps followed by a forced admit;
  * check (d): records admitted at the end of block k are invisible to block
    k's queries and visible to block k+1's;
  * g = +-1/2: anchor part equals brute force over the bank as committed
    before the block;
  * a block whose candidates do not fit the pending buffer raises the flag.
"""
import math

import numpy as np
import pytest
from scipy.special import softmax

import oracle
import synth_inputs as si
from _util import bf16_bits_to_f64_torch as f64, inputs_np, to_np


def _cfg(**kw):
    base = dict(batch=2, n_layers=1, n_groups=2, q_per_group=3, head_dim=16,
                ring_slots=7, bank_slots=6, pend_slots=4, softmax_scale=0.3)
    base.update(kw)
    return oracle.Config(**base)


def _state(cfg, seed, bank_fill, pend_fill=0, pos=0):
    arr = {k: to_np(v) for k, v in si.state_contents(cfg.n_layers, cfg.batch, cfg.n_groups, cfg.head_dim,
                                                     cfg.ring_slots, cfg.bank_slots, cfg.pend_slots,
                                                     seed=seed).items()}
    return oracle.state_from_arrays(cfg, arr, pos=pos, bank_fill=bank_fill, pend_fill=pend_fill)


def _block(cfg, seed, n=None):
    n = cfg.pend_slots if n is None else n
    return inputs_np(si.prefill_inputs(cfg.batch, n, cfg.n_groups, cfg.q_per_group, cfg.head_dim, seed=seed))


def _args(x):
    return [x[k] for k in ("q", "k", "v", "cand_k", "cand_v", "cand_score")]


@pytest.mark.parametrize("ring_slots,n,pend_slots", [(7, 4, 4), (3, 4, 4), (5, 5, 5), (9, 2, 2), (7, 3, 8)])
def test_gate_zero_equals_causal_window_bruteforce(ring_slots, n, pend_slots):
    cfg = _cfg(ring_slots=ring_slots, pend_slots=pend_slots)
    st = _state(cfg, seed=1, bank_fill=3)
    w = np.zeros((cfg.n_q_heads, cfg.head_dim), np.float32)
    bg = np.zeros(cfg.n_q_heads, np.float32)
    hist_k = [[[] for _ in range(cfg.n_groups)] for _ in range(cfg.batch)]
    hist_v = [[[] for _ in range(cfg.n_groups)] for _ in range(cfg.batch)]
    R = cfg.ring_slots
    for blk in range(6):
        x = _block(cfg, 100 + blk, n=n)
        s0 = st.pos.copy()
        _, out = oracle.prefill_block(st, 0, *_args(x), w, bg, return_f64=True)
        for b in range(cfg.batch):
            for g in range(cfg.n_groups):
                for i in range(n):
                    hist_k[b][g].append(x["k"][b, i, g])
                    hist_v[b][g].append(x["v"][b, i, g])
                K = f64(np.stack(hist_k[b][g]))
                V = f64(np.stack(hist_v[b][g]))
                for i in range(n):
                    p = int(s0[0, b, g]) + i
                    for h in range(cfg.q_per_group):
                        head = g * cfg.q_per_group + h
                        logits = cfg.softmax_scale * (K[:p + 1] @ f64(x["q"][b, i, head]))
                        logits[np.arange(p + 1) < p - R] = -np.inf
                        ref = softmax(logits) @ V[:p + 1]
                        np.testing.assert_allclose(out[b, i, head], ref, rtol=1e-11, atol=1e-12)


def test_block_equals_decode_steps():
    cfg = _cfg(ring_slots=7, pend_slots=4)
    st_p = _state(cfg, seed=2, bank_fill=5, pend_fill=0, pos=11)
    st_d = oracle.copy_state(st_p)
    w = si.f32_normal((cfg.n_q_heads, cfg.head_dim), 3, std=0.2).numpy()
    bg = si.f32_normal((cfg.n_q_heads,), 4, std=0.2).numpy()
    for blk in range(4):
        x = _block(cfg, 200 + blk)
        _, out_p = oracle.prefill_block(st_p, 0, *_args(x), w, bg, return_f64=True)
        for i in range(cfg.pend_slots):
            _, out_d = oracle.decode_step(st_d, 0, x["q"][:, i], x["k"][:, i], x["v"][:, i], x["cand_k"][:, i],
                                          x["cand_v"][:, i], x["cand_score"][:, i], w, bg, return_f64=True)
            oracle.admit(st_d, 0)
            np.testing.assert_allclose(out_p[:, i], out_d, rtol=1e-12, atol=1e-13)
        for name in ("ring_k", "ring_v", "bank_k", "bank_v", "bank_score", "pend_k", "pend_v", "pend_score",
                     "pos", "bank_fill", "pend_fill"):
            assert np.array_equal(getattr(st_p, name), getattr(st_d, name)), name


@pytest.mark.parametrize("n,pend0", [(1, 0), (3, 2), (5, 0), (6, 2), (8, 0)])
def test_ragged_block_equals_decode_steps_then_forced_admit(n, pend0):
    """Blocks shorter than P, after decode steps left candidates pending: the block's reads and
    writes are those of n decode steps, and its forced admit is the admit at the end."""
    cfg = _cfg(ring_slots=7, pend_slots=8)
    st_p = _state(cfg, seed=12, bank_fill=4, pend_fill=pend0, pos=9)
    st_d = oracle.copy_state(st_p)
    w = si.f32_normal((cfg.n_q_heads, cfg.head_dim), 13, std=0.2).numpy()
    bg = si.f32_normal((cfg.n_q_heads,), 14, std=0.2).numpy()
    for blk in range(3):
        x = _block(cfg, 300 + blk, n=n)
        _, out_p = oracle.prefill_block(st_p, 0, *_args(x), w, bg, return_f64=True)
        for i in range(n):
            _, out_d = oracle.decode_step(st_d, 0, x["q"][:, i], x["k"][:, i], x["v"][:, i], x["cand_k"][:, i],
                                          x["cand_v"][:, i], x["cand_score"][:, i], w, bg, return_f64=True)
            oracle.admit(st_d, 0)
            np.testing.assert_allclose(out_p[:, i], out_d, rtol=1e-12, atol=1e-13)
        oracle.admit(st_d, 0, force=True)
        for name in ("ring_k", "ring_v", "bank_k", "bank_v", "bank_score", "pend_k", "pend_v", "pend_score",
                     "pos", "bank_fill", "pend_fill"):
            assert np.array_equal(getattr(st_p, name), getattr(st_d, name)), name
        assert int(st_p.pend_fill.max()) == 0 and st_p.status == 0


def test_block_admits_are_invisible_to_own_block_and_visible_to_next():
    cfg = _cfg(batch=1)
    st = _state(cfg, seed=5, bank_fill=6, pos=20)
    w = np.zeros((cfg.n_q_heads, cfg.head_dim), np.float32)
    bg = np.full(cfg.n_q_heads, math.atanh(0.5), np.float32)
    x = _block(cfg, 300)
    x["cand_score"][:] = 50.0                      # every candidate is admitted at the end of the block
    y = dict(x)
    y["cand_v"] = oracle.f32_to_bf16(f64(x["cand_v"]) * -2.0 + 1.0)
    y["cand_k"] = oracle.f32_to_bf16(f64(x["cand_k"]) + 0.5)
    a, b = oracle.copy_state(st), oracle.copy_state(st)
    oa = oracle.prefill_block(a, 0, *_args(x), w, bg)
    ob = oracle.prefill_block(b, 0, *_args(y), w, bg)
    assert np.array_equal(oa, ob)                  # block k does not see its own admits
    assert int(a.bank_fill[0, 0, 0]) == cfg.bank_slots and not np.array_equal(a.bank_v, b.bank_v)
    z = _block(cfg, 301)
    oa = oracle.prefill_block(a, 0, *_args(z), w, bg)
    ob = oracle.prefill_block(b, 0, *_args(z), w, bg)
    assert not np.array_equal(oa, ob)              # block k+1 does


@pytest.mark.parametrize("gate", [0.5, -0.5])
def test_anchor_is_bank_as_committed_before_block(gate):
    cfg = _cfg()
    st0 = _state(cfg, seed=6, bank_fill=5, pos=13)
    st1 = oracle.copy_state(st0)
    w = np.zeros((cfg.n_q_heads, cfg.head_dim), np.float32)
    b1 = np.full(cfg.n_q_heads, math.atanh(gate), np.float32)
    g_exact = math.tanh(float(b1[0]))
    for blk in range(3):
        x = _block(cfg, 400 + blk)
        x["cand_score"][:] = 9.0
        bank_before = oracle.copy_state(st1)
        _, o0 = oracle.prefill_block(st0, 0, *_args(x), w, np.zeros_like(b1), return_f64=True)
        _, o1 = oracle.prefill_block(st1, 0, *_args(x), w, b1, return_f64=True)
        for b in range(cfg.batch):
            for g in range(cfg.n_groups):
                nb = int(bank_before.bank_fill[0, b, g])
                K = f64(bank_before.bank_k[0, b, g, :nb])
                V = f64(bank_before.bank_v[0, b, g, :nb])
                for i in range(cfg.pend_slots):
                    for h in range(cfg.q_per_group):
                        head = g * cfg.q_per_group + h
                        ref = softmax(cfg.softmax_scale * (K @ f64(x["q"][b, i, head]))) @ V
                        np.testing.assert_allclose((o1[b, i, head] - o0[b, i, head]) / g_exact, ref,
                                                   rtol=1e-9, atol=1e-11)


def test_candidates_that_do_not_fit_are_flagged_and_dropped():
    cfg = _cfg(batch=1)
    st = _state(cfg, seed=7, bank_fill=2, pend_fill=1, pos=8)
    before = oracle.copy_state(st)
    w = np.zeros((cfg.n_q_heads, cfg.head_dim), np.float32)
    oracle.prefill_block(st, 0, *_args(_block(cfg, 500)), w, np.zeros(cfg.n_q_heads, np.float32))
    assert st.status & oracle.STATUS_PREFILL_PENDING_OVERFLOW
    # the forced admit took in the one record that was already pending
    assert int(st.bank_fill[0, 0, 0]) == 3 and int(st.pend_fill[0, 0, 0]) == 0
    assert np.array_equal(st.bank_k[0, 0, :, 2], before.pend_k[0, 0, :, 0])
    assert int(st.pos[0, 0, 0]) == 8 + cfg.pend_slots
