"""Pin the oracle's decode step (retrieve, gate, ring write, candidate append).

Independent references used here, none of which is the oracle's own code path:
  * brute force: masked softmax attention (scipy's softmax) over the FULL
    history the test keeps by position, restricted to the last R+1 positions;
    this pins ring indexing, window length, the current token, the softmax
    scale and the query-head -> KV-group mapping (check (b), g = 0);
  * the gate set to exactly 1/2 (w_g = 0, b_g = atanh(1/2)) so that
    2 (out - local) must equal brute-force attention over the committed bank;
  * closed forms: one anchor -> its V; identical keys -> mean of V; empty bank
    -> out == local; first token -> v_cur;
  * byte checks of the ring slot, pending append and the overflow flag.
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
                ring_slots=7, bank_slots=5, pend_slots=3, softmax_scale=0.25)
    base.update(kw)
    return oracle.Config(**base)


def _random_state(cfg, seed, bank_fill, pend_fill=0, pos=0):
    arr = {k: to_np(v) for k, v in si.state_contents(cfg.n_layers, cfg.batch, cfg.n_groups, cfg.head_dim,
                                                     cfg.ring_slots, cfg.bank_slots, cfg.pend_slots,
                                                     seed=seed).items()}
    return oracle.state_from_arrays(cfg, arr, pos=pos, bank_fill=bank_fill, pend_fill=pend_fill)


def _brute_local(hist_k, hist_v, qh, pos, R, scale):
    """Masked attention over positions 0..pos of the full history, keeping p >= pos - R."""
    K = f64(np.stack(hist_k[:pos + 1]))
    V = f64(np.stack(hist_v[:pos + 1]))
    logits = scale * (K @ qh)
    logits[np.arange(pos + 1) < pos - R] = -np.inf
    return softmax(logits) @ V


def _brute_bank(st, layer, b, g, qh, scale):
    nb = int(st.bank_fill[layer, b, g])
    if nb == 0:
        return np.zeros(st.cfg.head_dim)
    K = f64(st.bank_k[layer, b, g, :nb])
    V = f64(st.bank_v[layer, b, g, :nb])
    return softmax(scale * (K @ qh)) @ V


def _run_with_history(cfg, n_steps, w_g, b_g, bank_fill=3, check_every=1, seed=11):
    st = _random_state(cfg, seed=seed, bank_fill=bank_fill)
    B, G, H = cfg.batch, cfg.n_groups, cfg.q_per_group
    hist_k = [[[] for _ in range(G)] for _ in range(B)]
    hist_v = [[[] for _ in range(G)] for _ in range(B)]
    worst = 0.0
    for t in range(n_steps):
        x = inputs_np(si.decode_inputs(B, G, H, cfg.head_dim, seed=1000 + t))
        for b in range(B):
            for g in range(G):
                hist_k[b][g].append(x["k_cur"][b, g])
                hist_v[b][g].append(x["v_cur"][b, g])
        pos0 = st.pos.copy()
        _, out = oracle.decode_step(st, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                                    x["cand_score"], w_g, b_g, return_f64=True)
        oracle.admit(st, 0)
        if t % check_every and t < n_steps - 3:
            continue
        for b in range(B):
            for g in range(G):
                for h in range(H):
                    head = g * H + h
                    qh = f64(x["q"][b, head])
                    ref = _brute_local(hist_k[b][g], hist_v[b][g], qh, int(pos0[0, b, g]), cfg.ring_slots,
                                       cfg.softmax_scale)
                    err = np.max(np.abs(out[b, head] - ref))
                    worst = max(worst, err)
    return worst


def test_gate_zero_equals_sliding_window_bruteforce_small():
    """Check (b): g = tanh(0) = 0, so out is local attention; ring wraps 4 times (R = 7, 30 steps)."""
    cfg = _cfg()
    w = np.zeros((cfg.n_q_heads, cfg.head_dim), np.float32)
    b = np.zeros(cfg.n_q_heads, np.float32)
    assert _run_with_history(cfg, 30, w, b) < 1e-12


def test_gate_zero_bruteforce_full_dims():
    """Same check at the pages' window (1,023 + 1) and head_dim 256, through two ring wraps' worth of steps."""
    cfg = oracle.Config(batch=1, n_layers=1, n_groups=1, q_per_group=2, head_dim=256,
                        ring_slots=1023, bank_slots=1024, pend_slots=256)
    w = np.zeros((2, 256), np.float32)
    b = np.zeros(2, np.float32)
    assert _run_with_history(cfg, 1100, w, b, bank_fill=0, check_every=97) < 1e-12


@pytest.mark.parametrize("gate", [0.5, -0.5])
def test_anchor_read_through_half_gate(gate):
    """g = +-1/2 exactly: (out - local) / g equals brute-force attention over the committed bank."""
    cfg = _cfg()
    st0 = _random_state(cfg, seed=3, bank_fill=4, pend_fill=2, pos=9)
    st1 = oracle.copy_state(st0)
    w = np.zeros((cfg.n_q_heads, cfg.head_dim), np.float32)
    b0 = np.zeros(cfg.n_q_heads, np.float32)
    b1 = np.full(cfg.n_q_heads, math.atanh(gate), np.float32)
    assert abs(math.tanh(float(b1[0])) - gate) < 1e-7
    g_exact = math.tanh(float(b1[0]))
    for t in range(8):
        x = inputs_np(si.decode_inputs(cfg.batch, cfg.n_groups, cfg.q_per_group, cfg.head_dim, seed=50 + t))
        ref_st = oracle.copy_state(st1)
        _, o0 = oracle.decode_step(st0, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                                   x["cand_score"], w, b0, return_f64=True)
        _, o1 = oracle.decode_step(st1, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                                   x["cand_score"], w, b1, return_f64=True)
        oracle.admit(st0, 0)
        oracle.admit(st1, 0)
        for bb in range(cfg.batch):
            for g in range(cfg.n_groups):
                for h in range(cfg.q_per_group):
                    head = g * cfg.q_per_group + h
                    ref = _brute_bank(ref_st, 0, bb, g, f64(x["q"][bb, head]), cfg.softmax_scale)
                    np.testing.assert_allclose((o1[bb, head] - o0[bb, head]) / g_exact, ref, rtol=1e-9, atol=1e-11)


def test_single_anchor_gives_its_value_and_identical_keys_give_mean():
    cfg = _cfg(batch=1)
    st = _random_state(cfg, seed=5, bank_fill=1, pos=4)
    st_ref = oracle.copy_state(st)
    w = np.zeros((cfg.n_q_heads, cfg.head_dim), np.float32)
    bg = np.full(cfg.n_q_heads, math.atanh(0.5), np.float32)
    g = math.tanh(float(bg[0]))
    x = inputs_np(si.decode_inputs(1, cfg.n_groups, cfg.q_per_group, cfg.head_dim, seed=7))
    _, o1 = oracle.decode_step(st, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                               x["cand_score"], w, bg, return_f64=True)
    _, o0 = oracle.decode_step(oracle.copy_state(st_ref), 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"],
                               x["cand_v"], x["cand_score"], w, np.zeros_like(bg), return_f64=True)
    for grp in range(cfg.n_groups):
        v0 = f64(st_ref.bank_v[0, 0, grp, 0])
        for h in range(cfg.q_per_group):
            head = grp * cfg.q_per_group + h
            np.testing.assert_allclose(o1[0, head] - o0[0, head], g * v0, rtol=1e-12, atol=1e-14)

    # identical bank keys: softmax weights are equal, anchor = mean of the valid V rows
    st2 = _random_state(cfg, seed=6, bank_fill=4, pos=4)
    st2.bank_k[0, 0, :, :, :] = st2.bank_k[0, 0, :, :1, :]
    st2_ref = oracle.copy_state(st2)
    _, o1 = oracle.decode_step(st2, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                               x["cand_score"], w, bg, return_f64=True)
    _, o0 = oracle.decode_step(oracle.copy_state(st2_ref), 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"],
                               x["cand_v"], x["cand_score"], w, np.zeros_like(bg), return_f64=True)
    for grp in range(cfg.n_groups):
        mean_v = f64(st2_ref.bank_v[0, 0, grp, :4]).mean(axis=0)
        for h in range(cfg.q_per_group):
            head = grp * cfg.q_per_group + h
            np.testing.assert_allclose(o1[0, head] - o0[0, head], g * mean_v, rtol=1e-12, atol=1e-13)


def test_empty_bank_output_is_local_and_first_token_reads_itself():
    cfg = _cfg(batch=1)
    st = _random_state(cfg, seed=8, bank_fill=0, pos=0)
    w = si.f32_normal((cfg.n_q_heads, cfg.head_dim), 9).numpy()
    bg = np.full(cfg.n_q_heads, 0.7, np.float32)
    x = inputs_np(si.decode_inputs(1, cfg.n_groups, cfg.q_per_group, cfg.head_dim, seed=10))
    _, out = oracle.decode_step(st, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                                x["cand_score"], w, bg, return_f64=True)
    for grp in range(cfg.n_groups):
        for h in range(cfg.q_per_group):
            # window = {current token}: softmax of one logit is 1, anchor = 0
            assert np.array_equal(out[0, grp * cfg.q_per_group + h], f64(x["v_cur"][0, grp]))


def test_gate_uses_own_head_query_and_row():
    """g_h = tanh(q_h . w_g[h] + b_g[h]) for every head, read back through a one-record bank."""
    cfg = _cfg(batch=1)
    st = _random_state(cfg, seed=12, bank_fill=1, pos=5)
    st_ref = oracle.copy_state(st)
    w = si.f32_normal((cfg.n_q_heads, cfg.head_dim), 13, std=0.1).numpy()
    bg = si.f32_normal((cfg.n_q_heads,), 14, std=0.3).numpy()
    x = inputs_np(si.decode_inputs(1, cfg.n_groups, cfg.q_per_group, cfg.head_dim, seed=15))
    _, o1 = oracle.decode_step(st, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                               x["cand_score"], w, bg, return_f64=True)
    _, o0 = oracle.decode_step(oracle.copy_state(st_ref), 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"],
                               x["cand_v"], x["cand_score"], np.zeros_like(w), np.zeros_like(bg),
                               return_f64=True)
    for grp in range(cfg.n_groups):
        v0 = f64(st_ref.bank_v[0, 0, grp, 0])
        j = int(np.argmax(np.abs(v0)))
        for h in range(cfg.q_per_group):
            head = grp * cfg.q_per_group + h
            g_measured = (o1[0, head, j] - o0[0, head, j]) / v0[j]
            qh = f64(x["q"][0, head])
            g_expected = math.tanh(math.fsum(float(a) * float(c) for a, c in zip(qh, w[head])) + float(bg[head]))
            assert abs(g_measured - g_expected) < 1e-12
    # the gates differ across heads, so a wrong head/row mapping could not pass
    gs = [math.tanh(float(f64(x["q"][0, hh]) @ w[hh]) + float(bg[hh])) for hh in range(cfg.n_q_heads)]
    assert len(set(np.round(gs, 6))) == cfg.n_q_heads


def test_writes_ring_slot_pending_and_counters():
    cfg = _cfg(batch=2)
    st = _random_state(cfg, seed=16, bank_fill=2, pend_fill=1, pos=12)
    w = np.zeros((cfg.n_q_heads, cfg.head_dim), np.float32)
    bg = np.zeros(cfg.n_q_heads, np.float32)
    x = inputs_np(si.decode_inputs(2, cfg.n_groups, cfg.q_per_group, cfg.head_dim, seed=17))
    before = oracle.copy_state(st)
    oracle.decode_step(st, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"], w, bg)
    slot = 12 % cfg.ring_slots
    for b in range(2):
        for g in range(cfg.n_groups):
            assert np.array_equal(st.ring_k[0, b, g, slot], x["k_cur"][b, g])
            assert np.array_equal(st.ring_v[0, b, g, slot], x["v_cur"][b, g])
            others = [s for s in range(cfg.ring_slots) if s != slot]
            assert np.array_equal(st.ring_k[0, b, g, others], before.ring_k[0, b, g, others])
            assert np.array_equal(st.pend_k[0, b, g, 1], x["cand_k"][b, g])
            assert np.array_equal(st.pend_v[0, b, g, 1], x["cand_v"][b, g])
            assert st.pend_score[0, b, g, 1] == x["cand_score"][b, g]
    assert (st.pos == 13).all() and (st.pend_fill == 2).all() and (st.bank_fill == 2).all()
    assert np.array_equal(st.bank_k, before.bank_k) and st.status == 0


def test_pending_overflow_flags_and_drops_candidate():
    cfg = _cfg(batch=1)
    st = _random_state(cfg, seed=18, bank_fill=2, pend_fill=cfg.pend_slots, pos=3)
    before = oracle.copy_state(st)
    w = np.zeros((cfg.n_q_heads, cfg.head_dim), np.float32)
    x = inputs_np(si.decode_inputs(1, cfg.n_groups, cfg.q_per_group, cfg.head_dim, seed=19))
    oracle.decode_step(st, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"], w,
                       np.zeros(cfg.n_q_heads, np.float32))
    assert st.status & oracle.STATUS_PENDING_OVERFLOW
    assert np.array_equal(st.pend_k, before.pend_k) and (st.pend_fill == cfg.pend_slots).all()
    assert (st.pos == 4).all()


def test_candidate_invisible_until_admitted_then_visible():
    """A candidate is never read from pending; after its admit it is read from the bank at the next step."""
    cfg = _cfg(batch=1, pend_slots=2, bank_slots=3)
    st = _random_state(cfg, seed=20, bank_fill=3, pend_fill=1, pos=6)
    w = np.zeros((cfg.n_q_heads, cfg.head_dim), np.float32)
    bg = np.full(cfg.n_q_heads, math.atanh(0.5), np.float32)
    x = inputs_np(si.decode_inputs(1, cfg.n_groups, cfg.q_per_group, cfg.head_dim, seed=21))
    x["cand_score"][:] = 100.0     # certain to be admitted
    x2 = dict(x)
    x2["cand_v"] = oracle.f32_to_bf16(f64(x["cand_v"]) + 3.0)
    a, b = oracle.copy_state(st), oracle.copy_state(st)
    oa = oracle.decode_step(a, 0, *[x[k] for k in ("q", "k_cur", "v_cur", "cand_k", "cand_v", "cand_score")], w, bg)
    ob = oracle.decode_step(b, 0, *[x2[k] for k in ("q", "k_cur", "v_cur", "cand_k", "cand_v", "cand_score")], w, bg)
    assert np.array_equal(oa, ob)            # same step: pending is not read
    oracle.admit(a, 0)
    oracle.admit(b, 0)                        # pend_fill hit P = 2: admit fires
    assert (a.pend_fill == 0).all()
    y = inputs_np(si.decode_inputs(1, cfg.n_groups, cfg.q_per_group, cfg.head_dim, seed=22))
    oa = oracle.decode_step(a, 0, *[y[k] for k in ("q", "k_cur", "v_cur", "cand_k", "cand_v", "cand_score")], w, bg)
    ob = oracle.decode_step(b, 0, *[y[k] for k in ("q", "k_cur", "v_cur", "cand_k", "cand_v", "cand_score")], w, bg)
    assert not np.array_equal(oa, ob)        # next step: the admitted record is read
