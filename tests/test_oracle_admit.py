"""Pin the oracle's admit step (check (c)).

The oracle sorts records by a key.  These tests do not sort: they check the
result against the definition of "keep the top k under a total order", pair
by pair, with a comparator written out below from the stated order (higher
score first, then committed before candidate, then lower slot; NaN last).
Exhaustive over all score patterns from {0, 1, 2} on a tiny bank (A = 4,
P = 2), which forces ties, plus closed forms and the signed-zero / NaN / inf
readings, plus random full-size cases with 16-level quantised scores.
"""
import itertools
import math

import numpy as np
import pytest

import oracle
import synth_inputs as si
from _util import to_np


def precedes(x, y):
    """True when record x must be kept before record y.  x, y = (score, is_candidate, slot)."""
    sx, cx, ix = x
    sy, cy, iy = y
    nx, ny = math.isnan(sx), math.isnan(sy)
    if nx != ny:
        return ny               # the non-NaN one comes first
    if not nx and sx != sy:     # (-0.0 != +0.0 is False: signed zeros tie)
        return sx > sy
    if cx != cy:
        return cx == 0          # committed before candidate
    return ix < iy


def _state(A, P, nb, npend, bank_scores, pend_scores, D=2):
    cfg = oracle.Config(batch=1, n_layers=1, n_groups=1, q_per_group=1, head_dim=D, ring_slots=3,
                        bank_slots=A, pend_slots=P)
    st = oracle.new_state(cfg)
    # distinct identity bytes per record: K row = (kind, slot), V row = (slot, kind) + 7
    for s in range(A):
        st.bank_k[0, 0, 0, s] = [1, s]
        st.bank_v[0, 0, 0, s] = [s + 7, 8]
    for t in range(P):
        st.pend_k[0, 0, 0, t] = [2, t]
        st.pend_v[0, 0, 0, t] = [t + 7, 9]
    st.bank_score[0, 0, 0, :len(bank_scores)] = bank_scores
    st.pend_score[0, 0, 0, :len(pend_scores)] = pend_scores
    st.bank_fill[...] = nb
    st.pend_fill[...] = npend
    return st


def check_admit_result(before, after, force=False):
    """Check one (sequence, group) admit against its definition. Returns the kept records."""
    cfg = before.cfg
    A, P = cfg.bank_slots, cfg.pend_slots
    nb, npend = int(before.bank_fill[0, 0, 0]), int(before.pend_fill[0, 0, 0])
    triggered = npend == P or (force and npend > 0)
    if not triggered:
        for name in ("bank_k", "bank_v", "bank_score", "pend_k", "pend_v", "pend_score", "bank_fill", "pend_fill"):
            assert np.array_equal(getattr(before, name), getattr(after, name), equal_nan=True)
        return None
    recs = ([(float(before.bank_score[0, 0, 0, s]), 0, s) for s in range(nb)] +
            [(float(before.pend_score[0, 0, 0, t]), 1, t) for t in range(npend)])
    k = min(A, len(recs))
    assert int(after.bank_fill[0, 0, 0]) == k
    assert int(after.pend_fill[0, 0, 0]) == 0
    # identify what sits in each valid bank slot after the admit
    kept = []
    for s in range(k):
        kind = {1: 0, 2: 1}[int(after.bank_k[0, 0, 0, s, 0])]
        src = int(after.bank_k[0, 0, 0, s, 1])
        kept.append((kind, src, s))
    assert len({(kd, src) for kd, src, _ in kept}) == k, "a record is duplicated"
    kept_ids = {(kd, src) for kd, src, _ in kept}
    kept_recs = [r for r in recs if (r[1], r[2]) in kept_ids]
    dropped = [r for r in recs if (r[1], r[2]) not in kept_ids]
    assert len(kept_recs) == k
    for x in kept_recs:
        for y in dropped:
            assert precedes(x, y), (x, y)
    # bytes: each kept record carries its own K, V and score
    for kind, src, dst in kept:
        store = "bank" if kind == 0 else "pend"
        for arr in ("_k", "_v"):
            assert np.array_equal(after.__dict__["bank" + arr][0, 0, 0, dst],
                                  before.__dict__[store + arr][0, 0, 0, src])
        a = after.bank_score[0, 0, 0, dst]
        bsc = before.__dict__[store + "_score"][0, 0, 0, src]
        assert (np.isnan(a) and np.isnan(bsc)) or a.tobytes() == bsc.tobytes()
    # retained anchors do not move
    for kind, src, dst in kept:
        if kind == 0:
            assert src == dst
    # admitted candidates, ascending pending slot, fill the vacated slots in ascending order
    kept_committed = {src for kind, src, _ in kept if kind == 0}
    vacated = [s for s in range(nb) if s not in kept_committed] + list(range(nb, A))
    admitted = sorted(src for kind, src, _ in kept if kind == 1)
    for j, src in enumerate(admitted):
        dst = vacated[j]
        assert after.bank_k[0, 0, 0, dst, 0] == 2 and after.bank_k[0, 0, 0, dst, 1] == src
    return kept_recs


def test_exhaustive_three_level_scores():
    A, P = 4, 2
    n_cases = 0
    for nb in range(A + 1):
        for npend, force in ((P, False), (1, True), (1, False)):
            for pattern in itertools.product((0.0, 1.0, 2.0), repeat=nb + npend):
                st = _state(A, P, nb, npend, list(pattern[:nb]), list(pattern[nb:]))
                before = oracle.copy_state(st)
                oracle.admit(st, 0, force=force)
                check_admit_result(before, st, force=force)
                assert st.status == 0
                n_cases += 1
    assert n_cases == 1089 + 2 * 363


def test_closed_form_candidates_all_higher_evict_exactly_P():
    A, P = 8, 3
    bank = [float(x) for x in (5, 1, 7, 2, 6, 3, 8, 4)]
    st = _state(A, P, A, P, bank, [10.0, 11.0, 12.0])
    before = oracle.copy_state(st)
    oracle.admit(st, 0)
    check_admit_result(before, st)
    # the three lowest anchors (scores 1, 2, 3 at slots 1, 3, 5) are evicted and refilled in order
    assert [int(st.bank_k[0, 0, 0, s, 1]) for s in (1, 3, 5)] == [0, 1, 2]
    assert all(int(st.bank_k[0, 0, 0, s, 0]) == 2 for s in (1, 3, 5))
    assert [float(st.bank_score[0, 0, 0, s]) for s in (1, 3, 5)] == [10.0, 11.0, 12.0]


def test_closed_form_candidates_all_lower_leave_bank_unchanged():
    A, P = 8, 3
    st = _state(A, P, A, P, [float(x) for x in range(10, 18)], [1.0, 2.0, 3.0])
    before = oracle.copy_state(st)
    oracle.admit(st, 0)
    for name in ("bank_k", "bank_v", "bank_score"):
        assert np.array_equal(getattr(before, name), getattr(st, name))
    assert int(st.pend_fill[0, 0, 0]) == 0 and int(st.bank_fill[0, 0, 0]) == A


def test_empty_bank_takes_all_candidates_in_order():
    A, P = 8, 3
    st = _state(A, P, 0, P, [], [0.5, -1.0, 2.0])
    oracle.admit(st, 0)
    assert int(st.bank_fill[0, 0, 0]) == 3
    assert [int(st.bank_k[0, 0, 0, s, 1]) for s in range(3)] == [0, 1, 2]


def test_signed_zero_ties_and_infinities():
    A, P = 2, 2
    # committed -0.0 vs candidate +0.0: equal scores, committed wins
    st = _state(A, P, 2, 2, [-0.0, -1.0], [0.0, -2.0])
    before = oracle.copy_state(st)
    oracle.admit(st, 0)
    check_admit_result(before, st)
    assert int(st.bank_k[0, 0, 0, 0, 0]) == 1 and int(st.bank_k[0, 0, 0, 0, 1]) == 0
    assert int(st.bank_k[0, 0, 0, 1, 0]) == 2 and int(st.bank_k[0, 0, 0, 1, 1]) == 0
    # +inf beats everything, -inf loses to every finite score
    st = _state(A, P, 2, 2, [-math.inf, 3.0], [math.inf, -5.0])
    before = oracle.copy_state(st)
    oracle.admit(st, 0)
    check_admit_result(before, st)
    assert int(st.bank_k[0, 0, 0, 0, 0]) == 2 and int(st.bank_k[0, 0, 0, 0, 1]) == 0   # inf replaced -inf


def test_nan_ranks_last_and_is_flagged():
    A, P = 2, 2
    st = _state(A, P, 2, 2, [float("nan"), 1.0], [0.5, float("nan")])
    before = oracle.copy_state(st)
    oracle.admit(st, 0)
    check_admit_result(before, st)
    assert st.status & oracle.STATUS_NAN_SCORE
    # NaN anchor evicted, replaced by the finite candidate
    assert int(st.bank_k[0, 0, 0, 0, 0]) == 2 and int(st.bank_k[0, 0, 0, 0, 1]) == 0


@pytest.mark.parametrize("nb,npend,seed", [(1024, 256, 1), (1000, 256, 2), (800, 256, 3), (0, 256, 4),
                                           (1024, 37, 5)])
def test_full_size_with_quantized_ties(nb, npend, seed):
    cfg = oracle.Config(batch=1, n_layers=1, n_groups=1, q_per_group=1, head_dim=2, ring_slots=3)
    A, P = cfg.bank_slots, cfg.pend_slots
    bank = to_np(si.f32_quantized_scores((A,), seed))
    pend = to_np(si.f32_quantized_scores((P,), seed + 100))
    st = _state(A, P, nb, npend, list(bank[:nb]), list(pend[:npend]))
    before = oracle.copy_state(st)
    oracle.admit(st, 0, force=True)
    recs = ([(float(bank[s]), 0, s) for s in range(nb)] + [(float(pend[t]), 1, t) for t in range(npend)])
    k = min(A, len(recs))
    # vectorised form of the pairwise check: every kept record precedes every dropped one
    kept_ids = set()
    for s in range(k):
        kind = 0 if st.bank_k[0, 0, 0, s, 0] == 1 else 1
        kept_ids.add((kind, int(st.bank_k[0, 0, 0, s, 1])))
    kept = [r for r in recs if (r[1], r[2]) in kept_ids]
    dropped = [r for r in recs if (r[1], r[2]) not in kept_ids]
    assert len(kept) == k
    if dropped:
        ks = np.array([r[0] for r in kept]); kc = np.array([r[1] for r in kept]); ki = np.array([r[2] for r in kept])
        ds = np.array([r[0] for r in dropped]); dc = np.array([r[1] for r in dropped]); di = np.array([r[2] for r in dropped])
        S1, S2 = ks[:, None], ds[None, :]
        ok = (S1 > S2) | ((S1 == S2) & ((kc[:, None] < dc[None, :]) |
                                       ((kc[:, None] == dc[None, :]) & (ki[:, None] < di[None, :]))))
        assert ok.all()
    assert int(st.bank_fill[0, 0, 0]) == k and int(st.pend_fill[0, 0, 0]) == 0
    if nb == 1024 and npend == 256:
        check_admit_result(before, st, force=True)
