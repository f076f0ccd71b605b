"""The benchmark's host-side fill tracking follows the oracle's counters step by step.

`bench.FillTracker` computes every decode launch's algorithmic bytes from counters it
advances on the host; here the same counters are advanced by the oracle's own decode
and admit on a small state, so a wrong admit rule or ring fill in the tracker shows up.
"""
import os
import sys

import numpy as np

import oracle
import synth_inputs as si
from _util import to_np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_fill_tracker_matches_the_oracle_counters():
    R, A, P, L, B, G = 12, 8, 4, 2, 3, 4
    cfg = oracle.Config(batch=B, n_layers=L, ring_slots=R, bank_slots=A, pend_slots=P)
    cont = si.state_contents(L, B, G, 256, R, A, P, seed=5)
    pos = to_np(si.uniform_int((L, B, G), 0, 20, seed=6))
    bank = to_np(si.uniform_int((L, B, G), 0, A, seed=7))
    pend = to_np(si.uniform_int((L, B, G), 0, P - 1, seed=8))
    st = oracle.state_from_arrays(cfg, {k: to_np(v) for k, v in cont.items()}, pos=pos, bank_fill=bank, pend_fill=pend)
    cnt = np.stack([pos, bank, pend, np.zeros_like(pos)], axis=-1)
    tr = bench.FillTracker(cnt, R=R, A=A, P=P)
    w, b = si.gate_params(L, G * 4, 256, seed=9)
    for t in range(2 * P + 3):
        x = {k: to_np(v) for k, v in si.decode_inputs(B, G, 4, 256, seed=50 + t).items()}
        for layer in range(L):
            expect = int(((np.minimum(st.pos[layer], R) + st.bank_fill[layer]) * 1024).sum() + B * 24576)
            assert tr.launch_bytes(layer) == expect, f"step {t} layer {layer}"
            oracle.decode_step(st, layer, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                               x["cand_score"], to_np(w[layer]), to_np(b[layer]))
            oracle.admit(st, layer)
            tr.advance(layer)
            assert np.array_equal(tr.pos[layer], st.pos[layer])
            assert np.array_equal(tr.bank[layer], st.bank_fill[layer])
            assert np.array_equal(tr.pend[layer], st.pend_fill[layer])


def test_fill_tracker_full_state_is_the_published_per_step_figure():
    cnt = np.zeros((8, 512, 4, 4), dtype=np.int64)
    cnt[..., 0] = 131_072
    cnt[..., 1] = 1024
    tr = bench.FillTracker(cnt)
    assert tr.launch_bytes(0) == 512 * bench.BYTES_FULL == 512 * 8_409_088


def test_admitted_counts_match_the_oracle_admit():
    """`bench.admitted_counts` (the admit workload's byte count) against the oracle's own admit on
    groups with every slot filled and 16-level scores (many ties, so the tie-break decides): the
    bank rows the admit replaced are the admitted candidates."""
    R, A, P, L, B, G = 5, 40, 12, 1, 6, 4
    cfg = oracle.Config(batch=B, n_layers=L, ring_slots=R, bank_slots=A, pend_slots=P)
    cont = si.state_contents(L, B, G, 256, R, A, P, seed=11, quantized_scores=True)
    st = oracle.state_from_arrays(cfg, {k: to_np(v) for k, v in cont.items()}, pos=100, bank_fill=A, pend_fill=P)
    counts = bench.admitted_counts(st.bank_score.copy(), st.pend_score.copy())
    before = st.bank_k.copy()
    oracle.admit(st, 0)
    replaced = (st.bank_k != before).any(axis=-1).sum(axis=-1)
    assert counts.shape == (L, B, G)
    assert np.array_equal(counts, replaced)
    assert 0 < counts.min() and counts.max() < P
