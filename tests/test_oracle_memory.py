"""Pin the oracle's state dimensions to the byte counts the pages print.

Check (a): per sequence over 8 RMA layers, committed anchors 32.00 MiB, pending
candidates 8.00 MiB, local window 31.97 MiB, about 72 MiB together; the source
model's 32 KiB per token, 2 GiB at 64K tokens, ~1 TiB at 512 sequences, 8 GiB
at 256K; the 99.1% reduction.  A wrong slot count (1,024 ring slots), head_dim,
group count or a dropped K/V factor fails one of these.
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth_inputs as si
from _util import inputs_np

MiB = 2 ** 20
GiB = 2 ** 30
TiB = 2 ** 40


@pytest.fixture(scope="module")
def golden(golden_dir):
    with open(os.path.join(golden_dir, "memory_accounting.json")) as f:
        return json.load(f)


def _printed(value, decimals):
    return round(value, decimals)


def test_component_bytes_match_printed_mib(golden):
    dims = golden["dimensions"]
    b = oracle.attention_kv_bytes_per_sequence(
        n_layers=dims["rma_layers"]["value"], n_groups=dims["kv_groups"]["value"], head_dim=256,
        ring_slots=dims["ring_stored_positions"]["value"], bank_slots=dims["anchors_per_group"]["value"],
        pend_slots=dims["pending_positions"]["value"])
    g = golden["mib_per_sequence"]
    assert _printed(b["committed_anchors"] / MiB, 2) == g["committed_anchors"]["value"]
    assert _printed(b["pending_candidates"] / MiB, 2) == g["pending_candidates"]["value"]
    assert _printed(b["local_window"] / MiB, 2) == g["local_window"]["value"]
    # exact byte counts (integers): 8*4*1024*1024, 8*4*256*1024, 8*4*1023*1024
    assert b["committed_anchors"] == 33_554_432
    assert b["pending_candidates"] == 8_388_608
    assert b["local_window"] == 33_521_664
    total = sum(b.values())
    assert _printed(total / MiB, 0) == golden["attention_kv_mib_per_sequence"]["value"]


def test_table_total_is_consistent(golden):
    b = oracle.attention_kv_bytes_per_sequence()
    g = golden["mib_per_sequence"]
    others = g["recurrent_matrices"]["value"] + g["convolution_state"]["value"] + g["metadata"]["value"]
    assert _printed(sum(b.values()) / MiB + others, 2) == g["total_persistent_history"]["value"]


def test_window_is_ring_plus_current(golden):
    d = golden["dimensions"]
    assert d["ring_stored_positions"]["value"] + 1 == d["window_positions"]["value"]
    cfg = oracle.Config()
    assert cfg.ring_slots + 1 == d["window_positions"]["value"]
    assert cfg.bank_slots == d["anchors_per_group"]["value"]
    assert cfg.pend_slots == d["pending_positions"]["value"] == d["commit_interval"]["value"]
    assert cfg.n_groups == d["kv_groups"]["value"]


def test_source_model_kv_figures(golden):
    per_tok = oracle.full_attention_kv_bytes_per_token(n_layers=8, n_kv_heads=4, head_dim=256)
    assert per_tok == golden["source_model_kv_kib_per_token"]["value"] * 1024
    assert per_tok * 65536 == golden["source_model_gib_per_sequence_64k"]["value"] * GiB
    assert per_tok * 65536 * 512 == golden["source_model_tib_at_512_sequences"]["value"] * TiB
    assert per_tok * 262144 == golden["source_model_gib_at_256k"]["value"] * GiB


def test_reduction_at_256k(golden):
    rma = sum(oracle.attention_kv_bytes_per_sequence().values())
    full = oracle.full_attention_kv_bytes_per_token() * 262144
    assert _printed(100.0 * (1.0 - rma / full), 1) == golden["reduction_percent_at_256k"]["value"]
    # with the rounded 72 MiB the pages quote, the same figure
    assert _printed(100.0 * (1.0 - 72 * MiB / full), 1) == golden["reduction_percent_at_256k"]["value"]


def test_state_size_constant_in_sequence_length():
    """Check (e), storage side: the oracle's arrays do not depend on how many tokens were seen."""
    cfg = oracle.Config(batch=1, n_layers=1, n_groups=1, q_per_group=1, head_dim=8,
                        ring_slots=5, bank_slots=4, pend_slots=2)
    st = oracle.new_state(cfg)
    shapes0 = {k: getattr(st, k).shape for k in ("ring_k", "bank_k", "pend_k", "bank_score", "pend_score")}
    w = np.zeros((1, 8), np.float32)
    bg = np.zeros(1, np.float32)
    for t in range(40):
        x = inputs_np(si.decode_inputs(1, 1, 1, 8, seed=t))
        oracle.decode_step(st, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                           x["cand_score"], w, bg)
        oracle.admit(st, 0)
    assert int(st.pos[0, 0, 0]) == 40
    assert {k: getattr(st, k).shape for k in shapes0} == shapes0
