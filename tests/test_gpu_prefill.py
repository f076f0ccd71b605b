"""GPU parity: rma_prefill_block (tcgen05 attention, commit, forced admit) against the oracle.

Outputs within 1e-2 max(1, |oracle|) element by element; the whole state
(ring, bank, scores, pending, counters) bit-exact after every block.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from _gpu import TOL, assert_state_equal, gpu_state_np, lib, make_pair, output_error
from _util import to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _block_both(rma, st, ost, layer, seed, w, b, ws, quantized=False, n=None, guard=0):
    """One block of n tokens (default pend_slots) through both sides; with guard > 0 the output
    sits at the front of a larger buffer whose tail must come back untouched."""
    cfg = st.cfg
    n = cfg.pend_slots if n is None else n
    x = si.prefill_inputs(cfg.batch, n, cfg.n_groups, cfg.q_per_group, cfg.head_dim, seed=seed,
                          quantized_scores=quantized)
    xd = {k: v.cuda() for k, v in x.items()}
    shape = (cfg.batch, n, cfg.n_groups * cfg.q_per_group, cfg.head_dim)
    numel = int(np.prod(shape))
    buf = torch.full((numel + guard,), -7.0, dtype=torch.bfloat16, device="cuda")
    out = buf[:numel].view(shape)
    rma.prefill_block(st, layer, xd["q"], xd["k"], xd["v"], xd["cand_k"], xd["cand_v"], xd["cand_score"],
                      w, b, out, ws)
    if guard:
        assert bool((buf[numel:] == -7.0).all()), "a store landed past the block's output"
    xn = {k: to_np(v) for k, v in x.items()}
    ref = oracle.prefill_block(ost, layer, xn["q"], xn["k"], xn["v"], xn["cand_k"], xn["cand_v"],
                               xn["cand_score"], to_np(w), to_np(b))
    torch.cuda.synchronize()
    return to_np(out), ref


def test_prefill_from_empty_state_five_blocks():
    """Blocks at s = 0, 256, 512, 768, 1024: empty, partial, full and wrapped rings; the bank fills by admits."""
    rma = lib()
    cfg = oracle.Config(batch=2, n_layers=1)
    st, ost = make_pair(cfg, seed=21, **si.workload_counters("empty", 1, 2, 4))
    w, b = si.gate_params(1, 16, 256, seed=21)
    w, b = w[0].cuda(), si.f32_normal((16,), 22, std=0.5).cuda()
    ws = st.workspace(256)
    for blk in range(5):
        g_out, ref = _block_both(rma, st, ost, 0, 500 + blk, w, b, ws)
        err = output_error(g_out, ref)
        assert err <= TOL, f"block {blk}: output error {err}"
        assert_state_equal(gpu_state_np(st), ost, f"block {blk}")
        assert rma.get_status(st) == 0, f"block {blk}"


def test_prefill_on_long_history_with_quantized_scores():
    """Ring full at an arbitrary rotation (pos = 131,089), bank full, ties in the admit."""
    rma = lib()
    cfg = oracle.Config(batch=3, n_layers=2)
    st, ost = make_pair(cfg, seed=23, pos=131_089, bank_fill=1024, pend_fill=0, quantized=True)
    w, b = si.gate_params(2, 16, 256, seed=23)
    w, b = w.cuda(), b.cuda()
    ws = st.workspace(256)
    for blk in range(3):
        for layer in (1, 0):
            g_out, ref = _block_both(rma, st, ost, layer, 600 + 2 * blk + layer, w[layer], b[layer], ws,
                                     quantized=True)
            err = output_error(g_out, ref)
            assert err <= TOL, f"block {blk} layer {layer}: output error {err}"
        assert_state_equal(gpu_state_np(st), ost, f"block {blk}")


def test_prefill_partial_bank_and_small_block():
    """P = 64 (two tiles per block), bank partly filled, ring partly filled."""
    rma = lib()
    cfg = oracle.Config(batch=2, n_layers=1, pend_slots=64, bank_slots=300, ring_slots=200)
    st, ost = make_pair(cfg, seed=25, pos=[[[70] * 4, [450] * 4]], bank_fill=[[[0] * 4, [137] * 4]],
                        pend_fill=0)
    w, b = si.gate_params(1, 16, 256, seed=25, std=0.2)
    w, b = w[0].cuda(), si.f32_normal((16,), 26, std=0.5).cuda()
    ws = st.workspace(64)
    for blk in range(6):
        g_out, ref = _block_both(rma, st, ost, 0, 700 + blk, w, b, ws)
        err = output_error(g_out, ref)
        assert err <= TOL, f"block {blk}: output error {err}"
        assert_state_equal(gpu_state_np(st), ost, f"block {blk}")


def test_prefill_candidates_that_do_not_fit_are_flagged():
    rma = lib()
    cfg = oracle.Config(batch=1, n_layers=1)
    st, ost = make_pair(cfg, seed=27, pos=5000, bank_fill=1000, pend_fill=3)
    w, b = si.gate_params(1, 16, 256, seed=27)
    w, b = w[0].cuda(), b[0].cuda()
    g_out, ref = _block_both(rma, st, ost, 0, 800, w, b, st.workspace(256))
    assert output_error(g_out, ref) <= TOL
    assert_state_equal(gpu_state_np(st), ost, "overflow block")
    assert rma.get_status(st) == rma.STATUS_PREFILL_PENDING_OVERFLOW
    assert ost.status == oracle.STATUS_PREFILL_PENDING_OVERFLOW


def test_prefill_then_decode_handoff():
    """A prefill block leaves pending empty; decode steps continue from it with the oracle in step."""
    rma = lib()
    cfg = oracle.Config(batch=2, n_layers=1)
    st, ost = make_pair(cfg, seed=29, pos=700, bank_fill=512, pend_fill=0)
    w, b = si.gate_params(1, 16, 256, seed=29)
    w, b = w[0].cuda(), b[0].cuda()
    g_out, ref = _block_both(rma, st, ost, 0, 900, w, b, st.workspace(256))
    assert output_error(g_out, ref) <= TOL
    ws1 = st.workspace(1)
    out = torch.empty(2, 16, 256, dtype=torch.bfloat16, device="cuda")
    for t in range(5):
        x = {k: v.cuda() for k, v in si.decode_inputs(2, 4, 4, 256, seed=950 + t).items()}
        rma.decode_step(st, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"],
                        w, b, out, ws1)
        rma.admit(st, 0)
        xn = {k: to_np(v) for k, v in x.items()}
        r = oracle.decode_step(ost, 0, xn["q"], xn["k_cur"], xn["v_cur"], xn["cand_k"], xn["cand_v"],
                               xn["cand_score"], to_np(w), to_np(b))
        oracle.admit(ost, 0)
        assert output_error(to_np(out), r) <= TOL
    assert_state_equal(gpu_state_np(st), ost, "after handoff")


def test_prefill_rescales_when_scores_keep_rising():
    """Keys along the queries' direction with growing magnitude: the running max of every row moves
    many times (ring slots, then the block, then a rising bank), so O and the row sums are rescaled
    repeatedly, in both query groups."""
    rma = lib()
    cfg = oracle.Config(batch=2, n_layers=1)
    st, ost = make_pair(cfg, seed=31, pos=3000, bank_fill=1024, pend_fill=0)
    L, B, G, D = 1, cfg.batch, cfg.n_groups, cfg.head_dim
    ring_k = si.aligned_ramp((L, B, G), cfg.ring_slots, D, seed=310, lo=0.0, hi=1.5)
    bank_k = si.aligned_ramp((L, B, G), cfg.bank_slots, D, seed=310, lo=-0.5, hi=2.0)
    for name, t in (("ring_k", ring_k), ("bank_k", bank_k)):
        getattr(st, name).copy_(t)
        getattr(ost, name)[...] = to_np(t)
    n = cfg.pend_slots
    x = si.prefill_inputs(B, n, G, cfg.q_per_group, D, seed=311)
    x["q"] = si.aligned_ramp((B,), n * G * cfg.q_per_group, D, seed=310, lo=1.0, hi=1.0).reshape(
        B, n, G * cfg.q_per_group, D)
    x["k"] = si.aligned_ramp((B, G), n, D, seed=310, lo=1.5, hi=2.5).permute(0, 2, 1, 3).contiguous()
    w, b = si.gate_params(1, 16, 256, seed=31)
    w, b = w[0].cuda(), si.f32_normal((16,), 32, std=0.5).cuda()
    xd = {k: v.cuda() for k, v in x.items()}
    out = torch.empty(B, n, G * cfg.q_per_group, D, dtype=torch.bfloat16, device="cuda")
    rma.prefill_block(st, 0, xd["q"], xd["k"], xd["v"], xd["cand_k"], xd["cand_v"], xd["cand_score"], w, b, out,
                      st.workspace(n))
    xn = {k: to_np(v) for k, v in x.items()}
    ref = oracle.prefill_block(ost, 0, xn["q"], xn["k"], xn["v"], xn["cand_k"], xn["cand_v"], xn["cand_score"],
                               to_np(w), to_np(b))
    torch.cuda.synchronize()
    err = output_error(to_np(out), ref)
    assert err <= TOL, f"output error {err}"
    assert_state_equal(gpu_state_np(st), ost, "rising scores")
    assert rma.get_status(st) == 0


def test_prefill_ragged_block_lengths():
    """Blocks of 100, 1, 17, 63, 64, 65, 129, 200, 255, 33 and 256 tokens on sequences that start
    with an empty, a partly filled and a wrapped ring, an empty, partial and full bank, and 0, 17
    and 200 pending candidates (the first block's do not fit for the last sequence only)."""
    rma = lib()
    cfg = oracle.Config(batch=3, n_layers=1)
    per_seq = lambda vals: [[[v] * 4 for v in vals]]
    st, ost = make_pair(cfg, seed=33, pos=per_seq([0, 777, 131_089]), bank_fill=per_seq([0, 300, 1024]),
                        pend_fill=per_seq([0, 17, 200]))
    w, b = si.gate_params(1, 16, 256, seed=33)
    w, b = w[0].cuda(), si.f32_normal((16,), 34, std=0.5).cuda()
    status = 0
    for blk, n in enumerate((100, 1, 17, 63, 64, 65, 129, 200, 255, 33, 256)):
        ws = st.workspace(n)
        g_out, ref = _block_both(rma, st, ost, 0, 1000 + blk, w, b, ws, n=n, guard=4096)
        err = output_error(g_out, ref)
        assert err <= TOL, f"block {blk} (n = {n}): output error {err}"
        assert_state_equal(gpu_state_np(st), ost, f"block {blk} (n = {n})")
        status |= rma.get_status(st)
        if blk == 0:
            assert status == rma.STATUS_PREFILL_PENDING_OVERFLOW
    assert status == ost.status == oracle.STATUS_PREFILL_PENDING_OVERFLOW


def test_prompt_of_300_tokens_then_decode_then_more_prefill():
    """A 300-token prompt as blocks of 256 and 44; 30 decode steps; a 100-token block that starts
    with 30 pending candidates (they fit, the forced admit takes 130); 5 decode steps; a 255-token
    block whose candidates do not fit next to the 5 pending ones (dropped and flagged)."""
    rma = lib()
    cfg = oracle.Config(batch=2, n_layers=1)
    st, ost = make_pair(cfg, seed=35, **si.workload_counters("empty", 1, 2, 4))
    w, b = si.gate_params(1, 16, 256, seed=35)
    w, b = w[0].cuda(), si.f32_normal((16,), 36, std=0.5).cuda()
    ws1 = st.workspace(1)
    out1 = torch.empty(2, 16, 256, dtype=torch.bfloat16, device="cuda")
    seed = [1100]

    def prefill(n, what):
        seed[0] += 1
        g_out, ref = _block_both(rma, st, ost, 0, seed[0], w, b, st.workspace(n), n=n, guard=256)
        err = output_error(g_out, ref)
        assert err <= TOL, f"{what}: output error {err}"
        assert_state_equal(gpu_state_np(st), ost, what)

    def decode(steps, what):
        for t in range(steps):
            seed[0] += 1
            x = {k: v.cuda() for k, v in si.decode_inputs(2, 4, 4, 256, seed=seed[0]).items()}
            rma.decode_step(st, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"],
                            w, b, out1, ws1)
            rma.admit(st, 0)
            xn = {k: to_np(v) for k, v in x.items()}
            r = oracle.decode_step(ost, 0, xn["q"], xn["k_cur"], xn["v_cur"], xn["cand_k"], xn["cand_v"],
                                   xn["cand_score"], to_np(w), to_np(b))
            oracle.admit(ost, 0)
            err = output_error(to_np(out1), r)
            assert err <= TOL, f"{what} step {t}: output error {err}"
        assert_state_equal(gpu_state_np(st), ost, what)

    prefill(256, "prompt block 1")
    prefill(44, "prompt block 2 (44 tokens)")
    assert rma.get_status(st) == 0
    decode(30, "30 decode steps")
    assert int(st.counters[0, 0, 0, 2]) == 30 and int(st.counters[0, 0, 0, 0]) == 330
    prefill(100, "100-token block after decode")
    assert int(st.counters[0, 0, 0, 2]) == 0 and int(st.counters[0, 0, 0, 1]) == 430
    assert rma.get_status(st) == 0
    decode(5, "5 more decode steps")
    prefill(255, "255-token block that overflows pending")
    assert rma.get_status(st) == rma.STATUS_PREFILL_PENDING_OVERFLOW
    assert ost.status == oracle.STATUS_PREFILL_PENDING_OVERFLOW
    assert int(st.counters[0, 0, 0, 0]) == 690


def test_prefill_block_length_checks():
    """Lengths the library refuses on the host, before any launch, and the workspace sizes."""
    rma = lib()
    cfg = rma.Config(batch=1, n_layers=1, ring_slots=100)
    st = rma.State(cfg)
    # a block's workspace never shrinks with its length; a decode step's (n_tok = 1) is positive
    assert st.workspace_bytes(256) >= st.workspace_bytes(100) > 0 and st.workspace_bytes(1) > 0
    for n, code in ((0, "RMA_ERR_INVALID_ARG"), (257, "RMA_ERR_UNSUPPORTED")):
        with pytest.raises(rma.RmaError) as e:
            st.workspace_bytes(n)
        assert rma.ERRORS[e.value.code] == code
    w = torch.zeros(16, 256, device="cuda")
    bias = torch.zeros(16, device="cuda")
    ws = st.workspace(256)
    for n, code in ((101, "RMA_ERR_UNSUPPORTED"), (257, "RMA_ERR_UNSUPPORTED")):
        x = {k: v.cuda() for k, v in si.prefill_inputs(1, n, 4, 4, 256, seed=5).items()}
        out = torch.empty(1, n, 16, 256, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(rma.RmaError) as e:
            rma.prefill_block(st, 0, x["q"], x["k"], x["v"], x["cand_k"], x["cand_v"], x["cand_score"],
                              w, bias, out, ws)
        assert rma.ERRORS[e.value.code] == code, n
    assert int(st.counters.abs().sum()) == 0
    assert rma.get_status(st) == 0
