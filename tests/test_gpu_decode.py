"""GPU parity: rma_decode_step + rma_admit against the oracle, through the C ABI.

Outputs: |gpu - oracle| <= 1e-2 max(1, |oracle|) element by element.
State (ring, bank, scores, pending, counters): bit-exact after every checked step.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from _gpu import TOL, assert_state_equal, decode_inputs_gpu, gpu_state_np, lib, make_pair, output_error
from _util import to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bounded_memory_attention_b200 import build
    build.build()


def _step_both(rma, st, ost, ws, layer, x, w, b, out):
    rma.decode_step(st, layer, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"],
                    w, b, out, ws)
    rma.admit(st, layer)
    xn = {k: to_np(v) for k, v in x.items()}
    ref = oracle.decode_step(ost, layer, xn["q"], xn["k_cur"], xn["v_cur"], xn["cand_k"], xn["cand_v"],
                             xn["cand_score"], to_np(w), to_np(b))
    oracle.admit(ost, layer)
    return to_np(out), ref


def test_tiny_decode_config_full_parity():
    """Batch 1, one layer, ring pre-filled with 1,023 positions, bank full, 512 steps -> 2 admits."""
    rma = lib()
    cfg = oracle.Config(batch=1, n_layers=1)
    c = si.workload_counters("tiny", 1, 1, 4)
    st, ost = make_pair(cfg, seed=0, **c)
    w, b = si.gate_params(1, 16, 256, seed=0)
    w, b = w[0].cuda(), b[0].cuda()
    ws = st.workspace(1)
    out = torch.empty(1, 16, 256, dtype=torch.bfloat16, device="cuda")
    worst = 0.0
    check_full = set(range(4)) | set(range(250, 262)) | {510, 511} | set(range(0, 512, 32))
    for t in range(512):
        x = decode_inputs_gpu(cfg, seed=10_000 + t)
        g_out, ref = _step_both(rma, st, ost, ws, 0, x, w, b, out)
        err = output_error(g_out, ref)
        worst = max(worst, err)
        assert err <= TOL, f"step {t}: output error {err}"
        if t in check_full:
            assert_state_equal(gpu_state_np(st), ost, f"step {t}")
    assert int(ost.bank_fill[0, 0, 0]) == 1024 and int(ost.pos[0, 0, 0]) == 1023 + 512
    assert rma.get_status(st) == 0
    print(f"tiny decode: worst output error {worst:.3e}")


# None is the default shape for this batch; (1, 1), (2, 3) and (8, 8) are the defaults the split
# heuristic picks at other batch sizes (16 and up, 8, and 1 or 2); (5, 5) and (1, 2) were earlier
# defaults and stay as extra shapes
@pytest.mark.parametrize("splits", [None, (1, 1), (3, 5), (16, 16), (32, 32), (1, 63), (5, 5), (2, 3), (1, 2), (8, 8)])
def test_ragged_fills_every_split_shape(splits):
    """Partial windows, empty and partial banks, pending about to fill; quantised scores force ties."""
    rma = lib()
    cfg = oracle.Config(batch=6, n_layers=2)
    pos = np.array([0, 1, 500, 1022, 5000, 131_071])[None, :, None].repeat(2, 0).repeat(4, 2)
    bank = np.array([0, 1, 777, 1024, 3, 1024])[None, :, None].repeat(2, 0).repeat(4, 2)
    pend = np.array([0, 255, 17, 254, 255, 100])[None, :, None].repeat(2, 0).repeat(4, 2)
    pos[1] = pos[1][::-1]
    st, ost = make_pair(cfg, seed=1, pos=pos, bank_fill=bank, pend_fill=pend, quantized=True)
    if splits is not None:
        rma.set_decode_splits(st, *splits)
    w, b = si.gate_params(2, 16, 256, seed=1)
    b = si.f32_normal((2, 16), 77, std=0.5)
    w, b = w.cuda(), b.cuda()
    ws = st.workspace(1)
    out = torch.empty(6, 16, 256, dtype=torch.bfloat16, device="cuda")
    for t in range(4):
        for layer in (0, 1):
            x = decode_inputs_gpu(cfg, seed=20_000 + 10 * t + layer, quantized=True)
            g_out, ref = _step_both(rma, st, ost, ws, layer, x, w[layer], b[layer], out)
            err = output_error(g_out, ref)
            assert err <= TOL, f"step {t} layer {layer}: output error {err}"
        assert_state_equal(gpu_state_np(st), ost, f"step {t}")
    assert rma.get_status(st) == 0


def test_small_state_many_admits_and_wraps():
    """R = 37, A = 20, P = 8: the ring wraps and the admit runs every 8 steps."""
    rma = lib()
    cfg = oracle.Config(batch=3, n_layers=1, ring_slots=37, bank_slots=20, pend_slots=8, softmax_scale=0.09)
    st, ost = make_pair(cfg, seed=2, pos=[[[0], [5], [40]]], bank_fill=[[[0], [20], [7]]],
                        pend_fill=[[[0], [3], [7]]], quantized=True)
    w, b = si.gate_params(1, 16, 256, seed=2, std=0.2)
    w, b = w[0].cuda(), si.f32_normal((16,), 5, std=0.3).cuda()
    ws = st.workspace(1)
    out = torch.empty(3, 16, 256, dtype=torch.bfloat16, device="cuda")
    for t in range(90):
        x = decode_inputs_gpu(cfg, seed=30_000 + t, quantized=True)
        g_out, ref = _step_both(rma, st, ost, ws, 0, x, w, b, out)
        assert output_error(g_out, ref) <= TOL, f"step {t}"
        assert_state_equal(gpu_state_np(st), ost, f"step {t}")


def test_pending_overflow_sets_status_and_drops_candidate():
    rma = lib()
    cfg = oracle.Config(batch=2, n_layers=1)
    st, ost = make_pair(cfg, seed=3, pos=2000, bank_fill=1024, pend_fill=256)
    w, b = si.gate_params(1, 16, 256, seed=3)
    w, b = w[0].cuda(), b[0].cuda()
    ws = st.workspace(1)
    out = torch.empty(2, 16, 256, dtype=torch.bfloat16, device="cuda")
    x = decode_inputs_gpu(cfg, seed=40_000)
    rma.decode_step(st, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"], w, b, out, ws)
    xn = {k: to_np(v) for k, v in x.items()}
    ref = oracle.decode_step(ost, 0, xn["q"], xn["k_cur"], xn["v_cur"], xn["cand_k"], xn["cand_v"],
                             xn["cand_score"], to_np(w), to_np(b))
    assert output_error(to_np(out), ref) <= TOL
    assert_state_equal(gpu_state_np(st), ost, "overflow step")
    assert rma.get_status(st) == rma.STATUS_PENDING_OVERFLOW == oracle.STATUS_PENDING_OVERFLOW
    assert rma.get_status(st) == 0   # read clears


def test_nan_score_at_admit_sets_status_and_ranks_last():
    rma = lib()
    cfg = oracle.Config(batch=1, n_layers=1)
    st, ost = make_pair(cfg, seed=4, pos=3000, bank_fill=1024, pend_fill=256)
    st.bank_score[0, 0, 1, 5] = float("nan")
    st.pend_score[0, 0, 2, 9] = float("nan")
    st.pend_score[0, 0, 3, 0] = -0.0
    st.bank_score[0, 0, 3, 0] = 0.0
    ost.bank_score[0, 0, 1, 5] = np.nan
    ost.pend_score[0, 0, 2, 9] = np.nan
    ost.pend_score[0, 0, 3, 0] = -0.0
    ost.bank_score[0, 0, 3, 0] = 0.0
    rma.admit(st, 0)
    oracle.admit(ost, 0)
    assert_state_equal(gpu_state_np(st), ost, "admit with NaN")
    assert rma.get_status(st) == rma.STATUS_NAN_SCORE
    assert ost.status == oracle.STATUS_NAN_SCORE


@pytest.mark.parametrize("force", [False, True])
def test_admit_alone_random_fills_bit_exact(force):
    rma = lib()
    cfg = oracle.Config(batch=16, n_layers=1)
    rng = np.random.default_rng(5)
    bank = rng.integers(0, 1025, size=(1, 16, 4))
    pend = np.where(rng.random((1, 16, 4)) < 0.5, 256, rng.integers(0, 256, size=(1, 16, 4)))
    st, ost = make_pair(cfg, seed=5, pos=4096, bank_fill=bank, pend_fill=pend, quantized=True)
    rma.admit(st, 0, force=force)
    oracle.admit(ost, 0, force=force)
    assert_state_equal(gpu_state_np(st), ost, f"admit force={force}")
