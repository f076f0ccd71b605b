"""Robustness of the state handling, on the GPU, with every failure made on the host.

* Checkpoint and restore: the state is one caller-owned buffer of fixed size
  ("EdgeRock" model card, "Constant history and GPU memory": one fixed-size
  allocation per sequence), so copying that buffer is a complete checkpoint.
  Decode steps and a prefill block run after a copy is taken; the copy is put
  back and the same calls run again: outputs and state agree bit for bit.
* Corrupted counters: counters written out of range on the host (as a damaged
  restore would leave them) make decode, admit and prefill raise
  RMA_STATUS_BAD_COUNTERS, clamp for their own indexing, and write nothing
  outside the state buffer or the output tensor (guard bytes on both sides of
  each stay as they were); a fresh state afterwards still matches the oracle.

No test here faults, traps or hangs a GPU: the bad values stay within what the
kernels' own range checks turn into a status bit.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from _gpu import TOL, assert_state_equal, decode_inputs_gpu, gpu_config, gpu_state_np, lib, make_pair, output_error
from _util import to_np

pytestmark = pytest.mark.gpu

GUARD = 4096           # bytes of canary on each side of a guarded buffer
CANARY = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bounded_memory_attention_b200 import build
    build.build()


def _guarded_state(cfg, seed, pos, bank_fill, pend_fill):
    """A GPU state laid over the middle of a larger allocation whose margins hold a canary."""
    rma = lib()
    gcfg = gpu_config(cfg)
    n = rma.state_bytes(gcfg)
    raw = torch.full((n + 2 * GUARD + 256,), CANARY, dtype=torch.uint8, device="cuda")
    off = GUARD + (-(raw.data_ptr() + GUARD)) % 256
    st = rma.State(gcfg, buffer=raw[off:off + n])
    contents = si.state_contents(cfg.n_layers, cfg.batch, cfg.n_groups, cfg.head_dim, cfg.ring_slots,
                                 cfg.bank_slots, cfg.pend_slots, seed=seed)
    for name, t in contents.items():
        getattr(st, name).copy_(t)
    shape = (cfg.n_layers, cfg.batch, cfg.n_groups)
    cnt = np.zeros(shape + (4,), np.int32)
    cnt[..., 0] = np.broadcast_to(np.asarray(pos), shape)
    cnt[..., 1] = np.broadcast_to(np.asarray(bank_fill), shape)
    cnt[..., 2] = np.broadcast_to(np.asarray(pend_fill), shape)
    st.counters.copy_(torch.from_numpy(cnt))
    torch.cuda.synchronize()
    return st, raw, off, n


def _guarded_out(shape):
    """An output tensor with canary elements on both sides; returns (whole, view)."""
    numel = int(np.prod(shape))
    pad = GUARD // 2
    whole = torch.empty(numel + 2 * pad, dtype=torch.bfloat16, device="cuda")
    whole.view(torch.int16).fill_(0x5A5A)
    return whole, whole[pad:pad + numel].view(*shape)


def _margins_intact(raw, off, n):
    head = raw[:off].cpu().numpy()
    tail = raw[off + n:].cpu().numpy()
    return bool((head == CANARY).all() and (tail == CANARY).all())


def _out_margins_intact(whole, numel):
    pad = GUARD // 2
    w = whole.view(torch.int16).cpu().numpy()
    return bool((w[:pad] == 0x5A5A).all() and (w[pad + numel:] == 0x5A5A).all())


def test_checkpoint_restore_replays_bit_identically():
    """Copy the state buffer, run decode steps (through admits) and a prefill block, restore, run again."""
    rma = lib()
    cfg = oracle.Config(batch=4, n_layers=2)
    pos = np.array([300, 1500, 131_072, 5])[None, :, None].repeat(2, 0).repeat(4, 2)
    bank = np.array([0, 700, 1024, 1024])[None, :, None].repeat(2, 0).repeat(4, 2)
    pend = np.array([250, 10, 255, 0])[None, :, None].repeat(2, 0).repeat(4, 2)
    st, _ = make_pair(cfg, seed=21, pos=pos, bank_fill=bank, pend_fill=pend)
    w, b = si.gate_params(2, 16, 256, seed=21)
    w, b = w.cuda(), si.f32_normal((2, 16), 22, std=0.5).cuda()
    ws1, wsp = st.workspace(1), st.workspace(100)
    out = torch.empty(4, 16, 256, dtype=torch.bfloat16, device="cuda")
    outp = torch.empty(4, 100, 16, 256, dtype=torch.bfloat16, device="cuda")
    xp = {k: v.cuda() for k, v in si.prefill_inputs(4, 100, 4, 4, 256, seed=23).items()}

    # N steps before the checkpoint
    for t in range(5):
        for layer in (0, 1):
            x = decode_inputs_gpu(cfg, seed=50_000 + 10 * t + layer)
            rma.decode_step(st, layer, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"],
                            w[layer], b[layer], out, ws1)
    torch.cuda.synchronize()
    snap = st.buffer.clone()

    def run_after():
        outs = []
        for t in range(12):          # crosses the admit of every group whose pending started at 250 / 255
            for layer in (0, 1):
                x = decode_inputs_gpu(cfg, seed=60_000 + 10 * t + layer)
                rma.decode_step(st, layer, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                                x["cand_score"], w[layer], b[layer], out, ws1)
                outs.append(out.clone())
            if t == 6:
                rma.prefill_block(st, 1, xp["q"], xp["k"], xp["v"], xp["cand_k"], xp["cand_v"], xp["cand_score"],
                                  w[1], b[1], outp, wsp)
                outs.append(outp.clone())
        torch.cuda.synchronize()
        return outs, st.buffer.clone()

    outs1, state1 = run_after()
    st.buffer.copy_(snap)                    # restore the checkpoint
    torch.cuda.synchronize()
    outs2, state2 = run_after()
    assert len(outs1) == len(outs2)
    for i, (a, c) in enumerate(zip(outs1, outs2)):
        assert torch.equal(a, c), f"call {i}: outputs differ after restore"
    assert torch.equal(state1, state2), "state bytes differ after restore"
    assert not torch.equal(state1, snap), "the calls after the checkpoint changed nothing"
    assert rma.get_status(st) == 0


@pytest.mark.parametrize("which", ["decode", "admit", "prefill"])
def test_corrupted_counters_raise_flag_and_stay_in_bounds(which):
    rma = lib()
    cfg = oracle.Config(batch=4, n_layers=1)
    # sequence 0 is sound; 1-3 carry counters no library call leaves behind
    pos = np.array([[[2000] * 4, [-7, 3000, 3000, 3000], [4000] * 4, [5000] * 4]])
    bank = np.array([[[1024] * 4, [1024] * 4, [5000, -1, 1024, 1024], [1024] * 4]])
    pend = np.array([[[3] * 4, [3] * 4, [3] * 4, [256, 999, -5, 1 << 30]]])
    st, raw, off, n = _guarded_state(cfg, seed=31, pos=pos, bank_fill=bank, pend_fill=pend)
    w, b = si.gate_params(1, 16, 256, seed=31)
    w, b = w[0].cuda(), b[0].cuda()
    if which == "decode":
        whole, out = _guarded_out((4, 16, 256))
        x = decode_inputs_gpu(cfg, seed=70_000)
        rma.decode_step(st, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"], w, b,
                        out, st.workspace(1))
        numel = out.numel()
    elif which == "admit":
        rma.admit(st, 0, force=True)
        whole, numel = None, 0
    else:
        whole, out = _guarded_out((4, 64, 16, 256))
        xp = {k: v.cuda() for k, v in si.prefill_inputs(4, 64, 4, 4, 256, seed=32).items()}
        rma.prefill_block(st, 0, xp["q"], xp["k"], xp["v"], xp["cand_k"], xp["cand_v"], xp["cand_score"], w, b,
                          out, st.workspace(64))
        numel = out.numel()
    torch.cuda.synchronize()
    flags = rma.get_status(st)
    assert flags & rma.STATUS_BAD_COUNTERS, f"{which}: flags {flags:#x}"
    assert not flags & rma.STATUS_TIMEOUT
    assert _margins_intact(raw, off, n), f"{which} wrote outside the state buffer"
    if whole is not None:
        assert _out_margins_intact(whole, numel), f"{which} wrote outside the output tensor"

    # the context is healthy: a sound state still matches the oracle
    cfg2 = oracle.Config(batch=2, n_layers=1)
    st2, ost2 = make_pair(cfg2, seed=33, pos=900, bank_fill=600, pend_fill=7)
    x = decode_inputs_gpu(cfg2, seed=70_001)
    out2 = torch.empty(2, 16, 256, dtype=torch.bfloat16, device="cuda")
    rma.decode_step(st2, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"], w, b, out2,
                    st2.workspace(1))
    xn = {k: to_np(v) for k, v in x.items()}
    ref = oracle.decode_step(ost2, 0, xn["q"], xn["k_cur"], xn["v_cur"], xn["cand_k"], xn["cand_v"],
                             xn["cand_score"], to_np(w), to_np(b))
    assert output_error(to_np(out2), ref) <= TOL
    assert_state_equal(gpu_state_np(st2), ost2, "sound state after the corrupted one")
    assert rma.get_status(st2) == 0
