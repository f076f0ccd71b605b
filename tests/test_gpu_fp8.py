"""GPU parity for FP8 storage (E4M3 codes + per-row power-of-two scales), through the C ABI.

Contract: the state's codes, exponents, scores and counters are bit-exact with
the FP8 oracle after every checked step (quantisation of the ring write and the
candidate append, admit copies, rma_state_quantize); outputs are within
1e-2 max(1, |oracle|) of the FP8 oracle, which attends over the same stored
values in FP64.  How far FP8 storage moves the outputs from BF16 storage is a
property of the format, reported by test_fp8_storage_error_against_bf16
(not a parity bound).
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from _gpu import TOL, decode_inputs_gpu, gpu_config, lib, make_pair, output_error
from _util import to_np

pytestmark = pytest.mark.gpu

_ROWS = ("ring_k", "ring_v", "bank_k", "bank_v", "pend_k", "pend_v")


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bounded_memory_attention_b200 import build
    build.build()


def _fp8_config(cfg):
    c = gpu_config(cfg)
    c.kv_format = lib().KV_FP8_E4M3
    return c


def make_fp8_pair(cfg, seed, pos, bank_fill, pend_fill, quantized=False):
    """A GPU FP8 state and an oracle FP8 state holding the same codes, exponents, scores and counters
    (the quantisation of a seeded BF16 state, done by the oracle)."""
    rma = lib()
    contents = si.state_contents(cfg.n_layers, cfg.batch, cfg.n_groups, cfg.head_dim, cfg.ring_slots,
                                 cfg.bank_slots, cfg.pend_slots, seed=seed, quantized_scores=quantized)
    shape = (cfg.n_layers, cfg.batch, cfg.n_groups)
    cnt = np.zeros(shape + (4,), np.int32)
    cnt[..., 0] = np.broadcast_to(np.asarray(pos), shape)
    cnt[..., 1] = np.broadcast_to(np.asarray(bank_fill), shape)
    cnt[..., 2] = np.broadcast_to(np.asarray(pend_fill), shape)
    bst = oracle.state_from_arrays(cfg, {k: to_np(v) for k, v in contents.items()},
                                   pos=cnt[..., 0], bank_fill=cnt[..., 1], pend_fill=cnt[..., 2])
    ost = oracle.quantize_state(bst)
    st = rma.State(_fp8_config(cfg))
    for name in _ROWS:
        getattr(st, name).copy_(torch.from_numpy(getattr(ost, name)))
        getattr(st, name + "_exp").copy_(torch.from_numpy(getattr(ost, name + "_exp")))
    st.bank_score.copy_(torch.from_numpy(ost.bank_score))
    st.pend_score.copy_(torch.from_numpy(ost.pend_score))
    st.counters.copy_(torch.from_numpy(cnt))
    torch.cuda.synchronize()
    return st, ost


def fp8_state_np(st) -> dict:
    out = {}
    for name in _ROWS:
        out[name] = getattr(st, name).cpu().numpy()
        out[name + "_exp"] = getattr(st, name + "_exp").cpu().numpy()
    out["bank_score"] = st.bank_score.cpu().numpy()
    out["pend_score"] = st.pend_score.cpu().numpy()
    c = st.counters.cpu().numpy()
    out["pos"], out["bank_fill"], out["pend_fill"] = c[..., 0], c[..., 1], c[..., 2]
    return out


def assert_fp8_state_equal(gpu: dict, ost, what=""):
    for name in _ROWS:
        for key in (name, name + "_exp"):
            a, b = gpu[key], getattr(ost, key)
            if not np.array_equal(a, b):
                idx = np.argwhere(a != b)[0]
                raise AssertionError(f"{what}: {key} differs first at {tuple(idx)}: gpu {a[tuple(idx)]} "
                                     f"oracle {b[tuple(idx)]}")
    for name in ("bank_score", "pend_score"):
        assert np.array_equal(gpu[name].view(np.uint32), getattr(ost, name).view(np.uint32)), f"{what}: {name}"
    for name in ("pos", "bank_fill", "pend_fill"):
        assert np.array_equal(gpu[name].astype(np.int64), getattr(ost, name)), f"{what}: counter {name}"


def _step_both(rma, st, ost, ws, layer, x, w, b, out):
    rma.decode_step(st, layer, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"],
                    w, b, out, ws)
    rma.admit(st, layer)
    xn = {k: to_np(v) for k, v in x.items()}
    ref = oracle.decode_step_fp8(ost, layer, xn["q"], xn["k_cur"], xn["v_cur"], xn["cand_k"], xn["cand_v"],
                                 xn["cand_score"], to_np(w), to_np(b))
    oracle.admit_fp8(ost, layer)
    return to_np(out), ref


def test_quantize_entry_matches_the_oracle():
    """rma_state_quantize of a seeded BF16 state: codes, exponents, scores, counters bit-exact."""
    rma = lib()
    cfg = oracle.Config(batch=3, n_layers=2, ring_slots=37, bank_slots=40, pend_slots=9)
    src, osrc = make_pair(cfg, seed=41, pos=[[[5], [50], [1000]], [[0], [7], [37]]], bank_fill=13, pend_fill=4)
    # some rows that stress the scale: all zero, one huge value, tiny values, exact powers of two
    src.ring_k[0, 0, 0, 0].zero_()
    src.ring_k[0, 0, 0, 1, 7] = 3.0e38
    src.bank_v[1, 2, 3, 5] *= 1e-30
    src.pend_k[0, 1, 2, 3] = 448.0
    for name in ("ring_k", "bank_v", "pend_k"):
        getattr(osrc, name)[...] = to_np(getattr(src, name))
    dst = rma.State(_fp8_config(cfg))
    rma.state_quantize(dst, src)
    torch.cuda.synchronize()
    assert_fp8_state_equal(fp8_state_np(dst), oracle.quantize_state(osrc), "rma_state_quantize")


def test_tiny_decode_config_fp8_full_parity():
    """Batch 1, one layer, ring pre-filled with 1,023 positions, bank full, 512 steps -> 2 admits."""
    rma = lib()
    cfg = oracle.Config(batch=1, n_layers=1)
    c = si.workload_counters("tiny", 1, 1, 4)
    st, ost = make_fp8_pair(cfg, seed=0, **c)
    w, b = si.gate_params(1, 16, 256, seed=0)
    w, b = w[0].cuda(), b[0].cuda()
    ws = st.workspace(1)
    out = torch.empty(1, 16, 256, dtype=torch.bfloat16, device="cuda")
    worst = 0.0
    check_full = set(range(4)) | set(range(250, 262)) | {510, 511} | set(range(0, 512, 64))
    for t in range(512):
        x = decode_inputs_gpu(cfg, seed=10_000 + t)
        g_out, ref = _step_both(rma, st, ost, ws, 0, x, w, b, out)
        err = output_error(g_out, ref)
        worst = max(worst, err)
        assert err <= TOL, f"step {t}: output error {err}"
        if t in check_full:
            assert_fp8_state_equal(fp8_state_np(st), ost, f"step {t}")
    assert int(ost.pos[0, 0, 0]) == 1023 + 512 and int(ost.pend_fill[0, 0, 0]) == 0
    assert rma.get_status(st) == 0
    print(f"tiny FP8 decode: worst output error {worst:.3e}")


@pytest.mark.parametrize("splits", [None, (1, 1), (3, 5), (32, 32)])
def test_fp8_ragged_fills_every_split_shape(splits):
    rma = lib()
    cfg = oracle.Config(batch=6, n_layers=2)
    pos = np.array([0, 1, 500, 1022, 5000, 131_071])[None, :, None].repeat(2, 0).repeat(4, 2)
    bank = np.array([0, 1, 777, 1024, 3, 1024])[None, :, None].repeat(2, 0).repeat(4, 2)
    pend = np.array([0, 255, 17, 254, 255, 100])[None, :, None].repeat(2, 0).repeat(4, 2)
    pos[1] = pos[1][::-1]
    st, ost = make_fp8_pair(cfg, seed=1, pos=pos, bank_fill=bank, pend_fill=pend, quantized=True)
    if splits is not None:
        rma.set_decode_splits(st, *splits)
    w, b = si.gate_params(2, 16, 256, seed=1)
    w, b = w.cuda(), si.f32_normal((2, 16), 77, std=0.5).cuda()
    ws = st.workspace(1)
    out = torch.empty(6, 16, 256, dtype=torch.bfloat16, device="cuda")
    for t in range(4):
        for layer in (0, 1):
            x = decode_inputs_gpu(cfg, seed=20_000 + 10 * t + layer, quantized=True)
            g_out, ref = _step_both(rma, st, ost, ws, layer, x, w[layer], b[layer], out)
            err = output_error(g_out, ref)
            assert err <= TOL, f"step {t} layer {layer}: output error {err}"
        assert_fp8_state_equal(fp8_state_np(st), ost, f"step {t}")
    assert rma.get_status(st) == 0


def test_fp8_small_state_many_admits_and_wraps():
    """R = 37, A = 20, P = 8 (exponent arrays padded to 48 / 32 / 16 slots)."""
    rma = lib()
    cfg = oracle.Config(batch=3, n_layers=1, ring_slots=37, bank_slots=20, pend_slots=8, softmax_scale=0.09)
    st, ost = make_fp8_pair(cfg, seed=2, pos=[[[0], [5], [40]]], bank_fill=[[[0], [20], [7]]],
                            pend_fill=[[[0], [3], [7]]], quantized=True)
    w, b = si.gate_params(1, 16, 256, seed=2, std=0.2)
    w, b = w[0].cuda(), si.f32_normal((16,), 5, std=0.3).cuda()
    ws = st.workspace(1)
    out = torch.empty(3, 16, 256, dtype=torch.bfloat16, device="cuda")
    for t in range(90):
        x = decode_inputs_gpu(cfg, seed=30_000 + t, quantized=True)
        g_out, ref = _step_both(rma, st, ost, ws, 0, x, w, b, out)
        assert output_error(g_out, ref) <= TOL, f"step {t}"
        assert_fp8_state_equal(fp8_state_np(st), ost, f"step {t}")


@pytest.mark.parametrize("force", [False, True])
def test_fp8_admit_alone_random_fills_bit_exact(force):
    rma = lib()
    cfg = oracle.Config(batch=16, n_layers=1)
    rng = np.random.default_rng(5)
    bank = rng.integers(0, 1025, size=(1, 16, 4))
    pend = np.where(rng.random((1, 16, 4)) < 0.5, 256, rng.integers(0, 256, size=(1, 16, 4)))
    st, ost = make_fp8_pair(cfg, seed=5, pos=4096, bank_fill=bank, pend_fill=pend, quantized=True)
    rma.admit(st, 0, force=force)
    oracle.admit_fp8(ost, 0, force=force)
    assert_fp8_state_equal(fp8_state_np(st), ost, f"admit force={force}")


def test_fp8_storage_error_against_bf16():
    """The same seeded state stored in BF16 and in FP8, one decode step each: the outputs differ by
    the E4M3 rounding of K and V (4 significant bits).  Reported, with a loose sanity bound."""
    rma = lib()
    cfg = oracle.Config(batch=8, n_layers=1)
    c = si.workload_counters("batch", 1, 8, 4)
    st16, _ = make_pair(cfg, seed=6, **c)
    st8 = rma.State(_fp8_config(cfg))
    rma.state_quantize(st8, st16)
    w, b = si.gate_params(1, 16, 256, seed=6)
    w, b = w[0].cuda(), b[0].cuda()
    x = decode_inputs_gpu(cfg, seed=60_000)
    o16 = torch.empty(8, 16, 256, dtype=torch.bfloat16, device="cuda")
    o8 = torch.empty_like(o16)
    rma.decode_step(st16, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"], w, b, o16,
                    st16.workspace(1))
    rma.decode_step(st8, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"], w, b, o8,
                    st8.workspace(1))
    torch.cuda.synchronize()
    a, d = o16.float(), o8.float()
    rel = float((d - a).norm() / a.norm())
    print(f"FP8 vs BF16 storage: relative RMS output difference {rel:.3e}, max abs {float((d - a).abs().max()):.3e}")
    assert rel < 0.1


def test_fp8_prefill_is_refused():
    rma = lib()
    st = rma.State(_fp8_config(oracle.Config(batch=1, n_layers=1)))
    z = torch.zeros(1, 4, 16, 256, dtype=torch.bfloat16, device="cuda")
    zk = torch.zeros(1, 4, 4, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rma.RmaError) as ei:
        rma.prefill_block(st, 0, z, zk, zk, zk, zk, torch.zeros(1, 4, 4, device="cuda"),
                          torch.zeros(16, 256, device="cuda"), torch.zeros(16, device="cuda"), torch.empty_like(z),
                          st.workspace(4))
    assert ei.value.code == -2
