"""GPU parity at the benchmark sizes, on sampled sequences.

The decode test runs the batch-512 x 8-layer configuration `bench.py` times (rings and
banks full, pending staggered so that some sequences admit in the step), through the
same launch shape (the library's split heuristic for batch 512), and checks a sample of
sequences and layers against the oracle run one sequence at a time.  The prefill test runs
the block-prefill configuration (8 sequences x 8 layers, blocks of 256 from an empty
state) and checks sampled (sequence, layer) pairs.  Outputs within 1e-2 max(1, |oracle|);
the sampled state slices bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from _gpu import TOL, lib, output_error
from _util import to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bounded_memory_attention_b200 import build
    build.build()


_SLOTS = ("ring_k", "ring_v", "bank_k", "bank_v", "bank_score", "pend_k", "pend_v", "pend_score")


def _fill_state_on_device(st, seed):
    """Seeded slot contents, drawn on the device one layer at a time (the same generators
    as the small tests; the bytes are copied to the oracle for the sampled sequences)."""
    L = st.cfg.n_layers
    for li in range(L):
        for k, name in enumerate(_SLOTS):
            t = getattr(st, name)[li]
            if t.dtype == torch.bfloat16:
                t.copy_(si.bf16_normal(tuple(t.shape), seed * 1000 + 10 * li + k, device="cuda"))
            else:
                t.copy_(si.f32_normal(tuple(t.shape), seed * 1000 + 10 * li + k, device="cuda"))


def _oracle_slice(st, cfg, layers, seqs):
    """The sampled (layer, sequence) slices of the device state as an oracle state."""
    ocfg = oracle.Config(batch=len(seqs), n_layers=len(layers))
    arrays = {}
    for name in _SLOTS:
        t = getattr(st, name)[layers][:, seqs]
        arrays[name] = to_np(t)
    c = st.counters[layers][:, seqs].cpu().numpy()
    return oracle.state_from_arrays(ocfg, arrays, pos=c[..., 0], bank_fill=c[..., 1], pend_fill=c[..., 2])


def _compare_slices(st, ost, layers, seqs, what):
    for name in _SLOTS:
        g = to_np(getattr(st, name)[layers][:, seqs])
        o = getattr(ost, name)
        if g.dtype == np.float32:
            g, o = g.view(np.uint32), o.view(np.uint32)
        if not np.array_equal(g, o):
            idx = np.argwhere(g != o)[0]
            raise AssertionError(f"{what}: {name} differs first at {tuple(idx)}")
    c = st.counters[layers][:, seqs].cpu().numpy()
    for k, name in enumerate(("pos", "bank_fill", "pend_fill")):
        assert np.array_equal(c[..., k].astype(np.int64), getattr(ost, name)), f"{what}: counter {name}"


def test_batch512_decode_sampled_parity():
    """Batch 512 x 8 layers, rings and banks full, pending staggered 0..255: two decode steps
    through the bench's launch shape; 6 sequences (two of them admitting in the first step,
    two in the second) x layers 0 and 7 against the oracle."""
    rma = lib()
    B, L, G, D = 512, 8, 4, 256
    cfg = rma.Config(batch=B, n_layers=L)
    st = rma.State(cfg)
    _fill_state_on_device(st, seed=41)
    cnt = torch.zeros(L, B, G, 4, dtype=torch.int32)
    cnt[..., 0] = 200_000
    cnt[..., 1] = 1024
    cnt[..., 2] = (torch.arange(B, dtype=torch.int32) % 256).view(1, B, 1)
    st.counters.copy_(cnt)
    torch.cuda.synchronize()
    layers, seqs = [0, 7], [0, 1, 254, 255, 511, 300]   # pend_fill 0, 1, 254, 255, 255, 44
    ost = _oracle_slice(st, cfg, layers, seqs)
    w, b = si.gate_params(L, 16, D, seed=41, device="cuda")
    ws = st.workspace(1)
    out = torch.empty(B, 16, D, dtype=torch.bfloat16, device="cuda")
    for t in range(2):
        x = {k: v for k, v in si.decode_inputs(B, G, 4, D, seed=4100 + t, device="cuda").items()}
        for li in range(L):
            rma.decode_step(st, li, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"],
                            w[li], b[li], out, ws)
            if li not in layers:
                continue
            oi = layers.index(li)
            xn = {k: to_np(v[seqs]) for k, v in x.items()}
            ref = oracle.decode_step(ost, oi, xn["q"], xn["k_cur"], xn["v_cur"], xn["cand_k"], xn["cand_v"],
                                     xn["cand_score"], to_np(w[li]), to_np(b[li]))
            oracle.admit(ost, oi)
            err = output_error(to_np(out[seqs]), ref)
            assert err <= TOL, f"step {t} layer {li}: output error {err}"
        torch.cuda.synchronize()
        _compare_slices(st, ost, layers, seqs, f"after step {t}")
    assert rma.get_status(st) == 0
    # the sequences that started at pend_fill 255 admitted in step 0, those at 254 in step 1
    assert int(ost.pend_fill[0, 3, 0]) == 1 and int(ost.pend_fill[0, 2, 0]) == 0


def test_block_prefill_bench_config_sampled_parity():
    """8 sequences x 8 layers, blocks of 256 from an empty state (the prefill bench workload),
    five blocks (empty, partial and full rings, the bank filling by forced admits); sequences
    0 and 5 at layers 0 and 7 against the oracle after every block."""
    rma = lib()
    B, L, G, D, n = 8, 8, 4, 256, 256
    cfg = rma.Config(batch=B, n_layers=L)
    st = rma.State(cfg)
    _fill_state_on_device(st, seed=43)      # stale bytes everywhere; counters start at zero
    st.counters.zero_()
    torch.cuda.synchronize()
    layers, seqs = [0, 7], [0, 5]
    ost = _oracle_slice(st, cfg, layers, seqs)
    w, b = si.gate_params(L, 16, D, seed=43, device="cuda")
    b = si.f32_normal((L, 16), 44, device="cuda", std=0.5)
    ws = st.workspace(n)
    out = torch.empty(B, n, 16, D, dtype=torch.bfloat16, device="cuda")
    for blk in range(5):
        for li in range(L):
            x = si.prefill_inputs(B, n, G, 4, D, seed=4300 + 10 * blk + li, device="cuda")
            rma.prefill_block(st, li, x["q"], x["k"], x["v"], x["cand_k"], x["cand_v"], x["cand_score"],
                              w[li], b[li], out, ws)
            if li not in layers:
                continue
            oi = layers.index(li)
            xn = {k: to_np(v[seqs]) for k, v in x.items()}
            ref = oracle.prefill_block(ost, oi, xn["q"], xn["k"], xn["v"], xn["cand_k"], xn["cand_v"],
                                       xn["cand_score"], to_np(w[li]), to_np(b[li]))
            err = output_error(to_np(out[seqs]), ref)
            assert err <= TOL, f"block {blk} layer {li}: output error {err}"
        torch.cuda.synchronize()
        _compare_slices(st, ost, layers, seqs, f"after block {blk}")
    assert rma.get_status(st) == 0
    assert int(ost.bank_fill[0, 0, 0]) == 1024 and int(ost.pos[0, 0, 0]) == 5 * 256
