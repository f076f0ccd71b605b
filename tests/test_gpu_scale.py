"""GPU parity at the benchmark sizes, on sampled sequences.

Decode: the batch-512 x 8-layer configuration `bench.py` times (rings full at
pos = 131,072 + (b mod 256), banks full, pending staggered b mod 256 so that two
sequences per layer admit in every step), through the same launch shape, for the first
300 steps; 8 sampled sequences x all 8 layers are run by the oracle (one process per
layer) and every step's outputs plus the final state are compared.  Prefill: the block
prefill configuration (8 sequences x 8 layers, 128 blocks of 256 from an empty state);
2 sequences x layers 0 and 7 are run by the oracle through all 128 blocks and compared
after blocks 0, 1, 4, 5 and 127.  Outputs within 1e-2 max(1, |oracle|); states bit-exact.
"""
import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

import _oracle_runs as runs
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


def _pool(n):
    """A spawned worker pool; each worker's numpy uses one thread (the workers run side by side)."""
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"
    return mp.get_context("spawn").Pool(processes=max(1, min(n, os.cpu_count() or 1)))


def _fill_state_on_device(st, seed):
    """Seeded slot contents drawn on the device, one layer at a time."""
    for li in range(st.cfg.n_layers):
        for k, name in enumerate(runs.SLOTS):
            t = getattr(st, name)[li]
            gen = si.bf16_normal if t.dtype == torch.bfloat16 else si.f32_normal
            t.copy_(gen(tuple(t.shape), seed * 1000 + 10 * li + k, device="cuda"))


def _slices(st, layer, seqs):
    """One layer's slot arrays and counters for the sampled sequences, as [1, S, ...] numpy."""
    arrays = {name: to_np(getattr(st, name)[layer:layer + 1, seqs]) for name in runs.SLOTS}
    c = st.counters[layer:layer + 1, seqs].cpu().numpy().astype(np.int64)
    return arrays, (c[..., 0], c[..., 1], c[..., 2])


def _compare(gpu_arrays, gpu_counters, snap, what):
    for name in runs.SLOTS:
        g, o = gpu_arrays[name], snap[name]
        if g.dtype == np.float32:
            g, o = g.view(np.uint32), o.view(np.uint32)
        if not np.array_equal(g, o):
            raise AssertionError(f"{what}: {name} differs first at {tuple(np.argwhere(g != o)[0])}")
    for k, name in enumerate(("pos", "bank_fill", "pend_fill")):
        assert np.array_equal(gpu_counters[k], snap["counters"][k]), f"{what}: counter {name}"


def test_batch512_decode_sampled_parity():
    rma = lib()
    B, L, G, D, STEPS, POOL = 512, 8, 4, 256, 300, 16
    seqs = [0, 37, 100, 129, 200, 254, 255, 511]          # pend_fill 0, 37, 100, 129, 200, 254, 255, 255
    cfg = rma.Config(batch=B, n_layers=L)
    st = rma.State(cfg)
    _fill_state_on_device(st, seed=41)
    cnt = torch.zeros(L, B, G, 4, dtype=torch.int32)
    stagger = (torch.arange(B, dtype=torch.int32) % 256).view(1, B, 1)
    cnt[..., 0] = 131_072 + stagger
    cnt[..., 1] = 1024
    cnt[..., 2] = stagger
    st.counters.copy_(cnt)
    w, b = si.gate_params(L, 16, D, seed=41, device="cuda")
    pool = [si.decode_inputs(B, G, 4, D, seed=4100 + k, device="cuda") for k in range(POOL)]
    torch.cuda.synchronize()
    start = [_slices(st, li, seqs) for li in range(L)]
    pool_np = [{k: to_np(v[seqs]) for k, v in x.items()} for x in pool]
    jobs = [({"batch": len(seqs), "n_layers": 1}, start[li][0], start[li][1],
             [pool_np[t % POOL] for t in range(STEPS)], to_np(w[li]), to_np(b[li])) for li in range(L)]
    with _pool(L) as p:
        pending = p.map_async(runs.decode_trajectory, jobs)
        ws = st.workspace(1)
        out = torch.empty(B, 16, D, dtype=torch.bfloat16, device="cuda")
        outs = torch.empty(STEPS, L, len(seqs), 16, D, dtype=torch.bfloat16, device="cuda")
        sel = torch.tensor(seqs, device="cuda")
        for t in range(STEPS):
            x = pool[t % POOL]
            for li in range(L):
                rma.decode_step(st, li, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"],
                                w[li], b[li], out, ws)
                outs[t, li].copy_(out.index_select(0, sel))
        torch.cuda.synchronize()
        assert rma.get_status(st) == 0
        gpu_outs = to_np(outs.cpu())
        final = [_slices(st, li, seqs) for li in range(L)]
        ref = pending.get()
    worst = 0.0
    for li in range(L):
        ref_outs, snap, status = ref[li]
        assert status == 0, f"layer {li}: oracle status {status}"
        for t in range(STEPS):
            err = output_error(gpu_outs[t, li], ref_outs[t])
            worst = max(worst, err)
            assert err <= TOL, f"layer {li} step {t}: output error {err}"
        _compare(final[li][0], final[li][1], snap, f"layer {li} after {STEPS} steps")
        assert int(snap["counters"][1].min()) == 1024
    # every sampled sequence admitted at least once (pending restarted from 0)
    assert all(int(ref[li][1]["counters"][2][0, s, 0]) == (seqs[s] % 256 + STEPS) % 256
               for li in range(L) for s in range(len(seqs)))
    print(f"batch-512 decode, 8 sequences x 8 layers x {STEPS} steps: worst output error {worst:.3e}")


def test_block_prefill_bench_config_sampled_parity():
    rma = lib()
    B, L, G, D, n, BLOCKS = 8, 8, 4, 256, 256, 128
    seqs, layers, check = [0, 5], [0, 7], [0, 1, 4, 5, 127]
    cfg = rma.Config(batch=B, n_layers=L)
    st = rma.State(cfg)
    _fill_state_on_device(st, seed=43)      # stale bytes everywhere; counters start at zero
    st.counters.zero_()
    w, b = si.gate_params(L, 16, D, seed=43, device="cuda")
    b = si.f32_normal((L, 16), 44, device="cuda", std=0.5)
    torch.cuda.synchronize()
    sampled_seed = lambda blk, li: 900_000 + 1000 * li + blk
    jobs = []
    for li in layers:
        arrays, counters = _slices(st, li, seqs)
        jobs.append(({"batch": len(seqs), "n_layers": 1}, arrays, counters,
                     [sampled_seed(blk, li) for blk in range(BLOCKS)], set(check), to_np(w[li]), to_np(b[li])))
    sel = torch.tensor(seqs, device="cuda")
    with _pool(len(layers)) as p:
        pending = p.map_async(runs.prefill_trajectory, jobs)
        ws = st.workspace(n)
        out = torch.empty(B, n, 16, D, dtype=torch.bfloat16, device="cuda")
        got = {}
        for blk in range(BLOCKS):
            for li in range(L):
                x = si.prefill_inputs(B, n, G, 4, D, seed=4300 + 10 * blk + li, device="cuda")
                if li in layers:
                    xs = si.prefill_inputs(len(seqs), n, G, 4, D, seed=sampled_seed(blk, li))
                    for k in x:
                        x[k][sel] = xs[k].cuda()
                rma.prefill_block(st, li, x["q"], x["k"], x["v"], x["cand_k"], x["cand_v"], x["cand_score"],
                                  w[li], b[li], out, ws)
                if blk in check and li in layers:
                    got[(blk, li)] = (to_np(out.index_select(0, sel).cpu()), _slices(st, li, seqs))
        torch.cuda.synchronize()
        assert rma.get_status(st) == 0
        ref = pending.get()
    for k, li in enumerate(layers):
        res, status = ref[k]
        assert status == 0, f"layer {li}: oracle status {status}"
        for blk in check:
            g_out, (g_arrays, g_counters) = got[(blk, li)]
            o_out, snap = res[blk]
            err = output_error(g_out, o_out)
            assert err <= TOL, f"layer {li} block {blk}: output error {err}"
            _compare(g_arrays, g_counters, snap, f"layer {li} after block {blk}")
        assert int(res[127][1]["counters"][0].min()) == BLOCKS * n
