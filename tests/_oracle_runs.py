"""Oracle trajectories for the benchmark-size parity tests, one RMA layer per worker process.

The workers are started with the "spawn" method, so they share nothing with the parent's
CUDA context; they import only the oracle and the input generators.
"""
import numpy as np

import oracle
import synth_inputs as si

SLOTS = ("ring_k", "ring_v", "bank_k", "bank_v", "bank_score", "pend_k", "pend_v", "pend_score")


def _np(t):
    """torch (CPU) -> numpy in storage form (bf16 as uint16 bits)."""
    import torch
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _state(cfg_kw, arrays, counters):
    cfg = oracle.Config(**cfg_kw)
    return oracle.state_from_arrays(cfg, arrays, pos=counters[0], bank_fill=counters[1], pend_fill=counters[2])


def _snapshot(st):
    snap = {name: getattr(st, name).copy() for name in SLOTS}
    snap["counters"] = (st.pos.copy(), st.bank_fill.copy(), st.pend_fill.copy())
    return snap


def decode_trajectory(job):
    """job: (cfg_kw, arrays, counters, inputs, w_g, b_g) for one layer of the sampled sequences;
    inputs is a list of per-step dicts (storage dtypes).  Returns the per-step outputs and the
    final state."""
    cfg_kw, arrays, counters, inputs, w_g, b_g = job
    st = _state(cfg_kw, arrays, counters)
    outs = []
    for x in inputs:
        outs.append(oracle.decode_step(st, 0, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                                       x["cand_score"], w_g, b_g))
        oracle.admit(st, 0)
    return outs, _snapshot(st), st.status


def prefill_trajectory(job):
    """job: (cfg_kw, arrays, counters, seeds, check_blocks, w_g, b_g): the block inputs of the
    sampled sequences are drawn here from their seeds (the same draw the test made); returns
    the outputs and state snapshots after the blocks in check_blocks."""
    cfg_kw, arrays, counters, seeds, check_blocks, w_g, b_g = job
    st = _state(cfg_kw, arrays, counters)
    cfg = st.cfg
    res = {}
    for blk, seed in enumerate(seeds):
        x = si.prefill_inputs(cfg.batch, cfg.pend_slots, cfg.n_groups, cfg.q_per_group, cfg.head_dim, seed=seed)
        xn = {k: _np(v) for k, v in x.items()}
        out = oracle.prefill_block(st, 0, xn["q"], xn["k"], xn["v"], xn["cand_k"], xn["cand_v"],
                                   xn["cand_score"], w_g, b_g)
        if blk in check_blocks:
            res[blk] = (out, _snapshot(st))
    return res, st.status
