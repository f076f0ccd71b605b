"""Shared set-up for the GPU parity tests: one seeded state, two copies.

The CUDA side gets a librma state buffer; the oracle side gets numpy arrays
with the same bytes.  Inputs come from ``synth_inputs`` only; nothing here
computes any part of the method.
"""
import numpy as np
import torch

import oracle
import synth_inputs as si
from _util import to_np

TOL = 1e-2   # |gpu - oracle| <= TOL * max(1, |oracle|), element by element


def lib():
    import bounded_memory_attention_b200 as rma
    return rma


def gpu_config(cfg: "oracle.Config"):
    rma = lib()
    return rma.Config(batch=cfg.batch, n_layers=cfg.n_layers, n_groups=cfg.n_groups, q_per_group=cfg.q_per_group,
                      head_dim=cfg.head_dim, ring_slots=cfg.ring_slots, bank_slots=cfg.bank_slots,
                      pend_slots=cfg.pend_slots, softmax_scale=cfg.softmax_scale)


def make_pair(cfg: "oracle.Config", seed: int, pos, bank_fill, pend_fill, quantized: bool = False):
    """A GPU state and an oracle state with identical slot bytes and counters.

    pos, bank_fill, pend_fill: ints or arrays broadcastable to [L, B, G].
    """
    rma = lib()
    contents = si.state_contents(cfg.n_layers, cfg.batch, cfg.n_groups, cfg.head_dim, cfg.ring_slots,
                                 cfg.bank_slots, cfg.pend_slots, seed=seed, quantized_scores=quantized)
    st = rma.State(gpu_config(cfg))
    for name, t in contents.items():
        getattr(st, name).copy_(t)
    shape = (cfg.n_layers, cfg.batch, cfg.n_groups)
    cnt = np.zeros(shape + (4,), np.int32)
    cnt[..., 0] = np.broadcast_to(np.asarray(pos), shape)
    cnt[..., 1] = np.broadcast_to(np.asarray(bank_fill), shape)
    cnt[..., 2] = np.broadcast_to(np.asarray(pend_fill), shape)
    st.counters.copy_(torch.from_numpy(cnt))
    ost = oracle.state_from_arrays(cfg, {k: to_np(v) for k, v in contents.items()},
                                   pos=cnt[..., 0], bank_fill=cnt[..., 1], pend_fill=cnt[..., 2])
    torch.cuda.synchronize()
    return st, ost


def gpu_state_np(st, layers=None, seqs=None) -> dict:
    """The GPU state's arrays as numpy, optionally restricted to some layers and sequences."""
    out = {}
    for name in ("ring_k", "ring_v", "bank_k", "bank_v", "bank_score", "pend_k", "pend_v", "pend_score"):
        t = getattr(st, name)
        if layers is not None:
            t = t[layers]
        if seqs is not None:
            t = t[:, seqs]
        out[name] = to_np(t)
    c = st.counters
    if layers is not None:
        c = c[layers]
    if seqs is not None:
        c = c[:, seqs]
    c = c.cpu().numpy()
    out["pos"], out["bank_fill"], out["pend_fill"] = c[..., 0], c[..., 1], c[..., 2]
    return out


def assert_state_equal(gpu: dict, ost: "oracle.State", what: str = "") -> None:
    """Bit-exact comparison of every slot byte and counter."""
    for name in ("ring_k", "ring_v", "bank_k", "bank_v", "pend_k", "pend_v"):
        a, b = gpu[name], getattr(ost, name)
        if not np.array_equal(a, b):
            idx = np.argwhere(a != b)[0]
            raise AssertionError(f"{what}: {name} differs first at {tuple(idx)}")
    for name in ("bank_score", "pend_score"):
        a, b = gpu[name].view(np.uint32), getattr(ost, name).view(np.uint32)
        if not np.array_equal(a, b):
            idx = np.argwhere(a != b)[0]
            raise AssertionError(f"{what}: {name} bits differ first at {tuple(idx)}")
    for name in ("pos", "bank_fill", "pend_fill"):
        if not np.array_equal(gpu[name].astype(np.int64), getattr(ost, name)):
            raise AssertionError(f"{what}: counter {name} differs: gpu {gpu[name].ravel()[:8]} "
                                 f"oracle {getattr(ost, name).ravel()[:8]}")


def output_error(gpu_bits: np.ndarray, oracle_bits: np.ndarray) -> float:
    """max over elements of |gpu - oracle| / max(1, |oracle|)."""
    g = oracle.bf16_to_f64(gpu_bits)
    o = oracle.bf16_to_f64(oracle_bits)
    return float(np.max(np.abs(g - o) / np.maximum(1.0, np.abs(o)))) if g.size else 0.0


def decode_inputs_gpu(cfg, seed, quantized=False):
    d = si.decode_inputs(cfg.batch, cfg.n_groups, cfg.q_per_group, cfg.head_dim, seed=seed,
                         quantized_scores=quantized)
    return {k: v.cuda() for k, v in d.items()}
