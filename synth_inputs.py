"""Seeded synthetic inputs for the RMA attention hot path.

This module only draws random numbers. It holds none of the method's
arithmetic, so both the CUDA path (through the tests and ``bench.py``) and the
CPU oracle can take their inputs from it without sharing any computation.

Distributions follow the workloads the pages measure with synthetic tokens
(EdgeRock model card, "Inference efficiency", runtime protocol): BF16 Q/K/V
drawn from N(0, 1) and rounded to BF16, FP32 scores from N(0, 1), and gate
weights from N(0, 1/256).  Scores can be quantised to 16 levels
``(clamp(floor(4 z) + 8, 0, 15) - 8) / 4`` so that ties are common; every
level is exact in FP32.

Every generator takes a seed and a device and returns torch tensors; the
caller copies them to wherever they are needed (numpy for the oracle, the
state buffer for the CUDA path).
"""
from __future__ import annotations

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def bf16_normal(shape, seed: int, device="cpu", std: float = 1.0) -> torch.Tensor:
    """BF16 tensor with entries N(0, std^2), drawn in FP32 and rounded to nearest even."""
    x = torch.randn(tuple(shape), generator=_gen(seed, device), device=device, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(torch.bfloat16)


def f32_normal(shape, seed: int, device="cpu", std: float = 1.0) -> torch.Tensor:
    x = torch.randn(tuple(shape), generator=_gen(seed, device), device=device, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x


def f32_quantized_scores(shape, seed: int, device="cpu") -> torch.Tensor:
    """Scores on 16 levels in [-2, 1.75], step 0.25; many exact ties by construction."""
    z = torch.randn(tuple(shape), generator=_gen(seed, device), device=device, dtype=torch.float32)
    return (torch.clamp(torch.floor(4.0 * z) + 8.0, 0.0, 15.0) - 8.0) / 4.0


def uniform_int(shape, low: int, high: int, seed: int, device="cpu") -> torch.Tensor:
    """Integers uniform on [low, high] (both ends included)."""
    return torch.randint(int(low), int(high) + 1, tuple(shape), generator=_gen(seed, device),
                         device=device, dtype=torch.int64)


def decode_inputs(batch: int, n_groups: int, q_per_group: int, head_dim: int, seed: int,
                  device="cpu", quantized_scores: bool = False) -> dict:
    """One decode step's per-token inputs for one layer.

    q [B, G*H, D] bf16; k_cur, v_cur, cand_k, cand_v [B, G, D] bf16; cand_score [B, G] f32.
    """
    B, G, H, D = batch, n_groups, q_per_group, head_dim
    s = int(seed) * 8
    score = (f32_quantized_scores((B, G), s + 5, device) if quantized_scores
             else f32_normal((B, G), s + 5, device))
    return {
        "q": bf16_normal((B, G * H, D), s + 0, device),
        "k_cur": bf16_normal((B, G, D), s + 1, device),
        "v_cur": bf16_normal((B, G, D), s + 2, device),
        "cand_k": bf16_normal((B, G, D), s + 3, device),
        "cand_v": bf16_normal((B, G, D), s + 4, device),
        "cand_score": score,
    }


def prefill_inputs(batch: int, n_tok: int, n_groups: int, q_per_group: int, head_dim: int,
                   seed: int, device="cpu", quantized_scores: bool = False) -> dict:
    """One prefill block's inputs for one layer.

    q [B, n, G*H, D]; k, v, cand_k, cand_v [B, n, G, D] bf16; cand_score [B, n, G] f32.
    """
    B, n, G, H, D = batch, n_tok, n_groups, q_per_group, head_dim
    s = int(seed) * 8 + 3
    score = (f32_quantized_scores((B, n, G), s + 5, device) if quantized_scores
             else f32_normal((B, n, G), s + 5, device))
    return {
        "q": bf16_normal((B, n, G * H, D), s + 0, device),
        "k": bf16_normal((B, n, G, D), s + 1, device),
        "v": bf16_normal((B, n, G, D), s + 2, device),
        "cand_k": bf16_normal((B, n, G, D), s + 3, device),
        "cand_v": bf16_normal((B, n, G, D), s + 4, device),
        "cand_score": score,
    }


def gate_params(n_layers: int, n_q_heads: int, head_dim: int, seed: int, device="cpu",
                std: float = 1.0 / 16.0) -> tuple:
    """w_g [L, G*H, D] f32 ~ N(0, std^2) and b_g [L, G*H] f32 = 0."""
    w = f32_normal((n_layers, n_q_heads, head_dim), int(seed) * 8 + 7, device, std=std)
    b = torch.zeros((n_layers, n_q_heads), dtype=torch.float32, device=device)
    return w, b


def state_contents(n_layers: int, batch: int, n_groups: int, head_dim: int, ring_slots: int,
                   bank_slots: int, pend_slots: int, seed: int, device="cpu",
                   quantized_scores: bool = False) -> dict:
    """Random contents for every slot of the ring, bank and pending buffers.

    Which slots are *valid* is set separately by the counters; these are only
    the bytes.  Shapes: ring_k/v [L,B,G,R,D], bank_k/v [L,B,G,A,D],
    bank_score [L,B,G,A], pend_k/v [L,B,G,P,D], pend_score [L,B,G,P].
    """
    L, B, G, D, R, A, P = n_layers, batch, n_groups, head_dim, ring_slots, bank_slots, pend_slots
    s = int(seed) * 16 + 1000
    sc = f32_quantized_scores if quantized_scores else f32_normal
    return {
        "ring_k": bf16_normal((L, B, G, R, D), s + 0, device),
        "ring_v": bf16_normal((L, B, G, R, D), s + 1, device),
        "bank_k": bf16_normal((L, B, G, A, D), s + 2, device),
        "bank_v": bf16_normal((L, B, G, A, D), s + 3, device),
        "bank_score": sc((L, B, G, A), s + 4, device),
        "pend_k": bf16_normal((L, B, G, P, D), s + 5, device),
        "pend_v": bf16_normal((L, B, G, P, D), s + 6, device),
        "pend_score": sc((L, B, G, P), s + 7, device),
    }


def workload_counters(kind: str, n_layers: int, batch: int, n_groups: int, ring_slots: int = 1023,
                      bank_slots: int = 1024, pend_slots: int = 256, seed: int = 0) -> dict:
    """Starting counters (pos, bank_fill, pend_fill), each int64 [L, B, G], for the named workloads.

    tiny     ring pre-filled (pos = R), bank full, pending empty
    batch    rings full (pos = 131072 + b mod P), banks full, pending staggered
             at b mod P so that pos mod P == pend_fill
    long     pos = 131072, ring and bank full, pending empty
    ragged   per (layer, sequence): ring fill U{1..R} (pos = fill), bank fill
             U{0..A}, pending fill U{0..P-1}
    empty    everything zero (block prefill starts here)
    """
    import numpy as np
    L, B, G, R, A, P = n_layers, batch, n_groups, ring_slots, bank_slots, pend_slots
    shape = (L, B, G)
    if kind == "tiny":
        pos, bank, pend = np.full(shape, R), np.full(shape, A), np.zeros(shape)
    elif kind == "batch":
        b = np.arange(B)[None, :, None] % P
        pos = np.broadcast_to(131072 + b, shape)
        bank = np.full(shape, A)
        pend = np.broadcast_to(b, shape)
    elif kind == "long":
        pos, bank, pend = np.full(shape, 131072), np.full(shape, A), np.zeros(shape)
    elif kind == "ragged":
        pos = uniform_int((L, B, 1), 1, R, seed * 3 + 1).numpy()
        bank = uniform_int((L, B, 1), 0, A, seed * 3 + 2).numpy()
        pend = uniform_int((L, B, 1), 0, P - 1, seed * 3 + 3).numpy()
        pos, bank, pend = (np.broadcast_to(x, shape) for x in (pos, bank, pend))
    elif kind == "empty":
        pos = bank = pend = np.zeros(shape)
    else:
        raise ValueError(kind)
    return {"pos": np.array(pos, dtype=np.int64), "bank_fill": np.array(bank, dtype=np.int64),
            "pend_fill": np.array(pend, dtype=np.int64)}


def aligned_ramp(lead_shape, n_rows: int, head_dim: int, seed: int, lo: float, hi: float,
                 noise: float = 0.25, device="cpu") -> torch.Tensor:
    """BF16 rows along one shared direction with magnitudes growing linearly from lo to hi.

    Row i of [*lead_shape, n_rows, head_dim] is ``c_i u + noise z`` with u ~ N(0, 1)^D drawn from
    ``seed`` (the same u for every call with that seed), c_i = lo + (hi - lo) i / (n_rows - 1) and
    z ~ N(0, 1).  Queries drawn with lo = hi = 1 and keys with a wide ramp give scores that keep
    rising along the rows, so a running maximum moves many times.
    """
    u = torch.randn((head_dim,), generator=_gen(seed, "cpu"), dtype=torch.float32).to(device)
    c = torch.linspace(float(lo), float(hi), n_rows, dtype=torch.float32, device=device)
    z = torch.randn(tuple(lead_shape) + (n_rows, head_dim), generator=_gen(int(seed) + 1, device),
                    device=device, dtype=torch.float32)
    return (c[:, None] * u + noise * z).to(torch.bfloat16)
