"""Pin the oracle's BF16 conversions to torch's own (an independent implementation)."""
import numpy as np
import torch

import oracle
from _util import bf16_bits_to_f64_torch


def test_expand_every_bit_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    a = oracle.bf16_to_f64(bits)
    b = bf16_bits_to_f64_torch(bits)
    assert np.array_equal(a, b, equal_nan=True)


def test_round_fp32_values_like_torch():
    g = torch.Generator().manual_seed(0)
    x = torch.cat([torch.randn(200000, generator=g) * s for s in (1e-3, 1.0, 1e3)])
    # exact halfway points between neighbouring bf16 values (ties go to even)
    base = torch.randn(5000, generator=g).to(torch.bfloat16).to(torch.float32)
    half = (base.view(torch.int32) + 0x8000).view(torch.float32)
    x = torch.cat([x, half])
    ours = oracle.f32_to_bf16(x.numpy())
    theirs = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)


def test_round_fp64_to_nearest_bf16():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))
    r = oracle.bf16_to_f64(oracle.f64_to_bf16(x))
    # neighbours: the bf16 values just below and above x
    lo = oracle.bf16_to_f64(oracle.f32_to_bf16(x.astype(np.float32)))
    ulp = np.ldexp(1.0, np.frexp(np.abs(x))[1] - 8)
    err = np.abs(r - x)
    assert (err <= ulp / 2 * (1 + 1e-12)).all()
    assert np.abs(r - lo).max() <= ulp.max()
