"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and answers the host-only calls (sizes, argument checks, error text)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from bounded_memory_attention_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "rma.h")).read()
    return sorted(set(re.findall(r"RMA_API\s+[\w\s\*]+?\b(rma_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/rma.h but not exported"


def test_state_bytes_is_the_sum_of_the_arrays():
    import bounded_memory_attention_b200 as rma
    cfg = rma.Config(batch=512, n_layers=8)
    kv = 2 * 512 * 8 * 4 * (1023 + 1024 + 256) * 256 * 2       # K and V rows of ring, bank, pending
    scores = 512 * 8 * 4 * (1024 + 256) * 4
    counters = 512 * 8 * 4 * (16 + 4) + 4
    n = rma.state_bytes(cfg)
    assert kv + scores + counters <= n <= kv + scores + counters + 11 * 256
    # per sequence this is the pages' 72 MiB of attention KV plus scores and counters
    assert abs(rma.state_bytes(rma.Config(batch=1, n_layers=8)) / 2 ** 20 - 72.1) < 0.2


def test_state_size_has_no_sequence_length_input():
    """Check (e) at the boundary: the size is a function of the configuration only."""
    import bounded_memory_attention_b200 as rma
    assert {f for f in rma.Config.__dataclass_fields__} == {
        "batch", "n_layers", "n_groups", "q_per_group", "head_dim", "ring_slots", "bank_slots",
        "pend_slots", "softmax_scale", "kv_format"}


def test_fp8_state_bytes_are_the_sum_of_codes_exponents_scores_and_counters():
    """An FP8 state: one byte per K/V element, one exponent byte per row (slots padded to 16),
    the same scores and counters; per sequence about half the BF16 state."""
    import bounded_memory_attention_b200 as rma
    cfg = rma.Config(batch=512, n_layers=8, kv_format=rma.KV_FP8_E4M3)
    rows = 512 * 8 * 4 * (1023 + 1024 + 256)
    kv = 2 * rows * 256
    exps = 2 * 512 * 8 * 4 * (1024 + 1024 + 256)
    scores = 512 * 8 * 4 * (1024 + 256) * 4
    counters = 512 * 8 * 4 * (16 + 4) + 4
    n = rma.state_bytes(cfg)
    assert kv + exps + scores + counters <= n <= kv + exps + scores + counters + 17 * 256
    one_bf16 = rma.state_bytes(rma.Config(batch=1, n_layers=8))
    one_fp8 = rma.state_bytes(rma.Config(batch=1, n_layers=8, kv_format=rma.KV_FP8_E4M3))
    assert 0.5 < one_fp8 / one_bf16 < 0.51


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 128, "RMA_ERR_UNSUPPORTED"), ("q_per_group", 8, "RMA_ERR_UNSUPPORTED"),
    ("batch", 0, "RMA_ERR_INVALID_ARG"), ("ring_slots", 0, "RMA_ERR_INVALID_ARG"),
    ("softmax_scale", float("nan"), "RMA_ERR_INVALID_ARG"), ("bank_slots", 4000, "RMA_ERR_UNSUPPORTED"),
    ("kv_format", 2, "RMA_ERR_INVALID_ARG")])
def test_bad_configs_are_rejected_on_the_host(field, value, code):
    import bounded_memory_attention_b200 as rma
    cfg = rma.Config(**{field: value})
    assert rma.state_bytes(cfg) == 0
    assert rma.lib.rma_last_error().decode() != ""
    buf = ctypes.c_void_p(256)   # never dereferenced: the config check fails first
    h = ctypes.c_void_p()
    rc = rma.lib.rma_state_alloc(ctypes.byref(cfg._c()), buf, 1 << 30, None, ctypes.byref(h))
    assert rma.ERRORS[rc] == code


def test_null_and_layer_errors_without_a_gpu():
    import bounded_memory_attention_b200 as rma
    assert rma.lib.rma_admit(None, 0, 0, None) == -1
    assert rma.lib.rma_decode_step(None, 0, *([None] * 10), 0, None) == -1
    assert rma.lib.rma_strerror(-3) == b"buffer too small"
    assert rma.lib.rma_strerror(0) == b"ok"


def test_setters_reject_null_states_without_a_gpu():
    import bounded_memory_attention_b200 as rma
    assert rma.lib.rma_set_decode_overlap(None, 1) == -1
    assert rma.lib.rma_set_decode_splits(None, 1, 1) == -1
