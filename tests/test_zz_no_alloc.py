"""The decode entry point for callers that cannot allocate device memory.

Some callers of this library cannot hand it a workspace: a plug-in running
inside a framework that owns all device memory, a serving loop that forbids
allocation once it has started, an embedded deployment that reserves its
memory once.  rma_decode_step_noalloc serves them from a scratch array built
into the library.  These tests call it through the C ABI and check it against
rma_decode_step with a caller-supplied workspace, on two calls in a row (the
second call finds the first call's leftovers in the shared scratch), and check
that a call too large for the built-in scratch is refused before any launch.

This file is collected last on purpose, so a stop-at-first-failure run has
already run every other test; it also passes on its own in a fresh process.
"""
import pytest
import torch

import oracle
import synth_inputs as si
from _gpu import TOL, decode_inputs_gpu, gpu_state_np, lib, make_pair, output_error
from _util import to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    rma = lib()
    cfg = oracle.Config(batch=24, n_layers=2)
    c = si.workload_counters("ragged", 2, 24, 4, seed=3)
    st_ws, _ = make_pair(cfg, seed=11, **c)
    st_na, _ = make_pair(cfg, seed=11, **c)
    assert torch.equal(st_ws.buffer, st_na.buffer)
    w, b = si.gate_params(2, 16, 256, seed=4)
    w, b = w.cuda(), si.f32_normal((2, 16), 6, std=0.4).cuda()
    ws = st_ws.workspace(1)
    out_ws = torch.empty(24, 16, 256, dtype=torch.bfloat16, device="cuda")
    out_na = torch.empty_like(out_ws)
    for call in range(2):
        for layer in (0, 1):
            x = decode_inputs_gpu(cfg, seed=900 + 10 * call + layer)
            rma.decode_step(st_ws, layer, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                            x["cand_score"], w[layer], b[layer], out_ws, ws)
            rma.decode_step_noalloc(st_na, layer, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                                    x["cand_score"], w[layer], b[layer], out_na)
            torch.cuda.synchronize()
            err = output_error(to_np(out_na), to_np(out_ws))
            assert err <= TOL, f"call {call} layer {layer}: {err}"
            # the same kernel, split shape and inputs: the outputs agree bit for bit, so a
            # partial read from the wrong place or left over from the previous call shows here
            assert torch.equal(out_na, out_ws), f"call {call} layer {layer}: outputs differ in some bit"
        a, bb = gpu_state_np(st_ws), gpu_state_np(st_na)
        for k in a:
            assert (a[k].tobytes() == bb[k].tobytes()), f"call {call}: state array {k} differs"
    assert rma.get_status(st_na) == rma.get_status(st_ws)


def test_noalloc_refuses_a_call_larger_than_its_scratch():
    rma = lib()
    cfg = rma.Config(batch=32, n_layers=1)
    st = rma.State(cfg)
    rma.set_decode_splits(st, 32, 32)   # 32 x 4 x 64 partials of 4,128 B = 33.8 MB > 32 MiB
    before = st.buffer.clone()
    z16 = torch.zeros(32, 16, 256, dtype=torch.bfloat16, device="cuda")
    z4 = torch.zeros(32, 4, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rma.RmaError) as ei:
        rma.decode_step_noalloc(st, 0, z16, z4, z4, z4, z4, torch.zeros(32, 4, device="cuda"),
                                torch.zeros(16, 256, device="cuda"), torch.zeros(16, device="cuda"),
                                torch.empty_like(z16))
    assert ei.value.code == -3 and "built-in scratch" in str(ei.value)
    torch.cuda.synchronize()
    assert torch.equal(before, st.buffer)   # nothing was launched
