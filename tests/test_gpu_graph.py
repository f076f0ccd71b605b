"""GPU parity of calls replayed from CUDA graphs.

The library's calls are asynchronous on the caller's stream and allocate nothing, so a
sequence of them captures into a CUDA graph.  Each replay must then read the state the
previous one left, exactly as the oracle does call by call: outputs within
1e-2 max(1, |oracle|), state bit-exact.
"""
import pytest
import torch

import oracle
import synth_inputs as si
from _gpu import TOL, assert_state_equal, gpu_state_np, lib, make_pair, output_error
from _util import to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bounded_memory_attention_b200 import build
    build.build()


def _decode_oracle(ost, layer, x, w, b):
    xn = {k: to_np(v) for k, v in x.items()}
    ref = oracle.decode_step(ost, layer, xn["q"], xn["k_cur"], xn["v_cur"], xn["cand_k"], xn["cand_v"],
                             xn["cand_score"], to_np(w), to_np(b))
    oracle.admit(ost, layer)
    return ref


def _prefill_oracle(ost, layer, x, w, b):
    xn = {k: to_np(v) for k, v in x.items()}
    return oracle.prefill_block(ost, layer, xn["q"], xn["k"], xn["v"], xn["cand_k"], xn["cand_v"],
                                xn["cand_score"], to_np(w), to_np(b))


def test_decode_steps_replayed_from_a_graph():
    """One graph holds a decode step of both layers (each launch runs the admit itself when it fills
    pending); 12 replays with fresh inputs copied into the captured buffers cross an admit in two
    of the (layer, sequence) pairs."""
    rma = lib()
    cfg = oracle.Config(batch=2, n_layers=2)
    st, ost = make_pair(cfg, seed=51,
                        pos=[[[1500] * 4, [300] * 4], [[2000] * 4, [77] * 4]],
                        bank_fill=[[[1024] * 4, [400] * 4], [[1024] * 4, [0] * 4]],
                        pend_fill=[[[250] * 4, [5] * 4], [[247] * 4, [0] * 4]])
    w, b = si.gate_params(2, 16, 256, seed=51)
    w, b = w.cuda(), si.f32_normal((2, 16), 52, std=0.5).cuda()
    ws = st.workspace(1)
    static = [{k: v.cuda() for k, v in si.decode_inputs(2, 4, 4, 256, seed=5100 + li).items()} for li in range(2)]
    outs = [torch.empty(2, 16, 256, dtype=torch.bfloat16, device="cuda") for _ in range(2)]

    def step():
        for li in range(2):
            x = static[li]
            rma.decode_step(st, li, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"],
                            w[li], b[li], outs[li], ws)
            rma.admit(st, li)

    step()   # one eager step first (the library's one-time set-up happens outside the capture)
    torch.cuda.synchronize()
    for li in range(2):
        assert output_error(to_np(outs[li]), _decode_oracle(ost, li, static[li], w[li], b[li])) <= TOL
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cs):
        step()
    torch.cuda.synchronize()
    assert_state_equal(gpu_state_np(st), ost, "after the capture (which runs nothing)")
    for t in range(12):
        fresh = [si.decode_inputs(2, 4, 4, 256, seed=5200 + 10 * t + li) for li in range(2)]
        for li in range(2):
            for k, v in fresh[li].items():
                static[li][k].copy_(v)
        graph.replay()
        torch.cuda.synchronize()
        for li in range(2):
            err = output_error(to_np(outs[li]), _decode_oracle(ost, li, fresh[li], w[li], b[li]))
            assert err <= TOL, f"replay {t} layer {li}: output error {err}"
    assert_state_equal(gpu_state_np(st), ost, "after 12 replays")
    assert int(ost.pend_fill[0, 0, 0]) == (250 + 13) % 256 and int(ost.pend_fill[1, 0, 0]) == (247 + 13) % 256
    assert rma.get_status(st) == 0
    del graph


def test_prefill_blocks_replayed_from_a_graph():
    """A 100-token prefill block captured once (its tensor maps are built at capture time over the
    captured buffers) and replayed three times with fresh inputs: the ring rotates, pos advances and
    each replay's forced admit fills the bank further."""
    rma = lib()
    cfg = oracle.Config(batch=2, n_layers=1)
    st, ost = make_pair(cfg, seed=53, pos=[[[900] * 4, [40] * 4]], bank_fill=[[[600] * 4, [0] * 4]],
                        pend_fill=[[[0] * 4, [12] * 4]])
    w, b = si.gate_params(1, 16, 256, seed=53)
    w, b = w[0].cuda(), si.f32_normal((16,), 54, std=0.5).cuda()
    n = 100
    ws = st.workspace(n)
    static = {k: v.cuda() for k, v in si.prefill_inputs(2, n, 4, 4, 256, seed=5300).items()}
    out = torch.empty(2, n, 16, 256, dtype=torch.bfloat16, device="cuda")

    def block():
        x = static
        rma.prefill_block(st, 0, x["q"], x["k"], x["v"], x["cand_k"], x["cand_v"], x["cand_score"], w, b, out, ws)

    block()
    torch.cuda.synchronize()
    assert output_error(to_np(out), _prefill_oracle(ost, 0, static, w, b)) <= TOL
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cs):
        block()
    torch.cuda.synchronize()
    for t in range(3):
        fresh = si.prefill_inputs(2, n, 4, 4, 256, seed=5301 + t)
        for k, v in fresh.items():
            static[k].copy_(v)
        graph.replay()
        torch.cuda.synchronize()
        err = output_error(to_np(out), _prefill_oracle(ost, 0, fresh, w, b))
        assert err <= TOL, f"replay {t}: output error {err}"
        assert_state_equal(gpu_state_np(st), ost, f"after replay {t}")
    assert int(ost.pos[0, 1, 0]) == 40 + 4 * n and int(ost.bank_fill[0, 1, 0]) == 12 + 4 * n
    assert rma.get_status(st) == 0
    del graph
