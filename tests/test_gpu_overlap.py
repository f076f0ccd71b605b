"""GPU parity with decode overlap on (rma_set_decode_overlap): launches that request their first
ring and bank tiles while the previous decode launch on the stream is finishing.

The library lets a decode launch touch its layer early only when the previous kernel on the
stream is a decode of another layer (or another state); inputs are always read after the wait.
These tests drive each case against the oracle: layers in turn (early), the same layer twice in a
row (waits first), a chain where one layer's output is the next call's query (early, the query read
after the wait), two states on one stream, and the same steps replayed from a CUDA graph.  Outputs
within 1e-2 max(1, |oracle|), state bit-exact.
"""
import pytest
import torch

import oracle
import synth_inputs as si
from _gpu import TOL, assert_state_equal, decode_inputs_gpu, gpu_state_np, lib, make_pair, output_error
from _util import to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bounded_memory_attention_b200 import build
    build.build()


def _oracle_step(ost, layer, x, w, b):
    xn = {k: to_np(v) for k, v in x.items()}
    ref = oracle.decode_step(ost, layer, xn["q"], xn["k_cur"], xn["v_cur"], xn["cand_k"], xn["cand_v"],
                             xn["cand_score"], to_np(w), to_np(b))
    oracle.admit(ost, layer)
    return ref


def _launch(rma, st, layer, x, w, b, out, ws):
    rma.decode_step(st, layer, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"],
                    w, b, out, ws)


def _state(seed, batch=2, layers=3):
    """Sequence 0 full and about to admit, sequence 1 (if any) partly filled."""
    cfg = oracle.Config(batch=batch, n_layers=layers)
    pos = [[1500] * 4, [300] * 4][:batch]
    bank = [[1024] * 4, [400] * 4][:batch]
    pend = [[250] * 4, [5] * 4][:batch]
    st, ost = make_pair(cfg, seed=seed, pos=[pos] * layers, bank_fill=[bank] * layers, pend_fill=[pend] * layers)
    return cfg, st, ost


@pytest.mark.parametrize("order", ["layers_in_turn", "same_layer_twice"])
def test_overlap_decode_sequences_match_the_oracle(order):
    rma = lib()
    cfg, st, ost = _state(61)
    rma.set_decode_overlap(st, True)
    w, b = si.gate_params(3, 16, 256, seed=61)
    w, b = w.cuda(), si.f32_normal((3, 16), 62, std=0.5).cuda()
    ws = st.workspace(1)
    seq = [0, 1, 2] * 4 if order == "layers_in_turn" else [0, 0, 1, 1, 2, 2, 2, 0]
    outs, refs = [], []
    for t, layer in enumerate(seq):              # no synchronisation between the launches
        x = decode_inputs_gpu(cfg, seed=6100 + t)
        out = torch.empty(2, 16, 256, dtype=torch.bfloat16, device="cuda")
        _launch(rma, st, layer, x, w[layer], b[layer], out, ws)
        outs.append(out)
        refs.append(_oracle_step(ost, layer, x, w[layer], b[layer]))
    torch.cuda.synchronize()
    for t, (o, r) in enumerate(zip(outs, refs)):
        err = output_error(to_np(o), r)
        assert err <= TOL, f"call {t} (layer {seq[t]}): {err}"
    assert_state_equal(gpu_state_np(st), ost, order)
    assert rma.get_status(st) == 0


def test_overlap_chain_where_the_query_is_the_previous_output():
    """Layer l + 1's query is layer l's output buffer, written by the launch it may overlap."""
    rma = lib()
    cfg, st, ost = _state(63)
    rma.set_decode_overlap(st, True)
    w, b = si.gate_params(3, 16, 256, seed=63)
    w, b = w.cuda(), b.cuda()
    ws = st.workspace(1)
    bufs = [torch.empty(2, 16, 256, dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    x0 = decode_inputs_gpu(cfg, seed=6300)
    bufs[0].copy_(x0["q"])
    xs = [decode_inputs_gpu(cfg, seed=6310 + layer) for layer in range(3)]
    for layer in range(3):
        x = dict(xs[layer])
        x["q"] = bufs[layer]
        _launch(rma, st, layer, x, w[layer], b[layer], bufs[layer + 1], ws)
    torch.cuda.synchronize()
    q = to_np(x0["q"])
    for layer in range(3):
        xn = {k: to_np(v) for k, v in xs[layer].items()}
        ref = oracle.decode_step(ost, layer, q, xn["k_cur"], xn["v_cur"], xn["cand_k"], xn["cand_v"],
                                 xn["cand_score"], to_np(w[layer]), to_np(b[layer]))
        oracle.admit(ost, layer)
        err = output_error(to_np(bufs[layer + 1]), ref)
        assert err <= TOL, f"layer {layer}: {err}"
        q = to_np(bufs[layer + 1])      # the GPU's output is the next query, as it was on the GPU
    assert_state_equal(gpu_state_np(st), ost, "chain")


def test_overlap_two_states_on_one_stream():
    rma = lib()
    cfg, s1, o1 = _state(64)
    _, s2, o2 = _state(65)
    for s in (s1, s2):
        rma.set_decode_overlap(s, True)
    w, b = si.gate_params(3, 16, 256, seed=64)
    w, b = w.cuda(), b.cuda()
    ws1, ws2 = s1.workspace(1), s2.workspace(1)
    outs, refs = [], []
    for t in range(6):                           # s1 layer 0, s2 layer 0, s1 layer 1, ...
        layer = t // 2
        for st, ost, ws in ((s1, o1, ws1), (s2, o2, ws2)):
            x = decode_inputs_gpu(cfg, seed=6400 + 10 * t + (st is s2))
            out = torch.empty(2, 16, 256, dtype=torch.bfloat16, device="cuda")
            _launch(rma, st, layer % 3, x, w[layer % 3], b[layer % 3], out, ws)
            outs.append(out)
            refs.append(_oracle_step(ost, layer % 3, x, w[layer % 3], b[layer % 3]))
    torch.cuda.synchronize()
    for t, (o, r) in enumerate(zip(outs, refs)):
        assert output_error(to_np(o), r) <= TOL, f"call {t}"
    assert_state_equal(gpu_state_np(s1), o1, "state 1")
    assert_state_equal(gpu_state_np(s2), o2, "state 2")


def test_overlap_steps_replayed_from_a_graph():
    """Three layers per step captured once with overlap on, replayed 10 times with fresh inputs."""
    rma = lib()
    cfg, st, ost = _state(66, batch=1)
    rma.set_decode_overlap(st, True)
    w, b = si.gate_params(3, 16, 256, seed=66)
    w, b = w.cuda(), b.cuda()
    ws = st.workspace(1)
    static = [decode_inputs_gpu(cfg, seed=6600 + layer) for layer in range(3)]
    outs = [torch.empty(1, 16, 256, dtype=torch.bfloat16, device="cuda") for _ in range(3)]

    def step(stream):
        for layer in range(3):
            _launch(rma, st, layer, static[layer], w[layer], b[layer], outs[layer], ws)

    cs = torch.cuda.Stream()
    snap = st.buffer.clone()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cs):
        step(cs)                                 # warm-up outside the capture
    cs.synchronize()
    st.buffer.copy_(snap)                        # the warm-up's effects undone
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cs):
        step(cs)
    st.buffer.copy_(snap)                        # capture runs nothing, but be explicit
    torch.cuda.synchronize()
    for r in range(10):
        fresh = [decode_inputs_gpu(cfg, seed=6700 + 10 * r + layer) for layer in range(3)]
        for layer in range(3):
            for k in static[layer]:
                static[layer][k].copy_(fresh[layer][k])
        g.replay()
        torch.cuda.synchronize()
        for layer in range(3):
            ref = _oracle_step(ost, layer, fresh[layer], w[layer], b[layer])
            err = output_error(to_np(outs[layer]), ref)
            assert err <= TOL, f"replay {r} layer {layer}: {err}"
        assert_state_equal(gpu_state_np(st), ost, f"replay {r}")
