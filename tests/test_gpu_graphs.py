"""Captured calls replay correctly: every piece of state a call reads and advances (the weights,
the index of the In-Place bf16 weight copy, the fp32 weight buffer, the gate's threshold,
cache and token position) lives on the device, so a caller can capture a scan in a CUDA graph
once and replay it over a stream of segments, copying each segment into the captured input
buffers first. Each test runs the same segments eagerly on a second state and asks for the same
bits: outputs, losses, final weights and gate state."""

import pytest
import torch

from gen import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cwl():
    from chunked_weight_layers_b200 import build
    build.build()
    import chunked_weight_layers_b200 as cwl
    return cwl


def _segments(x, names, T, n):
    """Split the token axis (the one before the last) of the named inputs into n segments."""
    return [{k: x[k][..., i * T:(i + 1) * T, :].contiguous() for k in names} for i in range(n)]


def _stream_both_ways(make_state, segments, outs_like, run, read_state):
    """Run the segments eagerly on one state and through one captured call on another; return
    (eager outputs per segment, graph outputs per segment, eager state, graph state)."""
    eager = make_state()
    outs_e = []
    for seg in segments:
        outs = outs_like()
        run(eager, seg, outs)
        outs_e.append([o.clone() for o in outs])
    state_e = read_state(eager)
    torch.cuda.synchronize()
    eager.poll()

    st = make_state()
    bufs = {k: v.clone() for k, v in segments[0].items()}
    outs = outs_like()
    run(st, bufs, outs)  # first use: scratch, schedules and tensor maps are built outside the capture
    st.reset()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            run(st, bufs, outs)
    torch.cuda.current_stream().wait_stream(side)
    outs_g = []
    for seg in segments:
        for k, v in seg.items():
            bufs[k].copy_(v)
        g.replay()
        outs_g.append([o.clone() for o in outs])
    state_g = read_state(st)
    torch.cuda.synchronize()
    st.poll()
    del g
    return outs_e, outs_g, state_e, state_g


def _assert_same(outs_e, outs_g, state_e, state_g):
    for i, (a, b) in enumerate(zip(outs_e, outs_g)):
        for j, (u, v) in enumerate(zip(a, b)):
            assert torch.equal(u, v), f"segment {i}, output {j}"
    for j, (u, v) in enumerate(zip(state_e, state_g)):
        assert torch.equal(u, v), f"state {j}"


def _weights(st, like):
    W = torch.empty_like(like)
    st.get_weights(W)
    return [W]


@pytest.mark.parametrize("model", ["linear", "linear_ln", "mlp"])
def test_ttt_linear_family_streams_through_a_graph(cwl, model):
    T, n = 128, 3
    if model == "linear":
        spec = workloads.scaled(workloads.LINEAR_GD, B=2, H=3, T=T * n, seed=511)
        x = workloads.linear_inputs(spec, device="cuda")
        cfg = cwl.config("linear", batch=spec.B, heads=spec.H, chunk=16, eta=spec.eta)
    else:
        base = workloads.LINEAR_LN if model == "linear_ln" else workloads.MLP
        spec = workloads.scaled(base, B=2, H=2, T=T * n, seed=512)
        x = workloads.inner_inputs(spec, device="cuda")
        cfg = cwl.config(model, batch=spec.B, heads=spec.H, eta=spec.eta, ln_eps=spec.eps)

    def make():
        st = cwl.FastWeightState(cfg, x["W0"])
        if model != "linear":
            st.set_layernorm(x["gamma"], x["beta"])
        return st

    shape = (spec.B, spec.H, T)

    def outs_like():
        return [torch.empty(shape + (64,), device="cuda", dtype=torch.bfloat16),
                torch.empty(shape, device="cuda")]

    def run(st, seg, outs):
        st.chunk_scan(seg["K"], seg["V"], seg["Q"], out=outs[0], loss_out=outs[1])

    _assert_same(*_stream_both_ways(make, _segments(x, ("K", "V", "Q"), T, n), outs_like, run,
                                    lambda st: _weights(st, x["W0"])))


def test_gated_scan_streams_through_a_graph(cwl):
    """The gate's τ, cache entries (with their token positions) and counts follow the replays;
    the cache read over all the streamed tokens then gives the same output on both states."""
    T, n, cap = 256, 3, 256
    spec = workloads.scaled(workloads.SR_TTT_GATE, B=1, H=2, T=T * n, with_queries=True, seed=513)
    x = workloads.linear_inputs(spec, device="cuda")
    cfg = cwl.config("linear", batch=spec.B, heads=spec.H, chunk=16, eta=spec.eta, gate_enable=1,
                     cache_capacity=cap)
    shape = (spec.B, spec.H, T)
    states = []

    def make():
        st = cwl.FastWeightState(cfg, x["W0"])
        states.append(st)
        return st

    def outs_like():
        return [torch.empty(shape + (64,), device="cuda", dtype=torch.bfloat16),
                torch.empty(shape, device="cuda")]

    def run(st, seg, outs):
        st.chunk_scan(seg["K"], seg["V"], seg["Q"], out=outs[0], loss_out=outs[1])

    def read_state(st):
        E = torch.empty((spec.B, spec.H, cap, 3), device="cuda", dtype=torch.int32)
        C = torch.empty((spec.B, spec.H, 2), device="cuda", dtype=torch.int32)
        tau = torch.empty((spec.B, spec.H), device="cuda")
        tau_set = torch.empty((spec.B, spec.H), device="cuda", dtype=torch.int32)
        st.cache_read(E, C)
        st.gate_read(tau, tau_set)
        return _weights(st, x["W0"]) + [E, C, tau, tau_set]

    outs_e, outs_g, state_e, state_g = _stream_both_ways(make, _segments(x, ("K", "V", "Q"), T, n), outs_like,
                                                         run, read_state)
    _assert_same(outs_e, outs_g, state_e, state_g)
    assert int(state_e[2][..., 0].sum()) > 0  # something was routed
    assert int(state_e[1][..., 2].max()) >= 2 * T  # positions from the last segment: they count the replays
    O_all = [torch.cat([o[0] for o in outs], dim=2) for outs in (outs_e, outs_g)]
    alpha = torch.full((spec.H, 64), 0.5, device="cuda")
    reads = [st.cache_attention(x["Q"], x["K"], x["V"], O, alpha, out=torch.empty_like(O))
             for st, O in zip(states, O_all)]
    torch.cuda.synchronize()
    for st in states:
        st.poll()
    assert torch.equal(reads[0], reads[1])


@pytest.mark.parametrize("form", ["scan", "prefix"])
def test_inplace_bf16_streams_through_a_graph(cwl, form):
    """Two chunks a call: the bf16 weight copy the next call starts from moves round the three
    buffers by two each call, and the captured call must follow it."""
    from chunked_weight_layers_b200 import abi
    T, n = 512, 4
    spec = workloads.scaled(workloads.INPLACE_4B, T=T * n, C=256, d=256, f=512, seed=514)
    x = workloads.inplace_inputs(spec, device="cuda")
    cfg = cwl.config("inplace", io_dtype=1, d_key=spec.f, d_val=spec.d, chunk=spec.C, eta=spec.eta)

    def make():
        st = cwl.FastWeightState(cfg, x["W0"])
        if form == "prefix":
            st.set_option(abi.TTT_OPT_INPLACE_PREFIX, 1)
        return st

    segs = [{"Z": x["Z"][i * T:(i + 1) * T].contiguous(), "Vhat": x["Vhat"][i * T:(i + 1) * T].contiguous()}
            for i in range(n)]

    def run(st, seg, outs):
        st.chunk_scan(seg["Z"], seg["Vhat"], out=outs[0])

    _assert_same(*_stream_both_ways(make, segs, lambda: [torch.empty((T, spec.d), device="cuda",
                                                                     dtype=torch.bfloat16)],
                                    run, lambda st: _weights(st, x["W0"])))


def test_inplace_f32_streams_through_a_graph(cwl):
    """Three chunks a call: the fp32 weight alternates between two buffers and must be back in
    the first one when the call ends."""
    T, n = 1536, 2
    spec = workloads.scaled(workloads.INPLACE_FP32, T=T * n, seed=515)
    x = workloads.inplace_inputs(spec, device="cuda")
    cfg = cwl.config("inplace", io_dtype=0, d_key=spec.f, d_val=spec.d, chunk=spec.C, eta=spec.eta)
    segs = [{"Z": x["Z"][i * T:(i + 1) * T].contiguous(), "Vhat": x["Vhat"][i * T:(i + 1) * T].contiguous()}
            for i in range(n)]

    def run(st, seg, outs):
        st.chunk_scan(seg["Z"], seg["Vhat"], out=outs[0])

    _assert_same(*_stream_both_ways(lambda: cwl.FastWeightState(cfg, x["W0"]), segs,
                                    lambda: [torch.empty((T, spec.d), device="cuda")], run,
                                    lambda st: _weights(st, x["W0"])))


def test_noalloc_target_call_captures():
    """ttt_target_values_noalloc after its first call on a device: capturing it in a graph
    (global capture mode, under which any call that allocates or synchronises fails the
    capture) succeeds, and replays over new inputs give the eager call's bits."""
    from chunked_weight_layers_b200 import abi, build
    build.build()
    lib = abi.load()
    spec = workloads.scaled(workloads.INPLACE_128K_TARGET, T=1024, C=256, d=512, f=384, seed=516)
    xs = [workloads.inplace_inputs(workloads.scaled(spec, seed=516 + i), device="cuda") for i in range(3)]
    status = torch.zeros((1,), device="cuda", dtype=torch.int32)

    def call(X0, V, stream):
        r = lib.ttt_target_values_noalloc(X0.data_ptr(), xs[0]["convw"].data_ptr(), xs[0]["Wtarget"].data_ptr(),
                                          spec.T, spec.d, spec.C, 3, 0, V.data_ptr(), status.data_ptr(), stream)
        assert r == abi.TTT_OK, lib.ttt_last_error_string()

    cur = torch.cuda.current_stream().cuda_stream or None
    eager = []
    for x in xs:
        V = torch.empty((spec.T, spec.d), device="cuda", dtype=torch.bfloat16)
        call(x["X0"], V, cur)
        eager.append(V)
    torch.cuda.synchronize()
    assert int(status.item()) == 0

    X0 = xs[0]["X0"].clone()
    V = torch.empty((spec.T, spec.d), device="cuda", dtype=torch.bfloat16)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side, capture_error_mode="global"):
            call(X0, V, side.cuda_stream)
    torch.cuda.current_stream().wait_stream(side)
    for x, ref in zip(xs, eager):
        X0.copy_(x["X0"])
        g.replay()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(V, ref)
