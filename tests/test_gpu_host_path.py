"""ttt_chunk_scan_host (host buffers): the call cuts T into segments whose copies in and out
overlap the scans of their neighbours, each segment continuing the scan as a separate call
would. Its outputs, losses, final weights and gate state must be the bits of one
ttt_chunk_scan over the same tokens in device memory, for every rule and form, with T cut
into unequal segments (a shorter last one) and, for the fused target's pad mode 1, not cut."""

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


def _pinned(t):
    return None if t is None else t.cpu().pin_memory()


def _both_paths(make, inputs, out_like, loss_like, read_state):
    """(device outputs, host outputs, device state, host state) for the same call."""
    keys, targets, queries = inputs
    st_d = make()
    out_d = None if out_like is None else torch.empty(out_like[0], dtype=out_like[1], device="cuda")
    loss_d = None if loss_like is None else torch.empty(loss_like, device="cuda")
    st_d.chunk_scan(keys, targets, queries, out=out_d, loss_out=loss_d)
    state_d = read_state(st_d)
    torch.cuda.synchronize()
    st_d.poll()

    st_h = make()
    out_h = None if out_like is None else torch.empty(out_like[0], dtype=out_like[1]).pin_memory()
    loss_h = None if loss_like is None else torch.empty(loss_like).pin_memory()
    T = keys.shape[-2]
    st_h.chunk_scan_host(_pinned(keys), _pinned(targets), _pinned(queries), out=out_h, loss_out=loss_h, T=T)
    state_h = read_state(st_h)
    torch.cuda.synchronize()
    st_h.poll()
    return [out_d, loss_d], [out_h, loss_h], state_d, state_h


def _assert_same(outs_d, outs_h, state_d, state_h):
    for j, (a, b) in enumerate(zip(outs_d, outs_h)):
        if a is not None:
            assert torch.equal(a.cpu(), b), f"output {j}"
    for j, (a, b) in enumerate(zip(state_d, state_h)):
        assert torch.equal(a, b), f"state {j}"


def _weights(like):
    def read(st):
        W = torch.empty_like(like)
        st.get_weights(W)
        return [W]
    return read


@pytest.mark.parametrize("model", ["linear", "linear_ln", "mlp"])
def test_ttt_linear_family(cwl, model):
    T = 16 * 13  # segments of 64, 64, 64 and 16 tokens
    if model == "linear":
        spec = workloads.scaled(workloads.LINEAR_GD, B=2, H=3, T=T, seed=521)
        x = workloads.linear_inputs(spec, device="cuda")
        cfg = cwl.config("linear", batch=spec.B, heads=spec.H, chunk=16, eta=spec.eta)
    else:
        base = workloads.LINEAR_LN if model == "linear_ln" else workloads.MLP
        spec = workloads.scaled(base, B=2, H=2, T=T, seed=522)
        x = workloads.inner_inputs(spec, device="cuda")
        cfg = cwl.config(model, batch=spec.B, heads=spec.H, eta=spec.eta, ln_eps=spec.eps)

    def make():
        st = cwl.FastWeightState(cfg, x["W0"])
        if model != "linear":
            st.set_layernorm(x["gamma"], x["beta"])
        return st

    shape = (spec.B, spec.H, T)
    _assert_same(*_both_paths(make, (x["K"], x["V"], x["Q"]), (shape + (64,), torch.bfloat16), shape,
                              _weights(x["W0"])))


def test_ttt_linear_without_queries(cwl):
    spec = workloads.scaled(workloads.LINEAR_GD, B=1, H=2, T=16 * 9, with_queries=False, seed=523)
    x = workloads.linear_inputs(spec, device="cuda")
    cfg = cwl.config("linear", batch=spec.B, heads=spec.H, chunk=16, eta=spec.eta)
    _assert_same(*_both_paths(lambda: cwl.FastWeightState(cfg, x["W0"]), (x["K"], x["V"], None), None,
                              (spec.B, spec.H, spec.T), _weights(x["W0"])))


def test_gated_scan(cwl):
    """Segments of 128, 128, 128 and 64 tokens (whole gate chunks): τ, cache and counts as well."""
    T, cap = 64 * 7, 256
    spec = workloads.scaled(workloads.SR_TTT_GATE, B=1, H=2, T=T, with_queries=True, seed=524)
    x = workloads.linear_inputs(spec, device="cuda")
    cfg = cwl.config("linear", batch=spec.B, heads=spec.H, chunk=16, eta=spec.eta, gate_enable=1,
                     cache_capacity=cap)

    def read_state(st):
        E = torch.empty((spec.B, spec.H, cap, 3), device="cuda", dtype=torch.int32)
        C = torch.empty((spec.B, spec.H, 2), device="cuda", dtype=torch.int32)
        tau = torch.empty((spec.B, spec.H), device="cuda")
        tau_set = torch.empty((spec.B, spec.H), device="cuda", dtype=torch.int32)
        st.cache_read(E, C)
        st.gate_read(tau, tau_set)
        return _weights(x["W0"])(st) + [E, C, tau, tau_set]

    shape = (spec.B, spec.H, T)
    outs_d, outs_h, state_d, state_h = _both_paths(lambda: cwl.FastWeightState(cfg, x["W0"]),
                                                   (x["K"], x["V"], x["Q"]), (shape + (64,), torch.bfloat16),
                                                   shape, read_state)
    _assert_same(outs_d, outs_h, state_d, state_h)
    assert int(state_d[2][..., 0].sum()) > 0


@pytest.mark.parametrize("target_mode,pad_mode", [(0, 0), (1, 0), (1, 1)])
def test_inplace_bf16(cwl, target_mode, pad_mode):
    """Five chunks: segments of two, two and one chunk (pad mode 1: the whole call at once)."""
    C = 256
    base = workloads.INPLACE_128K_TARGET if target_mode else workloads.INPLACE_4B
    spec = workloads.scaled(base, T=5 * C, C=C, d=256, f=384, seed=525 + target_mode + pad_mode)
    x = workloads.inplace_inputs(spec, device="cuda")
    cfg = cwl.config("inplace", io_dtype=1, d_key=spec.f, d_val=spec.d, chunk=C, eta=spec.eta,
                     target_mode=target_mode, conv_pad_mode=pad_mode)

    def make():
        if target_mode:
            return cwl.FastWeightState(cfg, x["W0"], x["Wtarget"], x["convw"])
        return cwl.FastWeightState(cfg, x["W0"])

    targets = x["X0"] if target_mode else x["Vhat"]
    _assert_same(*_both_paths(make, (x["Z"], targets, None), ((spec.T, spec.d), torch.bfloat16), None,
                              _weights(x["W0"])))


def test_inplace_f32(cwl):
    """Five chunks of 512: segments of two, two and one chunk (an odd count in the last)."""
    spec = workloads.scaled(workloads.INPLACE_FP32, T=5 * 512, seed=528)
    x = workloads.inplace_inputs(spec, device="cuda")
    cfg = cwl.config("inplace", io_dtype=0, d_key=spec.f, d_val=spec.d, chunk=spec.C, eta=spec.eta)
    _assert_same(*_both_paths(lambda: cwl.FastWeightState(cfg, x["W0"]), (x["Z"], x["Vhat"], None),
                              ((spec.T, spec.d), torch.float32), None, _weights(x["W0"])))


def test_pageable_host_buffers(cwl):
    """Host buffers that are not pinned: the copies do not overlap, the results are the same."""
    spec = workloads.scaled(workloads.LINEAR_GD, B=2, H=2, T=16 * 11, seed=529)
    x = workloads.linear_inputs(spec, device="cuda")
    cfg = cwl.config("linear", batch=spec.B, heads=spec.H, chunk=16, eta=spec.eta)
    shape = (spec.B, spec.H, spec.T)
    st_d = cwl.FastWeightState(cfg, x["W0"])
    O_d, L_d = torch.empty(shape + (64,), device="cuda", dtype=torch.bfloat16), torch.empty(shape, device="cuda")
    st_d.chunk_scan(x["K"], x["V"], x["Q"], out=O_d, loss_out=L_d)
    st_h = cwl.FastWeightState(cfg, x["W0"])
    O_h, L_h = torch.empty(shape + (64,), dtype=torch.bfloat16), torch.empty(shape)
    st_h.chunk_scan_host(x["K"].cpu(), x["V"].cpu(), x["Q"].cpu(), out=O_h, loss_out=L_h)
    torch.cuda.synchronize()
    assert torch.equal(O_d.cpu(), O_h) and torch.equal(L_d.cpu(), L_h)
    assert torch.equal(_weights(x["W0"])(st_d)[0], _weights(x["W0"])(st_h)[0])
