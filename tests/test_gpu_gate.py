"""GPU parity of the surprisal gate (standalone and fused after the TTT-Linear scan).

The integer outputs (cache entries, counts) are compared bit for bit with the oracle's
gate run on the same fp32 loss array; τ is compared bit for bit as well."""

import json
import os

import numpy as np
import pytest
import torch

from gen import workloads
from oracle import gate as ogate
from oracle import linear as olin
from tests._util import rel_err

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def cwl():
    from chunked_weight_layers_b200 import build
    build.build()
    import chunked_weight_layers_b200 as cwl
    return cwl


def gate_state(cwl, B, H, cap=256, form=None):
    W0 = torch.eye(64, device="cuda").expand(B, H, 64, 64).contiguous()
    cfg = cwl.config("linear", batch=B, heads=H, chunk=16, gate_enable=1, cache_capacity=cap)
    st = cwl.FastWeightState(cfg, W0)
    if form is not None:
        st.set_option(cwl.abi.TTT_OPT_LINEAR_CHUNK, form)
    return st


def read_gate(st, B, H, cap):
    E = torch.empty((B, H, cap, 3), device="cuda", dtype=torch.int32)
    C = torch.empty((B, H, 2), device="cuda", dtype=torch.int32)
    tau = torch.empty((B, H), device="cuda", dtype=torch.float32)
    ts = torch.empty((B, H), device="cuda", dtype=torch.int32)
    st.cache_read(E, C)
    st.gate_read(tau, ts)
    torch.cuda.synchronize()
    st.poll()
    return E.cpu().numpy(), C.cpu().numpy(), tau.cpu().numpy(), ts.cpu().numpy()


def assert_same_as_oracle(E, C, tau, ts, ref: ogate.GateState):
    assert np.array_equal(E, ref.entries)
    assert np.array_equal(C, ref.counts())
    # τ bit for bit; a NaN τ only as NaN (IEEE 754 leaves NaN payloads open: the GPU's
    # arithmetic returns its canonical NaN, numpy's propagates the operand's).
    both_nan = np.isnan(tau) & np.isnan(ref.tau)
    assert np.array_equal(np.where(both_nan, 0, tau.view(np.uint32)), np.where(both_nan, 0, ref.tau.view(np.uint32)))
    assert np.array_equal(ts.astype(bool), ref.tau_set)


def test_hand_cases_bit_exact(cwl):
    g = json.load(open(os.path.join(GOLDEN, "gate_hand.json")))
    for name in ("needles", "all_equal", "mean_boundary", "mean_just_below", "ema"):
        loss = np.concatenate([np.asarray(x, np.float32) for x in g[name]["loss"]])[None, None]
        st = gate_state(cwl, 1, 1)
        st.surprisal_route(torch.from_numpy(loss).cuda())
        E, C, tau, ts = read_gate(st, 1, 1, 256)
        routed = [int(e[2]) for e in E[0, 0] if e[2] >= 0]
        assert routed == g[name]["routed_t"], name
        assert tau[0, 0] == np.float32(g[name]["tau"][-1])
    c = g["capacity"]
    loss = np.ones(64 * c["chunks"], np.float32)
    for k in range(c["chunks"]):
        for o in c["needle_offsets"]:
            loss[64 * k + o] = 100.0
    st = gate_state(cwl, 1, 1, c["capacity"])
    st.surprisal_route(torch.from_numpy(loss[None, None]).cuda())
    E, C, _, _ = read_gate(st, 1, 1, c["capacity"])
    assert C[0, 0, 0] == c["routed"] and C[0, 0, 1] == c["dropped"]
    assert E[0, 0, -1, 2] == c["last_stored_t"]


def _random_losses(B, H, T, seed):
    rng = np.random.default_rng(seed)
    L = (rng.standard_normal((B, H, T)) ** 2 + rng.standard_normal((B, H, T)) ** 2).astype(np.float32)
    idx = rng.integers(0, T, (B, H, T // 80))
    for b in range(B):
        for h in range(H):
            L[b, h, idx[b, h]] *= np.float32(40.0)
    L[0, 0, :64] = 1.0  # a chunk of ties
    return L


@pytest.mark.parametrize("cap", [256, 8])
def test_random_losses_bit_exact(cwl, cap):
    B, H, T = 4, 16, 8192
    L = _random_losses(B, H, T, 3 + cap)
    st = gate_state(cwl, B, H, cap)
    st.surprisal_route(torch.from_numpy(L).cuda())
    ref = ogate.GateState(B, H, cap)
    ogate.surprisal_route(L, ref)
    assert_same_as_oracle(*read_gate(st, B, H, cap), ref)


def test_streaming_calls_and_reset(cwl):
    B, H, T = 2, 3, 64 * 70
    L = _random_losses(B, H, T, 11)
    st = gate_state(cwl, B, H, 64)
    Ld = torch.from_numpy(L).cuda()
    st.surprisal_route(Ld[:, :, :64 * 13].contiguous())
    st.surprisal_route(Ld[:, :, 64 * 13:].contiguous())
    ref = ogate.GateState(B, H, 64)
    ogate.surprisal_route(L, ref)
    assert_same_as_oracle(*read_gate(st, B, H, 64), ref)
    st.reset()
    st.surprisal_route(Ld)
    assert_same_as_oracle(*read_gate(st, B, H, 64), ref)


@pytest.fixture(scope="module")
def gate_workload_ref():
    spec = workloads.SR_TTT_GATE
    x = workloads.linear_inputs(spec, device="cpu")
    _, Wref, Lref = olin.ttt_linear_scan(x["K"], x["V"], None, x["W0"], spec.eta, spec.b)
    ref2 = ogate.GateState(spec.B, spec.H, 256)
    ogate.surprisal_route(Lref.astype(np.float32), ref2)
    return Wref, Lref, ref2


@pytest.mark.parametrize("form", [1, 2, 4])
def test_gated_scan_workload(cwl, gate_workload_ref, form):
    """The SR-TTT workload: losses within tolerance of the oracle's; the oracle's gate on
    the GPU's losses reproduces the GPU cache exactly; against the oracle's own losses,
    routing may differ only for tokens or chunks within rounding of τ. For the step-by-step
    form and both chunked forms of the scan."""
    spec = workloads.SR_TTT_GATE
    x = workloads.linear_inputs(spec, device="cuda")
    B, H, T = spec.B, spec.H, spec.T
    st = gate_state(cwl, B, H, form=form)
    L = torch.empty((B, H, T), device="cuda")
    st.chunk_scan(x["K"], x["V"], None, out=None, loss_out=L)
    W = torch.empty_like(x["W0"])
    st.get_weights(W)
    E, C, tau, ts = read_gate(st, B, H, 256)
    Wref, Lref, ref2 = gate_workload_ref
    el, ew = rel_err(L, Lref), rel_err(W, Wref)
    print(f"SR-TTT workload: loss {el:.3e}  W {ew:.3e}  routed {int(C[..., 0].sum())}")
    assert el <= 2e-2 and ew <= 2e-2
    Lgpu = L.cpu().numpy()
    ref = ogate.GateState(B, H, 256)
    ogate.surprisal_route(Lgpu, ref)
    assert_same_as_oracle(E, C, tau, ts, ref)
    # Needles are what the gate catches.
    assert int(C[..., 0].sum()) > 0
    # Against the oracle's own losses: differences only at the rounding margin.
    diff = 0
    for b in range(B):
        for h in range(H):
            a = set(int(e[2]) for e in E[b, h] if e[2] >= 0)
            r = set(int(e[2]) for e in ref2.entries[b, h] if e[2] >= 0)
            diff += len(a ^ r)
    print(f"routing differences vs oracle losses: {diff}")
    assert diff <= 0.02 * max(1, int(C[..., 0].sum()))


@pytest.mark.parametrize("form", [1, 2, 4])
@pytest.mark.parametrize("with_q", [False, True])
def test_gate_inside_the_scan_streams_and_saturates(cwl, with_q, form):
    """The b = 16 scan runs the gate in its own kernel, tile by tile. Two calls (tokens
    0..319 and 320..767) with a cache of 8 entries, so it fills up and drops: the cache,
    counts and τ equal the oracle's gate run over the GPU's losses of both calls, bit for
    bit, with or without query outputs."""
    spec = workloads.scaled(workloads.SR_TTT_GATE, B=2, H=3, T=768, seed=91)
    x = workloads.linear_inputs(spec, device="cuda")
    B, H, T, cap = spec.B, spec.H, spec.T, 8
    st = gate_state(cwl, B, H, cap, form=form)
    losses = []
    for a, z in ((0, 320), (320, T)):
        K, V = (x[n][:, :, a:z].contiguous() for n in ("K", "V"))
        L = torch.empty((B, H, z - a), device="cuda")
        if with_q:
            st.chunk_scan(K, V, K, out=torch.empty_like(K), loss_out=L)
        else:
            st.chunk_scan(K, V, None, out=None, loss_out=L)
        losses.append(L)
    E, C, tau, ts = read_gate(st, B, H, cap)
    ref = ogate.GateState(B, H, cap)
    ogate.surprisal_route(torch.cat(losses, 2).cpu().numpy(), ref)
    assert_same_as_oracle(E, C, tau, ts, ref)
    assert int(C[..., 1].sum()) > 0, "the small cache should overflow"


def test_wide_range_and_negative_losses_bit_exact(cwl):
    """Chunks whose losses span far more than 2^23 (so their double sums are not exact in
    every order and are taken in index order), and a head of signed values: cache, counts
    and τ equal the oracle's bit for bit."""
    rng = np.random.default_rng(5)
    B, H, T = 2, 2, 64 * 40
    L = (rng.standard_normal((B, H, T)) ** 2).astype(np.float32)
    L *= np.exp2(rng.integers(-40, 40, (B, H, T))).astype(np.float32)
    L[1, 1] = rng.standard_normal(T).astype(np.float32)
    st = gate_state(cwl, B, H, 64)
    st.surprisal_route(torch.from_numpy(L).cuda())
    ref = ogate.GateState(B, H, 64)
    ogate.surprisal_route(L, ref)
    assert_same_as_oracle(*read_gate(st, B, H, 64), ref)


@pytest.mark.parametrize("pct", [0.95, 0.5, 0.05])
def test_percentile_ranks_and_nans_bit_exact(cwl, pct):
    """Top ranks take the max-peeling selection, others the counting one; chunks with ties,
    NaNs (sorted last) and infinities give the oracle's percentile, τ and routing."""
    rng = np.random.default_rng(int(pct * 100))
    B, H, T = 1, 3, 64 * 24
    L = np.round(rng.standard_normal((B, H, T)) * 4).astype(np.float32) ** 2  # many ties
    L[0, 1, 64:66] = np.nan
    L[0, 1, 130:140] = np.nan
    L[0, 1, 200] = np.inf
    L[0, 2, 64 * 5:64 * 6] = np.nan
    W0 = torch.eye(64, device="cuda").expand(B, H, 64, 64).contiguous()
    st = cwl.FastWeightState(cwl.config("linear", batch=B, heads=H, chunk=16, gate_enable=1, gate_pct=pct), W0)
    st.surprisal_route(torch.from_numpy(L).cuda())
    ref = ogate.GateState(B, H, 256)
    ogate.surprisal_route(L, ref, pct=pct)
    assert_same_as_oracle(*read_gate(st, B, H, 256), ref)


def test_token_position_is_kept_and_checked_on_the_device(cwl):
    """The gate's token position lives on the device (so replays of captured calls advance it):
    set there to 1000, a scan's routed positions are those of a fresh state plus 1000, and the
    cache read then wants T = 1256 (found on the device: the host counted 256); set near 2^31,
    a scan that passes 2^31 - 1 is reported by ttt_state_poll."""
    from chunked_weight_layers_b200 import TTTError, abi
    spec = workloads.scaled(workloads.SR_TTT_GATE, B=1, H=2, T=256, with_queries=True, seed=531)
    x = workloads.linear_inputs(spec, device="cuda")
    cfg = cwl.config("linear", batch=1, heads=2, chunk=16, eta=spec.eta, gate_enable=1)

    def run(base):
        st = cwl.FastWeightState(cfg, x["W0"])
        if base is not None:
            st.set_option(abi.TTT_OPT_GATE_TOKENS, base)
        O = torch.empty_like(x["K"])
        st.chunk_scan(x["K"], x["V"], x["Q"], out=O, loss_out=torch.empty((1, 2, spec.T), device="cuda"))
        E = torch.empty((1, 2, 256, 3), device="cuda", dtype=torch.int32)
        C = torch.empty((1, 2, 2), device="cuda", dtype=torch.int32)
        st.cache_read(E, C)
        torch.cuda.synchronize()
        return st, O, E.cpu(), C.cpu()

    st0, _, E0, C0 = run(None)
    st0.poll()
    st1, O1, E1, C1 = run(1000)
    st1.poll()
    assert torch.equal(C0, C1)
    valid = E0[..., 2] >= 0
    assert torch.equal(E1[..., 2][valid], E0[..., 2][valid] + 1000)
    assert torch.equal(E1[..., :2], E0[..., :2])
    alpha = torch.full((2, 64), 0.5, device="cuda")
    st1.cache_attention(x["Q"], x["K"], x["V"], O1, alpha, out=torch.empty_like(O1))
    with pytest.raises(TTTError) as e:
        st1.poll()
    assert e.value.status == abi.TTT_ERR_INVALID_ARG
    st2, _, _, _ = run(2**31 - 64)
    with pytest.raises(TTTError) as e:
        st2.poll()
    assert e.value.status == abi.TTT_ERR_UNSUPPORTED
    st2.poll()  # the record was cleared
    with pytest.raises(TTTError) as e:
        cwl.FastWeightState(cwl.config("inplace", io_dtype=1, d_key=128, d_val=128, chunk=128),
                            torch.zeros((128, 128), device="cuda")).set_option(abi.TTT_OPT_GATE_TOKENS, 5)
    assert e.value.status == abi.TTT_ERR_UNSUPPORTED
