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


def gate_state(cwl, B, H, cap=256):
    W0 = torch.eye(64, device="cuda").expand(B, H, 64, 64).contiguous()
    cfg = cwl.config("linear", batch=B, heads=H, chunk=16, gate_enable=1, cache_capacity=cap)
    return cwl.FastWeightState(cfg, W0)


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
    assert np.array_equal(tau.view(np.uint32), ref.tau.view(np.uint32))
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


def test_gated_scan_workload(cwl):
    """The SR-TTT workload: losses within tolerance of the oracle's; the oracle's gate on
    the GPU's losses reproduces the GPU cache exactly; against the oracle's own losses,
    routing may differ only for tokens or chunks within rounding of τ."""
    spec = workloads.SR_TTT_GATE
    x = workloads.linear_inputs(spec, device="cuda")
    B, H, T = spec.B, spec.H, spec.T
    st = gate_state(cwl, B, H)
    L = torch.empty((B, H, T), device="cuda")
    st.chunk_scan(x["K"], x["V"], None, out=None, loss_out=L)
    W = torch.empty_like(x["W0"])
    st.get_weights(W)
    E, C, tau, ts = read_gate(st, B, H, 256)
    _, Wref, Lref = olin.ttt_linear_scan(x["K"].cpu(), x["V"].cpu(), None, x["W0"].cpu(), spec.eta, spec.b)
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
    ref2 = ogate.GateState(B, H, 256)
    ogate.surprisal_route(Lref.astype(np.float32), ref2)
    diff = 0
    for b in range(B):
        for h in range(H):
            a = set(int(e[2]) for e in E[b, h] if e[2] >= 0)
            r = set(int(e[2]) for e in ref2.entries[b, h] if e[2] >= 0)
            diff += len(a ^ r)
    print(f"routing differences vs oracle losses: {diff}")
    assert diff <= 0.02 * max(1, int(C[..., 0].sum()))
