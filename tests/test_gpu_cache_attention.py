"""GPU parity of the residual-cache read path (ttt_cache_attention) against the oracle.

The cache is the one the GPU's gate built during the scan (its parity with the oracle's gate is
tested bit for bit elsewhere); the oracle reads the same entries, the same K, V, Q and the
GPU's own TTT outputs, so the comparison isolates the read path: the attention over the
visible entries and the α fusion."""

import numpy as np
import pytest
import torch

from gen import workloads
from oracle import cache_attention as oca
from tests._util import rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-2  # bf16 operands and output, fp32 softmax and accumulation


@pytest.fixture(scope="module")
def cwl():
    from chunked_weight_layers_b200 import build
    build.build()
    import chunked_weight_layers_b200 as cwl
    return cwl


def _scan_with_gate(cwl, spec, cap=256, calls=1):
    x = workloads.linear_inputs(spec, device="cuda")
    B, H, T = spec.B, spec.H, spec.T
    cfg = cwl.config("linear", batch=B, heads=H, chunk=16, eta=spec.eta, gate_enable=1, cache_capacity=cap)
    st = cwl.FastWeightState(cfg, x["W0"])
    O = torch.empty_like(x["K"])
    L = torch.empty((B, H, T), device="cuda")
    step = T // calls
    for a in range(0, T, step):
        sl = slice(a, a + step)
        Oc = torch.empty_like(x["K"][:, :, sl])
        Lc = torch.empty((B, H, step), device="cuda")
        st.chunk_scan(x["K"][:, :, sl].contiguous(), x["V"][:, :, sl].contiguous(), x["Q"][:, :, sl].contiguous(),
                      out=Oc, loss_out=Lc)
        O[:, :, sl] = Oc
        L[:, :, sl] = Lc
    E = torch.empty((B, H, cap, 3), device="cuda", dtype=torch.int32)
    C = torch.empty((B, H, 2), device="cuda", dtype=torch.int32)
    st.cache_read(E, C)
    torch.cuda.synchronize()
    st.poll()
    return st, x, O, E.cpu().numpy(), C.cpu().numpy()


def _alpha(H, seed):
    # Values below 0 and above 1 as well: the read path clamps them.
    g = torch.Generator().manual_seed(seed)
    return (torch.rand((H, 64), generator=g) * 1.6 - 0.3).cuda()


def _oracle(x, O, E, C, alpha, heads=None):
    """Oracle output for (b, h) pairs `heads` (all when None), as {(b, h): [T, 64]}."""
    Q, K, V = (x[n].cpu() for n in ("Q", "K", "V"))
    B, H, T, D = K.shape
    out = {}
    for b, h in heads or [(b, h) for b in range(B) for h in range(H)]:
        Eb = E[b:b + 1, h:h + 1].copy()
        n = min(int(C[b, h, 0]), Eb.shape[2])
        Eb[0, 0, :n, 0] = 0  # the oracle checks that entries name the (sequence, head) it reads
        Eb[0, 0, :n, 1] = 0
        A = oca.cache_attention(Q[b:b + 1, h:h + 1], K[b:b + 1, h:h + 1], V[b:b + 1, h:h + 1], Eb,
                                C[b:b + 1, h:h + 1])
        out[(b, h)] = oca.alpha_fusion(O[b:b + 1, h:h + 1].cpu(), A, alpha[h:h + 1].cpu())[0, 0]
    return out


@pytest.mark.parametrize("cap,calls", [(256, 1), (8, 1), (256, 3)])
def test_read_path_small(cwl, cap, calls):
    """B=2, H=3, T=1536 with queries: every (sequence, head) against the oracle; a cache of 8
    that overflows; the scan split over three calls (the cache and token positions carry on)."""
    spec = workloads.scaled(workloads.SR_TTT_GATE, B=2, H=3, T=1536, with_queries=True, seed=610 + cap)
    st, x, O, E, C = _scan_with_gate(cwl, spec, cap, calls)
    assert int(C[..., 0].sum()) > 0, "the needles should be routed"
    alpha = _alpha(spec.H, cap)
    out = st.cache_attention(x["Q"], x["K"], x["V"], O, alpha, out=torch.empty_like(O))
    torch.cuda.synchronize()
    st.poll()
    ref = _oracle(x, O, E, C, alpha)
    for (b, h), r in ref.items():
        assert rel_err(out[b, h], r) <= TOL, (b, h)
    # Tokens of the first gate chunk see no entry: their outputs are the TTT outputs exactly.
    assert torch.equal(out[:, :, :64], O[:, :, :64])


def test_read_path_in_place_and_empty_cache(cwl):
    """out may be o_ttt itself; with nothing routed (every token identical to the fixed point)
    the output is the TTT output bit for bit."""
    spec = workloads.scaled(workloads.SR_TTT_GATE, B=1, H=2, T=512, with_queries=True, seed=77)
    st, x, O, E, C = _scan_with_gate(cwl, spec)
    alpha = _alpha(spec.H, 3)
    ref = _oracle(x, O, E, C, alpha)
    O2 = O.clone()
    st.cache_attention(x["Q"], x["K"], x["V"], O2, alpha)  # in place
    torch.cuda.synchronize()
    for (b, h), r in ref.items():
        assert rel_err(O2[b, h], r) <= TOL
    # Empty cache: V = K and W0 = I make every residual, loss and p95 zero: nothing passes L > τ.
    x2 = dict(x)
    x2["V"] = x["K"].clone()
    cfg = cwl.config("linear", batch=1, heads=2, chunk=16, gate_enable=1)
    st2 = cwl.FastWeightState(cfg, x["W0"])
    O3 = torch.empty_like(x["K"])
    st2.chunk_scan(x2["K"], x2["V"], x2["Q"], out=O3, loss_out=torch.empty((1, 2, spec.T), device="cuda"))
    C3 = torch.empty((1, 2, 2), device="cuda", dtype=torch.int32)
    st2.cache_read(None, C3)
    out3 = st2.cache_attention(x2["Q"], x2["K"], x2["V"], O3, alpha, out=torch.empty_like(O3))
    torch.cuda.synchronize()
    assert int(C3.sum()) == 0 and torch.equal(out3, O3)


def test_read_path_rejects_bad_arguments(cwl):
    from chunked_weight_layers_b200 import TTTError, abi
    spec = workloads.scaled(workloads.SR_TTT_GATE, B=1, H=2, T=256, with_queries=True, seed=5)
    st, x, O, E, C = _scan_with_gate(cwl, spec)
    alpha = _alpha(2, 1)
    with pytest.raises(TTTError) as e:  # T must be the tokens scanned since the reset
        st.cache_attention(x["Q"][:, :, :128].contiguous(), x["K"][:, :, :128].contiguous(),
                           x["V"][:, :, :128].contiguous(), O[:, :, :128].contiguous(), alpha, T=128)
    assert e.value.status == abi.TTT_ERR_INVALID_ARG
    # A T beyond the tokens gated is caught on the device, which holds the count (the host's
    # misses replays of captured calls): the call returns and ttt_state_poll reports it once.
    two = {k: torch.cat([x[k], x[k]], dim=2).contiguous() for k in ("Q", "K", "V")}
    O2 = torch.cat([O, O], dim=2).contiguous()
    st.cache_attention(two["Q"], two["K"], two["V"], O2, alpha, out=torch.empty_like(O2), T=2 * spec.T)
    with pytest.raises(TTTError) as e:
        st.poll()
    assert e.value.status == abi.TTT_ERR_INVALID_ARG
    st.poll()
    W0 = torch.eye(64, device="cuda").expand(1, 2, 64, 64).contiguous()
    no_gate = cwl.FastWeightState(cwl.config("linear", batch=1, heads=2, chunk=16), W0)
    with pytest.raises(TTTError) as e:
        no_gate.cache_attention(x["Q"], x["K"], x["V"], O, alpha)
    assert e.value.status == abi.TTT_ERR_UNSUPPORTED


def test_read_path_gate_workload_sampled(cwl):
    """The SR-TTT workload (B=4, H=16, T=8192, queries drawn as well): four (sequence, head)
    pairs against the oracle in full (8192 queries each), the rest checked for what holds at any
    size: first-chunk outputs equal the TTT outputs, everything finite."""
    spec = workloads.scaled(workloads.SR_TTT_GATE, with_queries=True)
    st, x, O, E, C = _scan_with_gate(cwl, spec)
    alpha = _alpha(spec.H, 11)
    out = st.cache_attention(x["Q"], x["K"], x["V"], O, alpha, out=torch.empty_like(O))
    torch.cuda.synchronize()
    st.poll()
    assert torch.isfinite(out.float()).all()
    assert torch.equal(out[:, :, :64], O[:, :, :64])
    ref = _oracle(x, O, E, C, alpha, heads=[(0, 0), (1, 5), (2, 10), (3, 15)])
    for (b, h), r in ref.items():
        assert rel_err(out[b, h], r) <= TOL, (b, h)
    assert np.any(C[..., 0] > 0)
