"""Bounded device-side waits that run out (failure detection without a GPU fault).

Every spin-wait of the library's kernels gives up after the state's wait limit, records
TTT_ERR_TIMEOUT in the state's status word, drains its own copies and tensor-core work in
flight, frees its tensor memory and returns. Here a host-side injection (TTT_OPT_INJECT_STALL)
makes one wait wait for something that never comes — an In-Place APPLY tile waits for one
more finished UPDATE tile than exists; the TTT-Linear scan never loads its second tile — with
a short limit (5 ms). The launch returns, ttt_state_poll reports TTT_ERR_TIMEOUT, and the
device stays usable: the same state after a reset and a fresh state both scan again to the
oracle's results (an In-Place kernel that had kept its tensor memory would leave the next
launch unable to allocate it)."""

import pytest
import torch

from gen import workloads
from oracle import inplace as oinp
from oracle import linear as olin
from tests._util import rel_err

pytestmark = pytest.mark.gpu
LIMIT_NS = 5_000_000


@pytest.fixture(scope="module")
def cwl():
    from chunked_weight_layers_b200 import build
    build.build()
    import chunked_weight_layers_b200 as cwl
    return cwl


def _expect_timeout(st):
    from chunked_weight_layers_b200 import TTTError, abi
    with pytest.raises(TTTError) as e:
        st.poll()
    assert e.value.status == abi.TTT_ERR_TIMEOUT
    st.poll()  # the record is cleared by the poll that returned it


@pytest.mark.parametrize("form", [1, 2])
def test_linear_scan_wait_runs_out(cwl, form):
    from chunked_weight_layers_b200 import abi
    spec = workloads.scaled(workloads.LINEAR_GD, B=1, H=4, T=256, seed=404)
    x = workloads.linear_inputs(spec, device="cuda")
    cfg = cwl.config("linear", batch=1, heads=4, chunk=16, eta=1.0)

    def scan(st):
        O = torch.empty_like(x["K"])
        L = torch.empty((1, 4, spec.T), device="cuda")
        st.chunk_scan(x["K"], x["V"], x["Q"], out=O, loss_out=L)
        W = torch.empty_like(x["W0"])
        st.get_weights(W)
        return O, W, L

    st = cwl.FastWeightState(cfg, x["W0"])
    st.set_option(abi.TTT_OPT_LINEAR_CHUNK, form)
    st.set_option(abi.TTT_OPT_WAIT_LIMIT_NS, LIMIT_NS)
    st.set_option(abi.TTT_OPT_INJECT_STALL, 1)
    scan(st)
    _expect_timeout(st)

    Oref, Wref, Lref = olin.ttt_linear_scan(x["K"].cpu(), x["V"].cpu(), x["Q"].cpu(), x["W0"].cpu(), 1.0, 16)
    st.reset()
    O, W, L = scan(st)  # the injection was used up: this scan runs normally
    st.poll()
    assert rel_err(O, Oref) <= 1e-2 and rel_err(W, Wref) <= 5e-3 and rel_err(L, Lref) <= 5e-3
    fresh = cwl.FastWeightState(cfg, x["W0"])
    fresh.set_option(abi.TTT_OPT_LINEAR_CHUNK, form)
    O2, W2, L2 = scan(fresh)
    fresh.poll()
    assert torch.equal(O2, O) and torch.equal(W2, W) and torch.equal(L2, L)


@pytest.mark.parametrize("C", [128, 256])
def test_inplace_tensor_core_scan_wait_runs_out(cwl, C):
    """C = 128: one CTA per tile; C = 256 (d = 256): clusters of two CTAs per tile, where the
    CTAs of a pair also wait on each other."""
    from chunked_weight_layers_b200 import abi
    spec = workloads.scaled(workloads.INPLACE_4B, T=2 * C, C=C, d=256, f=256, seed=405)
    x = workloads.inplace_inputs(spec, device="cuda")
    cfg = cwl.config("inplace", io_dtype=1, d_key=256, d_val=256, chunk=C, eta=spec.eta)

    def scan(st):
        O = torch.empty((spec.T, spec.d), device="cuda", dtype=torch.bfloat16)
        st.chunk_scan(x["Z"], x["Vhat"], out=O)
        W = torch.empty_like(x["W0"])
        st.get_weights(W)
        return O, W

    st = cwl.FastWeightState(cfg, x["W0"])
    st.set_option(abi.TTT_OPT_WAIT_LIMIT_NS, LIMIT_NS)
    st.set_option(abi.TTT_OPT_INJECT_STALL, 1)
    scan(st)  # two chunks: one launch of two rounds; round 1's APPLY tiles wait in vain
    _expect_timeout(st)

    Oref, Wref = oinp.inplace_scan(x["Z"].cpu(), x["Vhat"].cpu(), x["W0"].cpu(), spec.eta, C)
    st.reset()
    O, W = scan(st)
    st.poll()
    assert rel_err(O, Oref) <= 2e-2 and rel_err(W, Wref) <= 2e-2
    fresh = cwl.FastWeightState(cfg, x["W0"])
    O2, W2 = scan(fresh)
    fresh.poll()
    assert torch.equal(O2, O) and torch.equal(W2, W)


def test_option_ranges(cwl):
    from chunked_weight_layers_b200 import TTTError, abi
    W0 = torch.eye(64, device="cuda").expand(1, 1, 64, 64).contiguous()
    st = cwl.FastWeightState(cwl.config("linear", batch=1, heads=1, chunk=16), W0)
    for opt, bad in ((abi.TTT_OPT_WAIT_LIMIT_NS, 999), (abi.TTT_OPT_WAIT_LIMIT_NS, 60_000_000_001),
                     (abi.TTT_OPT_INJECT_STALL, 2), (abi.TTT_OPT_SM_PAIR, 2)):
        with pytest.raises(TTTError) as e:
            st.set_option(opt, bad)
        assert e.value.status == abi.TTT_ERR_INVALID_ARG
    st.set_option(abi.TTT_OPT_WAIT_LIMIT_NS, 2_000_000_000)
    st.set_option(abi.TTT_OPT_INJECT_STALL, 0)


@pytest.mark.parametrize("model", ["linear_ln", "mlp"])
def test_inner_model_scan_wait_runs_out(cwl, model):
    """The LayerNorm TTT-Linear and TTT-MLP scans never get their second 64-token tile: their
    waits give up, TTT_ERR_TIMEOUT is reported, and a reset state then scans like a fresh one
    (bit for bit) and like the oracle."""
    from chunked_weight_layers_b200 import abi
    from oracle import inner as oinn
    base = workloads.LINEAR_LN if model == "linear_ln" else workloads.MLP
    spec = workloads.scaled(base, B=1, H=3, T=256, seed=406)
    x = workloads.inner_inputs(spec, device="cuda")
    cfg = cwl.config(model, batch=1, heads=3, eta=spec.eta, ln_eps=spec.eps)

    def make():
        st = cwl.FastWeightState(cfg, x["W0"])
        st.set_layernorm(x["gamma"], x["beta"])
        return st

    def scan(st):
        O = torch.empty_like(x["K"])
        L = torch.empty((1, 3, spec.T), device="cuda")
        st.chunk_scan(x["K"], x["V"], x["Q"], out=O, loss_out=L)
        W = torch.empty_like(x["W0"])
        st.get_weights(W)
        return O, W, L

    st = make()
    st.set_option(abi.TTT_OPT_WAIT_LIMIT_NS, LIMIT_NS)
    st.set_option(abi.TTT_OPT_INJECT_STALL, 1)
    scan(st)
    _expect_timeout(st)
    st.reset()
    O, W, L = scan(st)  # the injection was used up: this scan runs normally
    st.poll()
    O2, W2, L2 = scan(make())
    torch.cuda.synchronize()
    assert torch.equal(O, O2) and torch.equal(W, W2) and torch.equal(L, L2)
    c = {k: v.cpu() for k, v in x.items() if isinstance(v, torch.Tensor)}
    if model == "linear_ln":
        Oref = oinn.ttt_linear_ln_scan(c["K"], c["V"], c["Q"], c["W0"], c["gamma"], c["beta"], spec.eta, 16, spec.eps)[0]
    else:
        Oref = oinn.ttt_mlp_scan(c["K"], c["V"], c["Q"], c["W1"], c["W2"], c["gamma"], c["beta"], spec.eta, 16,
                                 spec.eps)[0]
    assert rel_err(O, Oref) <= 2e-2
