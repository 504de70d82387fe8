"""GPU parity of packed sequences for the TTT-Linear family (plain, LayerNorm and MLP rules:
per-document resets to the pretrained weights, mini-batches counted from each document's first
token, a shorter last mini-batch stepping on its own loss) and of per-token weights for the
plain rule, against the oracle ("In-Place Test-Time Training", §6 notes; the TTT layers page)."""

import numpy as np
import pytest
import torch

from gen import workloads
from oracle import linear as olin
from oracle import packed as opk
from tests._util import rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def cwl():
    from chunked_weight_layers_b200 import build
    build.build()
    import chunked_weight_layers_b200 as cwl
    return cwl


def inputs(model, B, H, T, seed):
    base = {"linear": workloads.LINEAR_LN, "linear_ln": workloads.LINEAR_LN, "mlp": workloads.MLP}[model]
    spec = workloads.scaled(base, B=B, H=H, T=T, seed=seed)
    x = workloads.inner_inputs(spec, device="cuda")
    if model == "linear":
        # The plain rule at the TTT-Linear workload's step size and a weight away from I.
        x["W0"] = x["W0"] + 0.05 * torch.randn(x["W0"].shape, generator=torch.Generator().manual_seed(seed)).cuda()
    return spec, x


def state(cwl, model, spec, x, token_weights=0):
    eta = 1.0 if model == "linear" else spec.eta
    cfg = cwl.config(model, batch=spec.B, heads=spec.H, chunk=16, eta=eta, ln_eps=spec.eps, token_weights=token_weights)
    st = cwl.FastWeightState(cfg, x["W0"])
    if model != "linear":
        st.set_layernorm(x["gamma"], x["beta"])
    return st, eta


def run_packed(cwl, model, spec, x, starts, token_weights=0):
    st, eta = state(cwl, model, spec, x, token_weights)
    O = torch.full_like(x["K"], float("nan"))
    L = torch.full(x["K"].shape[:3], float("nan"), device="cuda")
    st.chunk_scan_packed(x["K"], x["V"], starts, queries=x["Q"], out=O, loss_out=L)
    W = torch.empty_like(x["W0"])
    st.get_weights(W)
    torch.cuda.synchronize()
    st.poll()
    return O, W, L, eta


def oracle_packed(model, spec, x, starts, eta, token_weights=False):
    c = {k: v.cpu() for k, v in x.items() if isinstance(v, torch.Tensor)}
    if model == "linear":
        return opk.ttt_linear_scan_docs(c["K"], c["V"], c["Q"], c["W0"], eta, 16, starts, token_weights=token_weights)
    W0 = (c["W1"], c["W2"]) if model == "mlp" else c["W0"]
    O, W, L = opk.inner_scan_docs(model, c["K"], c["V"], c["Q"], W0, c["gamma"], c["beta"], eta, 16, spec.eps, starts,
                                  token_weights=token_weights)
    if model == "mlp":
        W = np.concatenate([W[0].reshape(spec.B, spec.H, -1), W[1].reshape(spec.B, spec.H, -1)], axis=2)
    return O, W, L


def weight_err(model, spec, W, Wref):
    if model != "mlp":
        return rel_err(W, Wref)
    n1 = 64 * spec.hidden
    return max(rel_err(W[..., :n1], Wref[..., :n1]), rel_err(W[..., n1:], Wref[..., n1:]))


MODELS = ["linear", "linear_ln", "mlp"]
LAYOUTS = [
    # T, per-sequence document starts: ragged documents, a one-token document, a document that
    # ends mid-mini-batch, a sequence of one document, T not a multiple of 16.
    (200, [[0, 37, 38, 120], [0], [0, 16, 100, 199]]),
    (64, [[0, 1, 2, 3], [0, 63], [0, 32]]),
]


@pytest.mark.parametrize("model", MODELS)
@pytest.mark.parametrize("token_weights", [0, 1])
@pytest.mark.parametrize("layout", range(len(LAYOUTS)))
def test_packed_against_oracle(cwl, model, token_weights, layout):
    T, starts = LAYOUTS[layout]
    spec, x = inputs(model, 3, 2, T, 3100 + layout)
    O, W, L, eta = run_packed(cwl, model, spec, x, starts, token_weights)
    Oref, Wref, Lref = oracle_packed(model, spec, x, starts, eta, bool(token_weights))
    eo, ew, el = rel_err(O, Oref), weight_err(model, spec, W, Wref), rel_err(L, Lref)
    print(f"{model} tw={token_weights} T={T}: O {eo:.3e}  W {ew:.3e}  loss {el:.3e}")
    assert eo <= TOL and ew <= TOL and el <= TOL


@pytest.mark.parametrize("model", ["linear_ln", "mlp"])
def test_one_document_equals_the_scan(cwl, model):
    """One document of whole mini-batches per sequence is the plain scan, bit for bit (the same
    launch over a copy, started from W0)."""
    spec, x = inputs(model, 2, 2, 128, 3200)
    O, W, L, eta = run_packed(cwl, model, spec, x, [[0], [0]])
    st, _ = state(cwl, model, spec, x)
    O2, L2 = torch.empty_like(O), torch.empty_like(L)
    st.chunk_scan(x["K"], x["V"], x["Q"], out=O2, loss_out=L2)
    W2 = torch.empty_like(W)
    st.get_weights(W2)
    torch.cuda.synchronize()
    assert torch.equal(O, O2) and torch.equal(W, W2) and torch.equal(L, L2)


@pytest.mark.parametrize("T", [208, 2048])
def test_plain_rule_token_weights(cwl, T):
    """Per-token weights for the plain TTT-Linear rule (the dual form, run by the LayerNorm
    kernel's plain mode): outputs against the oracle, losses and weights as the default form's."""
    spec = workloads.scaled(workloads.LINEAR_GD, B=2 if T < 2048 else 8, H=3 if T < 2048 else 12, T=T, seed=3300)
    x = workloads.linear_inputs(spec, device="cuda")
    cfg = cwl.config("linear", batch=spec.B, heads=spec.H, chunk=16, eta=spec.eta, token_weights=1)
    st = cwl.FastWeightState(cfg, x["W0"])
    O = torch.empty_like(x["K"])
    L = torch.empty(x["K"].shape[:3], device="cuda")
    st.chunk_scan(x["K"], x["V"], x["Q"], out=O, loss_out=L)
    W = torch.empty_like(x["W0"])
    st.get_weights(W)
    torch.cuda.synchronize()
    st.poll()
    Oref, Wref, Lref = olin.ttt_linear_scan(x["K"].cpu(), x["V"].cpu(), x["Q"].cpu(), x["W0"].cpu(), spec.eta, 16,
                                            token_weights=True)
    eo, ew, el = rel_err(O, Oref), rel_err(W, Wref), rel_err(L, Lref)
    print(f"plain TTT-Linear per-token weights T={T}: O {eo:.3e}  W {ew:.3e}  loss {el:.3e}")
    assert eo <= TOL and ew <= TOL and el <= TOL


def test_packed_rejects(cwl):
    from chunked_weight_layers_b200 import TTTError, abi
    spec, x = inputs("linear_ln", 2, 1, 64, 3400)
    st, _ = state(cwl, "linear_ln", spec, x)
    O = torch.empty_like(x["K"])
    for starts in ([[1], [0]], [[0, 5, 5], [0]], [[0], [0, 64]], [[0]]):
        with pytest.raises((TTTError, ValueError)) as e:
            st.chunk_scan_packed(x["K"], x["V"], starts, queries=x["Q"], out=O)
        if isinstance(e.value, TTTError):
            assert e.value.status == abi.TTT_ERR_INVALID_ARG, starts
    gated = cwl.FastWeightState(cwl.config("linear", batch=2, heads=1, gate_enable=1), x["W0"])
    with pytest.raises(TTTError) as e:
        gated.chunk_scan_packed(x["K"], x["V"], [[0], [0]], loss_out=torch.empty(2, 1, 64, device="cuda"))
    assert e.value.status == abi.TTT_ERR_UNSUPPORTED
