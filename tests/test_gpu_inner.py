"""GPU parity of the richer inner models (TTT-Linear with LayerNorm and residual, TTT-MLP)
against the oracle: the TTT layers page's two instances, with the LayerNorm and residual that
its DeltaNet remark places in the full TTT-Linear."""

import numpy as np
import pytest
import torch

from gen import workloads
from oracle import inner as ora
from tests._util import rel_err, to_np

pytestmark = pytest.mark.gpu

TOL = 2e-2  # max|err| / max|ref| for bf16 inputs with fp32 state and accumulation


@pytest.fixture(scope="module")
def cwl():
    from chunked_weight_layers_b200 import build
    build.build()
    import chunked_weight_layers_b200 as cwl
    return cwl


def make_state(cwl, spec, x, token_weights=0):
    cfg = cwl.config(spec.model, batch=spec.B, heads=spec.H, eta=spec.eta, ln_eps=spec.eps,
                     token_weights=int(token_weights))
    st = cwl.FastWeightState(cfg, x["W0"])
    st.set_layernorm(x["gamma"], x["beta"])
    return st


def run(cwl, spec, x, with_q=True, loss=True, splits=None, token_weights=False):
    st = make_state(cwl, spec, x, token_weights)
    K, V = x["K"], x["V"]
    Q = x.get("Q") if with_q else None
    O = torch.full_like(K, float("nan")) if Q is not None else None
    L = torch.full(K.shape[:3], float("nan"), device="cuda", dtype=torch.float32) if loss else None
    for a, e in (splits or [(0, spec.T)]):
        # Each call takes contiguous [B, H, e - a, 64] buffers; its outputs are copied into place.
        Op = None if O is None else torch.empty_like(O[:, :, a:e])
        Lp = None if L is None else torch.empty_like(L[:, :, a:e])
        st.chunk_scan(K[:, :, a:e].contiguous(), V[:, :, a:e].contiguous(),
                      None if Q is None else Q[:, :, a:e].contiguous(), out=Op, loss_out=Lp, T=e - a)
        if O is not None:
            O[:, :, a:e] = Op
        if L is not None:
            L[:, :, a:e] = Lp
    W = torch.empty_like(x["W0"])
    st.get_weights(W)
    torch.cuda.synchronize()
    st.poll()
    return O, W, L


def oracle(spec, x, with_q=True, token_weights=False):
    cpu = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    Q = cpu.get("Q") if with_q else None
    if spec.model == "linear_ln":
        O, W, L = ora.ttt_linear_ln_scan(cpu["K"], cpu["V"], Q, cpu["W0"], cpu["gamma"], cpu["beta"], spec.eta,
                                         spec.b, spec.eps, token_weights=token_weights)
        return O, W, L
    O, W1, W2, L = ora.ttt_mlp_scan(cpu["K"], cpu["V"], Q, cpu["W1"], cpu["W2"], cpu["gamma"], cpu["beta"],
                                    spec.eta, spec.b, spec.eps, token_weights=token_weights)
    B, H = spec.B, spec.H
    return O, np.concatenate([W1.reshape(B, H, -1), W2.reshape(B, H, -1)], axis=2), L


def weight_errs(spec, W, Wref):
    """max-relative errors of the weights; TTT-MLP's two layers are compared separately (their
    scales differ by an order of magnitude)."""
    if spec.model == "linear_ln":
        return [rel_err(W, Wref)]
    n1 = spec.D * spec.hidden
    return [rel_err(W[..., :n1], Wref[..., :n1]), rel_err(W[..., n1:], Wref[..., n1:])]


MODELS = ["linear_ln", "mlp"]


def spec_of(model, **changes):
    base = workloads.LINEAR_LN if model == "linear_ln" else workloads.MLP
    return workloads.scaled(base, **changes)


@pytest.mark.parametrize("model", MODELS)
@pytest.mark.parametrize("T", [256, 208, 16])
def test_small_against_oracle(cwl, model, T):
    """Several 64-token tiles, a ragged last tile (T = 208) and a single mini-batch."""
    spec = spec_of(model, B=2, H=3, T=T, seed=2100 + T)
    x = workloads.inner_inputs(spec, device="cuda")
    O, W, L = run(cwl, spec, x)
    Oref, Wref, Lref = oracle(spec, x)
    eo, ew, el = rel_err(O, Oref), max(weight_errs(spec, W, Wref)), rel_err(L, Lref)
    print(f"{model} T={T}: O {eo:.3e}  W {ew:.3e}  loss {el:.3e}")
    assert eo <= TOL and ew <= TOL and el <= TOL


@pytest.mark.parametrize("model", MODELS)
@pytest.mark.parametrize("with_q,loss", [(False, True), (True, False), (False, False)])
def test_without_queries_or_losses(cwl, model, with_q, loss):
    spec = spec_of(model, B=1, H=2, T=192, seed=2200)
    x = workloads.inner_inputs(spec, device="cuda")
    O, W, L = run(cwl, spec, x, with_q=with_q, loss=loss)
    Oref, Wref, Lref = oracle(spec, x, with_q=with_q)
    assert max(weight_errs(spec, W, Wref)) <= TOL
    if with_q:
        assert rel_err(O, Oref) <= TOL
    if loss:
        assert rel_err(L, Lref) <= TOL


@pytest.mark.parametrize("model", MODELS)
def test_streaming_calls_equal_one_call(cwl, model):
    """Successive calls continue one scan: splits at tile and at mini-batch boundaries give the
    same bits as one call."""
    spec = spec_of(model, B=2, H=2, T=320, seed=2300)
    x = workloads.inner_inputs(spec, device="cuda")
    O1, W1, L1 = run(cwl, spec, x)
    O2, W2, L2 = run(cwl, spec, x, splits=[(0, 64), (64, 80), (80, 320)])
    assert torch.equal(O1, O2) and torch.equal(W1, W2) and torch.equal(L1, L2)


@pytest.mark.parametrize("model", MODELS)
def test_zero_gain_leaves_only_the_residual(cwl, model):
    """γ = β = 0: f(x) = x exactly, so O = Q bit for bit and the weights do not move; the loss
    is ‖k − v‖²."""
    spec = spec_of(model, B=1, H=2, T=128, seed=2400)
    x = workloads.inner_inputs(spec, device="cuda")
    x["gamma"] = torch.zeros_like(x["gamma"])
    x["beta"] = torch.zeros_like(x["beta"])
    O, W, L = run(cwl, spec, x)
    assert torch.equal(O, x["Q"])
    assert torch.equal(W, x["W0"])
    ref = ((x["K"].double() - x["V"].double()) ** 2).sum(-1)
    assert rel_err(L, ref) <= 1e-5


@pytest.mark.parametrize("model", MODELS)
def test_heads_and_sequences_are_independent(cwl, model):
    """Changing one (sequence, head)'s inputs changes no other's outputs, weights or losses."""
    spec = spec_of(model, B=2, H=3, T=128, seed=2500)
    x = workloads.inner_inputs(spec, device="cuda")
    O1, W1, L1 = run(cwl, spec, x)
    y = dict(x)
    y["V"] = x["V"].clone()
    y["V"][1, 2] += 0.25
    O2, W2, L2 = run(cwl, spec, y)
    mask = torch.ones(spec.B, spec.H, dtype=torch.bool)
    mask[1, 2] = False
    assert torch.equal(O1[mask], O2[mask]) and torch.equal(W1[mask], W2[mask]) and torch.equal(L1[mask], L2[mask])
    assert not torch.equal(W1[1, 2], W2[1, 2])


def test_rejects_what_is_not_built(cwl):
    from chunked_weight_layers_b200 import TTTError, abi
    W0 = torch.eye(64, device="cuda").expand(1, 1, 64, 64).contiguous()
    for fields, status in ((dict(chunk=32), abi.TTT_ERR_UNSUPPORTED), (dict(gate_enable=1), abi.TTT_ERR_UNSUPPORTED),
                           (dict(io_dtype=0), abi.TTT_ERR_UNSUPPORTED), (dict(ln_eps=0.0), abi.TTT_ERR_INVALID_ARG)):
        with pytest.raises(TTTError) as e:
            cwl.FastWeightState(cwl.config("linear_ln", **fields), W0)
        assert e.value.status == status, fields
    lin = cwl.FastWeightState(cwl.config("linear", batch=1, heads=1), W0)
    g = torch.ones(1, 64, device="cuda")
    with pytest.raises(TTTError) as e:
        lin.set_layernorm(g, g)
    assert e.value.status == abi.TTT_ERR_UNSUPPORTED


@pytest.mark.parametrize("model", MODELS)
def test_workload_full_size(cwl, model):
    """The workload itself (B=8, H=12, T=2048, every head) against the oracle."""
    spec = workloads.LINEAR_LN if model == "linear_ln" else workloads.MLP
    x = workloads.inner_inputs(spec, device="cuda")
    O, W, L = run(cwl, spec, x)
    Oref, Wref, Lref = oracle(spec, x)
    eo, ew, el = rel_err(O, Oref), max(weight_errs(spec, W, Wref)), rel_err(L, Lref)
    print(f"{spec.name}: O {eo:.3e}  W {ew:.3e}  loss {el:.3e}")
    assert eo <= TOL and ew <= TOL and el <= TOL
    assert np.isfinite(to_np(O)).all()


TW_MODELS = ["linear_ln", "mlp"]


@pytest.mark.parametrize("model", TW_MODELS)
@pytest.mark.parametrize("T", [208, 16])
def test_token_weights_small_against_oracle(cwl, model, T):
    """Per-token weights within the mini-batch: outputs against the oracle; losses and the final
    weight equal the default form's bit for bit (only the outputs change)."""
    spec = spec_of(model, B=2, H=3, T=T, seed=2600 + T)
    x = workloads.inner_inputs(spec, device="cuda")
    O, W, L = run(cwl, spec, x, token_weights=True)
    Oref, Wref, Lref = oracle(spec, x, token_weights=True)
    eo = rel_err(O, Oref)
    print(f"{model} T={T} per-token weights: O {eo:.3e}")
    assert eo <= TOL and max(weight_errs(spec, W, Wref)) <= TOL and rel_err(L, Lref) <= TOL
    O0, W0_, L0 = run(cwl, spec, x)
    assert torch.equal(W, W0_) and torch.equal(L, L0)
    assert rel_err(O, to_np(O0)) > 1e-3


@pytest.mark.parametrize("model", TW_MODELS)
def test_token_weights_streaming(cwl, model):
    spec = spec_of(model, B=1, H=2, T=192, seed=2700)
    x = workloads.inner_inputs(spec, device="cuda")
    O1, W1, L1 = run(cwl, spec, x, token_weights=True)
    O2, W2, L2 = run(cwl, spec, x, splits=[(0, 48), (48, 192)], token_weights=True)
    assert torch.equal(O1, O2) and torch.equal(W1, W2) and torch.equal(L1, L2)


@pytest.mark.parametrize("model", TW_MODELS)
def test_token_weights_workload_full_size(cwl, model):
    spec = workloads.LINEAR_LN if model == "linear_ln" else workloads.MLP
    x = workloads.inner_inputs(spec, device="cuda")
    O, W, L = run(cwl, spec, x, token_weights=True)
    Oref, Wref, Lref = oracle(spec, x, token_weights=True)
    eo, ew, el = rel_err(O, Oref), max(weight_errs(spec, W, Wref)), rel_err(L, Lref)
    print(f"{spec.name} per-token weights: O {eo:.3e}  W {ew:.3e}  loss {el:.3e}")
    assert eo <= TOL and ew <= TOL and el <= TOL


@pytest.mark.parametrize("model", MODELS)
def test_reset_rescan_and_weight_roundtrip(cwl, model):
    """reset() returns every head to W0 (a rescan repeats the first scan bit for bit); get/set of
    the weights resumes a scan exactly at a mini-batch boundary; T = 0 is a no-op."""
    spec = spec_of(model, B=2, H=2, T=192, seed=2800)
    x = workloads.inner_inputs(spec, device="cuda")
    st = make_state(cwl, spec, x)
    K, V, Q = x["K"], x["V"], x["Q"]

    def call(a, e):
        O = torch.empty_like(K[:, :, a:e])
        L = torch.empty(K.shape[0], K.shape[1], e - a, device="cuda")
        st.chunk_scan(K[:, :, a:e].contiguous(), V[:, :, a:e].contiguous(), Q[:, :, a:e].contiguous(), out=O,
                      loss_out=L, T=e - a)
        return O, L

    O1, L1 = call(0, 192)
    W1 = torch.empty_like(x["W0"])
    st.get_weights(W1)
    st.reset()
    O2, L2 = call(0, 192)
    assert torch.equal(O1, O2) and torch.equal(L1, L2)
    st.reset()
    call(0, 96)
    Wmid = torch.empty_like(x["W0"])
    st.get_weights(Wmid)
    st.reset()
    st.set_weights(Wmid)
    O3, L3 = call(96, 192)
    W3 = torch.empty_like(x["W0"])
    st.get_weights(W3)
    torch.cuda.synchronize()
    assert torch.equal(O3, O1[:, :, 96:]) and torch.equal(L3, L1[:, :, 96:]) and torch.equal(W3, W1)
    st.chunk_scan(K, V, Q, out=torch.empty_like(K), T=0)
    W4 = torch.empty_like(x["W0"])
    st.get_weights(W4)
    torch.cuda.synchronize()
    assert torch.equal(W4, W1)


@pytest.mark.parametrize("model", MODELS)
def test_more_heads_than_sms(cwl, model):
    """160 (sequence, head) pairs, one CTA each: more than the 148 SMs hold at once."""
    spec = spec_of(model, B=10, H=16, T=48, seed=2900)
    x = workloads.inner_inputs(spec, device="cuda")
    O, W, L = run(cwl, spec, x)
    Oref, Wref, Lref = oracle(spec, x)
    assert rel_err(O, Oref) <= TOL and max(weight_errs(spec, W, Wref)) <= TOL and rel_err(L, Lref) <= TOL
