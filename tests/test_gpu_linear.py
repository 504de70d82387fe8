"""GPU parity of the TTT-Linear mini-batch scan against the oracle."""

import numpy as np
import pytest
import torch

from gen import workloads
from oracle import linear as ora
from tests._util import rel_err

pytestmark = pytest.mark.gpu

TOL = 2e-2  # max|err| / max|ref| for bf16 inputs with fp32 accumulation


@pytest.fixture(scope="module")
def cwl():
    from chunked_weight_layers_b200 import build
    build.build()
    import chunked_weight_layers_b200 as cwl
    return cwl


# Inner mini-batches per chunk of the b = 16 scan (TTT_OPT_LINEAR_CHUNK): the step-by-step
# form and the two chunked forms.
FORMS = [1, 2, 4]


def new_state(cwl, cfg, W0, form=None):
    st = cwl.FastWeightState(cfg, W0)
    if form is not None:
        st.set_option(cwl.abi.TTT_OPT_LINEAR_CHUNK, form)
    return st


def run_linear(cwl, x, b, eta, with_q=True, loss=True, form=None):
    K, V = x["K"], x["V"]
    B, H, T, D = K.shape
    cfg = cwl.config("linear", batch=B, heads=H, d_key=D, d_val=D, chunk=b, eta=eta)
    st = new_state(cwl, cfg, x["W0"], form)
    Q = x.get("Q") if with_q else None
    O = torch.empty_like(K) if Q is not None else None
    L = torch.empty((B, H, T), device="cuda", dtype=torch.float32) if loss else None
    st.chunk_scan(K, V, Q, out=O, loss_out=L)
    W = torch.empty_like(x["W0"])
    st.get_weights(W)
    torch.cuda.synchronize()
    st.poll()
    return O, W, L, st


@pytest.fixture(scope="module")
def workload_ref():
    spec = workloads.LINEAR_GD
    x = workloads.linear_inputs(spec, device="cpu")
    return ora.ttt_linear_scan(x["K"], x["V"], x["Q"], x["W0"], spec.eta, spec.b)


@pytest.mark.parametrize("form", FORMS)
def test_linear_workload_full_size(cwl, workload_ref, form):
    spec = workloads.LINEAR_GD
    x = workloads.linear_inputs(spec, device="cuda")
    O, W, L, st = run_linear(cwl, x, spec.b, spec.eta, form=form)
    Oref, Wref, Lref = workload_ref
    eo, ew, el = rel_err(O, Oref), rel_err(W, Wref), rel_err(L, Lref)
    print(f"TTT-Linear workload, {form} mini-batch(es) per chunk: O {eo:.3e}  W {ew:.3e}  loss {el:.3e}")
    assert eo <= TOL and ew <= TOL and el <= TOL
    # Well inside the tolerance (bf16 operands, fp32 state and accumulation); a regression in
    # the operand handling would show up here first.
    assert max(eo, ew, el) <= 5e-3
    assert st.launch_count() >= 1


@pytest.mark.parametrize("form", FORMS)
def test_identity_fixed_point_is_exact(cwl, form):
    """W0 = I and V = K: every residual is exactly 0, W stays I, O = Q, losses 0."""
    spec = workloads.scaled(workloads.LINEAR_GD, B=2, H=3, T=320)
    x = workloads.linear_inputs(spec, device="cuda")
    x["V"] = x["K"].clone()
    O, W, L, _ = run_linear(cwl, x, 16, 1.0, form=form)
    assert torch.equal(W, x["W0"])
    assert torch.equal(O, x["Q"])
    assert torch.count_nonzero(L).item() == 0


@pytest.mark.parametrize("b,T,B,H,form", [(16, 208, 2, 3, 1), (16, 208, 2, 3, 2), (16, 208, 2, 3, 4),
                                          (16, 240, 2, 3, 2), (16, 240, 2, 3, 4), (16, 224, 2, 3, 4),
                                          (32, 224, 2, 3, None), (64, 192, 2, 3, None),
                                          (16, 64, 2, 3, 1), (16, 64, 2, 3, 2), (16, 64, 2, 3, 4),
                                          (16, 208, 1, 80, 1), (16, 208, 1, 80, 2), (16, 208, 1, 80, 4)])
def test_small_shapes_and_ragged_tiles(cwl, b, T, B, H, form):
    """Ragged last tiles (T = 208, 224, 240 leave 1, 2, 3 mini-batches of 16 after the full
    64-token tiles), each inner mini-batch size and each chunked form, and more heads than fit
    one wave at a time."""
    spec = workloads.scaled(workloads.LINEAR_GD, B=B, H=H, T=T, b=b, seed=77 + b + H)
    x = workloads.linear_inputs(spec, device="cuda")
    W0 = x["W0"].clone()
    W0 += 0.05 * torch.randn(W0.shape, generator=torch.Generator().manual_seed(b)).cuda()
    x["W0"] = W0
    O, W, L, _ = run_linear(cwl, x, b, 0.5, form=form)
    Oref, Wref, Lref = ora.ttt_linear_scan(x["K"].cpu(), x["V"].cpu(), x["Q"].cpu(), W0.cpu(), 0.5, b)
    errs = rel_err(O, Oref), rel_err(W, Wref), rel_err(L, Lref)
    # O is stored in bf16 (rounding up to 2^-9 of an element) and computed from W rounded to
    # bf16; W and the losses stay far tighter.
    assert errs[0] <= 1e-2 and max(errs[1:]) <= 5e-3, errs


@pytest.mark.parametrize("form", FORMS)
def test_without_queries_same_state_and_loss(cwl, form):
    spec = workloads.scaled(workloads.LINEAR_GD, B=1, H=4, T=256)
    x = workloads.linear_inputs(spec, device="cuda")
    _, W1, L1, _ = run_linear(cwl, x, 16, 1.0, form=form)
    _, W2, L2, _ = run_linear(cwl, x, 16, 1.0, with_q=False, form=form)
    assert torch.equal(W1, W2) and torch.equal(L1, L2)


@pytest.mark.parametrize("form,split", [(1, 112), (2, 96), (4, 128)])
def test_streaming_split_equals_one_call(cwl, form, split):
    """Two calls split at a multiple of the chunk (16·form tokens) reproduce one call bit for
    bit."""
    spec = workloads.scaled(workloads.LINEAR_GD, B=2, H=2, T=320)
    x = workloads.linear_inputs(spec, device="cuda")
    O1, W1, L1, _ = run_linear(cwl, x, 16, 1.0, form=form)
    B, H, T, D = x["K"].shape
    cfg = cwl.config("linear", batch=B, heads=H, chunk=16, eta=1.0)
    st = new_state(cwl, cfg, x["W0"], form)
    outs, losses = [], []
    for a, z in ((0, split), (split, T)):
        K, V, Q = (x[n][:, :, a:z].contiguous() for n in ("K", "V", "Q"))
        O = torch.empty_like(K)
        L = torch.empty((B, H, z - a), device="cuda")
        st.chunk_scan(K, V, Q, out=O, loss_out=L)
        outs.append(O)
        losses.append(L)
    W = torch.empty_like(x["W0"])
    st.get_weights(W)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(outs, 2), O1) and torch.equal(torch.cat(losses, 2), L1)
    assert torch.equal(W, W1)


def test_rejects_bad_arguments(cwl):
    from chunked_weight_layers_b200 import TTTError, abi
    W0 = torch.eye(64, device="cuda").expand(1, 2, 64, 64).contiguous()
    st = cwl.FastWeightState(cwl.config("linear", batch=1, heads=2, chunk=16), W0)
    K = torch.zeros(1, 2, 40, 64, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(TTTError) as e:
        st.chunk_scan(K, K, K, out=torch.empty_like(K))  # 40 is not a multiple of 16
    assert e.value.status == abi.TTT_ERR_INVALID_ARG
    with pytest.raises(TTTError) as e:
        st.chunk_scan(K[:, :, :32].contiguous(), K[:, :, :32].contiguous(), K[:, :, :32].contiguous(), out=None)
    assert e.value.status == abi.TTT_ERR_INVALID_ARG
    with pytest.raises(TTTError) as e:
        cwl.FastWeightState(cwl.config("linear", batch=1, heads=2, chunk=24), W0)
    assert e.value.status == abi.TTT_ERR_UNSUPPORTED


@pytest.mark.parametrize("form,splits", [(1, (48, 176)), (2, (32, 160)), (4, (64, 192))])
def test_streaming_split_inside_tiles(cwl, form, splits):
    """Calls split inside 64-token tiles (so each call has a ragged last tile and the next starts
    a fresh tile mid-sequence) at multiples of the chunk (16·form tokens) reproduce one call bit
    for bit: every chunk runs the same arithmetic wherever the tile boundaries fall."""
    spec = workloads.scaled(workloads.LINEAR_GD, B=1, H=80, T=256, seed=123)
    x = workloads.linear_inputs(spec, device="cuda")
    O1, W1, L1, _ = run_linear(cwl, x, 16, 1.0, form=form)
    B, H, T, D = x["K"].shape
    st = new_state(cwl, cwl.config("linear", batch=B, heads=H, chunk=16, eta=1.0), x["W0"], form)
    outs, losses = [], []
    a_, b_ = splits
    for a, z in ((0, a_), (a_, b_), (b_, T)):
        K, V, Q = (x[n][:, :, a:z].contiguous() for n in ("K", "V", "Q"))
        O = torch.empty_like(K)
        L = torch.empty((B, H, z - a), device="cuda")
        st.chunk_scan(K, V, Q, out=O, loss_out=L)
        outs.append(O)
        losses.append(L)
    W = torch.empty_like(x["W0"])
    st.get_weights(W)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(outs, 2), O1) and torch.equal(torch.cat(losses, 2), L1)
    assert torch.equal(W, W1)
    Oref, Wref, Lref = ora.ttt_linear_scan(x["K"].cpu(), x["V"].cpu(), x["Q"].cpu(), x["W0"].cpu(), 1.0, 16)
    assert rel_err(O1, Oref) <= 1e-2 and rel_err(W1, Wref) <= 5e-3 and rel_err(L1, Lref) <= 5e-3


@pytest.mark.parametrize("form", [2, 4])
def test_streaming_split_off_chunk_is_within_tolerance(cwl, form):
    """Splits that cut a chunk of the chunked form (48 and 176 tokens) regroup its steps, so
    the calls are no longer bit-identical to one call, but they still follow the rule: outputs,
    losses and final weights against the oracle."""
    spec = workloads.scaled(workloads.LINEAR_GD, B=1, H=8, T=256, seed=321)
    x = workloads.linear_inputs(spec, device="cuda")
    B, H, T, D = x["K"].shape
    st = new_state(cwl, cwl.config("linear", batch=B, heads=H, chunk=16, eta=1.0), x["W0"], form)
    outs, losses = [], []
    for a, z in ((0, 48), (48, 176), (176, T)):
        K, V, Q = (x[n][:, :, a:z].contiguous() for n in ("K", "V", "Q"))
        O = torch.empty_like(K)
        L = torch.empty((B, H, z - a), device="cuda")
        st.chunk_scan(K, V, Q, out=O, loss_out=L)
        outs.append(O)
        losses.append(L)
    W = torch.empty_like(x["W0"])
    st.get_weights(W)
    torch.cuda.synchronize()
    Oref, Wref, Lref = ora.ttt_linear_scan(x["K"].cpu(), x["V"].cpu(), x["Q"].cpu(), x["W0"].cpu(), 1.0, 16)
    assert rel_err(torch.cat(outs, 2), Oref) <= 1e-2 and rel_err(W, Wref) <= 5e-3
    assert rel_err(torch.cat(losses, 2), Lref) <= 5e-3


def test_option_values(cwl):
    from chunked_weight_layers_b200 import TTTError, abi
    W0 = torch.eye(64, device="cuda").expand(1, 2, 64, 64).contiguous()
    st = cwl.FastWeightState(cwl.config("linear", batch=1, heads=2, chunk=16), W0)
    for v in (0, 1, 2, 4):
        st.set_option(abi.TTT_OPT_LINEAR_CHUNK, v)
    for v in (-1, 3, 8):
        with pytest.raises(TTTError) as e:
            st.set_option(abi.TTT_OPT_LINEAR_CHUNK, v)
        assert e.value.status == abi.TTT_ERR_INVALID_ARG
    with pytest.raises(TTTError) as e:
        st.set_option(12345, 1)
    assert e.value.status == abi.TTT_ERR_INVALID_ARG


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("T,B,H", [(16, 1, 3), (48, 2, 2), (112, 1, 1), (1024, 2, 160)])
def test_edge_lengths_and_more_heads_than_sms(cwl, T, B, H, form):
    """One 16-token step, a single ragged tile (48 tokens), a full tile plus a ragged one
    (112), and 320 heads (more CTAs than SMs: they run in waves): each against the oracle,
    with and without queries, and the loss."""
    spec = workloads.scaled(workloads.LINEAR_GD, B=B, H=H, T=T, seed=500 + T + H)
    x = workloads.linear_inputs(spec, device="cuda")
    O, W, L, _ = run_linear(cwl, x, 16, 1.0, form=form)
    Oref, Wref, Lref = ora.ttt_linear_scan(x["K"].cpu(), x["V"].cpu(), x["Q"].cpu(), x["W0"].cpu(), 1.0, 16)
    errs = rel_err(O, Oref), rel_err(W, Wref), rel_err(L, Lref)
    assert errs[0] <= 1e-2 and max(errs[1:]) <= 5e-3, errs
    _, W2, L2, _ = run_linear(cwl, x, 16, 1.0, with_q=False, form=form)
    assert torch.equal(W2, W) and torch.equal(L2, L)
