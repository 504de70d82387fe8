"""GPU parity of packed sequences (ttt_chunk_scan_docs): per-document resets to the pretrained
weight and update-norm clipping ("In-Place Test-Time Training", §6 and its implementation
notes), against the oracle's packed scan."""

import numpy as np
import pytest
import torch

from gen import workloads
from oracle import packed as opk
from tests._util import bf16_round, rel_err, to_np

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def cwl():
    from chunked_weight_layers_b200 import build
    build.build()
    import chunked_weight_layers_b200 as cwl
    return cwl


def new_state(cwl, W0, C, eta):
    d, f = W0.shape
    return cwl.FastWeightState(cwl.config("inplace", io_dtype=1, d_key=f, d_val=d, chunk=C, eta=eta), W0)


def run_docs(cwl, x, C, eta, doc_starts, clip=None):
    st = new_state(cwl, x["W0"], C, eta)
    T, d = x["Z"].shape[0], x["W0"].shape[0]
    O = torch.full((T, d), float("nan"), device="cuda", dtype=torch.bfloat16)
    st.chunk_scan_docs(x["Z"], x["Vhat"], doc_starts, clip=clip, out=O)
    W = torch.empty_like(x["W0"])
    st.get_weights(W)
    torch.cuda.synchronize()
    st.poll()
    return O, W


def test_single_document_equals_context_parallel_form(cwl):
    """One document of whole chunks and no clipping is the context-parallel scan, bit for bit."""
    spec = workloads.scaled(workloads.INPLACE_4B, T=512, C=128, d=256, f=384, seed=71)
    x = workloads.inplace_inputs(spec, device="cuda")
    O1, W1 = run_docs(cwl, x, spec.C, spec.eta, [0])
    st = new_state(cwl, x["W0"], spec.C, spec.eta)
    st.set_option(cwl.abi.TTT_OPT_INPLACE_PREFIX, 1)
    O2 = torch.empty_like(O1)
    st.chunk_scan(x["Z"], x["Vhat"], out=O2)
    W2 = torch.empty_like(W1)
    st.get_weights(W2)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(W1, W2)


@pytest.mark.parametrize("T,starts", [(700, [0, 200, 330, 512]), (384, [0, 1, 129]), (300, [0])])
def test_exact_integers_ragged_documents(cwl, T, starts):
    """Sparse {-1,0,1} inputs, W0 in steps of 1/64, η = 2^-6, documents of ragged lengths (a
    one-token document, a document that ends mid-chunk, T not a multiple of the chunk): every
    delta and sum is exact, so O equals bf16(oracle) and the last document's weight equals the
    oracle's bit for bit."""
    g = torch.Generator().manual_seed(29 + T)
    C, d, f = 128, 136, 200

    def sparse(shape, p):
        v = torch.randint(-1, 2, shape, generator=g).float()
        return v * (torch.rand(shape, generator=g) < p)

    Z, V = sparse((T, f), 0.15), sparse((T, d), 0.15)
    W0 = torch.randint(-32, 33, (d, f), generator=g).float() / 64
    O_ref, W_ref = opk.inplace_scan_docs(Z, V, W0, 2.0 ** -6, C, starts)
    x = {"Z": Z.to(torch.bfloat16).cuda(), "Vhat": V.to(torch.bfloat16).cuda(), "W0": W0.cuda()}
    O, W = run_docs(cwl, x, C, 2.0 ** -6, starts)
    assert np.array_equal(to_np(O), bf16_round(O_ref))
    assert np.array_equal(to_np(W), W_ref)


def test_clipping_random_documents(cwl):
    """Random inputs, three documents, the clip threshold halfway between the smallest and the
    largest chunk delta's norm (the full chunks are clipped, the short last chunks of the
    documents are not): against the oracle, and different from the unclipped scan."""
    spec = workloads.scaled(workloads.INPLACE_4B, T=1000, C=128, d=256, f=384, seed=83)
    x = workloads.inplace_inputs(spec, device="cuda")
    starts = [0, 300, 650]
    Zc, Vc, W0c = x["Z"].cpu(), x["Vhat"].cpu(), x["W0"].cpu()
    Zd, Vd = Zc.double().numpy(), Vc.double().numpy()
    norms = []
    for a, e in zip(starts, starts[1:] + [spec.T]):
        for c0 in range(a, e, spec.C):
            r = slice(c0, min(c0 + spec.C, e))
            norms.append(np.linalg.norm(spec.eta * (Vd[r].T @ Zd[r])))
    clip = 0.5 * (min(norms) + max(norms))
    assert min(norms) < 0.95 * clip and max(norms) > 1.05 * clip
    O_ref, W_ref = opk.inplace_scan_docs(Zc, Vc, W0c, spec.eta, spec.C, starts, clip)
    O, W = run_docs(cwl, x, spec.C, spec.eta, starts, clip)
    eo, ew = rel_err(O, O_ref), rel_err(W, W_ref)
    print(f"packed + clip: O {eo:.3e}  W {ew:.3e}")
    assert eo <= TOL and ew <= TOL
    O_nc, W_nc = run_docs(cwl, x, spec.C, spec.eta, starts)
    assert rel_err(W_nc, W_ref) > 10 * ew


def test_rejects_bad_arguments(cwl):
    from chunked_weight_layers_b200 import TTTError, abi
    spec = workloads.scaled(workloads.INPLACE_4B, T=256, C=128, d=256, f=256, seed=3)
    x = workloads.inplace_inputs(spec, device="cuda")
    st = new_state(cwl, x["W0"], spec.C, spec.eta)
    O = torch.empty((spec.T, spec.d), device="cuda", dtype=torch.bfloat16)
    for starts, clip in (([1], None), ([0, 100, 100], None), ([0, 256], None), ([0], -1.0)):
        with pytest.raises(TTTError) as e:
            st.chunk_scan_docs(x["Z"], x["Vhat"], starts, clip=clip, out=O)
        assert e.value.status == abi.TTT_ERR_INVALID_ARG, (starts, clip)
    W0 = torch.eye(64, device="cuda").expand(1, 1, 64, 64).contiguous()
    lin = cwl.FastWeightState(cwl.config("linear", batch=1, heads=1, chunk=16), W0)
    with pytest.raises(TTTError) as e:
        lin.chunk_scan_docs(x["Z"], x["Vhat"], [0], out=O)
    assert e.value.status == abi.TTT_ERR_UNSUPPORTED


def _target_state(cwl, x, C, eta, pad_mode):
    d, f = x["W0"].shape
    cfg = cwl.config("inplace", io_dtype=1, d_key=f, d_val=d, chunk=C, eta=eta, target_mode=1,
                     conv_pad_mode=pad_mode)
    return cwl.FastWeightState(cfg, x["W0"], x["Wtarget"], x["convw"])


def _run(st, Z, targets, doc_starts, clip=None):
    O = torch.full((Z.shape[0], st.cfg.d_val), float("nan"), device="cuda", dtype=torch.bfloat16)
    st.chunk_scan_docs(Z, targets, doc_starts, clip=clip, out=O)
    W = torch.empty((st.cfg.d_val, st.cfg.d_key), device="cuda")
    st.get_weights(W)
    torch.cuda.synchronize()
    st.poll()
    return O, W


@pytest.mark.parametrize("pad_mode", [0, 1])
@pytest.mark.parametrize("clip", [None, 0.04])
def test_fused_target_documents_against_oracle(cwl, pad_mode, clip):
    """The target made inside the scan from X0, per document: documents of 256 tokens (whole
    chunks: in pad mode 1 its last taps would reach the next document without the extra
    padding), 44, 211 and 189 tokens, with and without clipping, against the oracle."""
    spec = workloads.scaled(workloads.INPLACE_128K_TARGET, T=700, C=128, d=256, f=384, seed=91 + pad_mode)
    x = workloads.inplace_inputs(spec, device="cuda")
    starts = [0, 256, 300, 511]
    c = {k: x[k].cpu() for k in ("Z", "X0", "convw", "Wtarget", "W0")}
    O_ref, W_ref = opk.inplace_scan_docs_target(c["Z"], c["X0"], c["convw"], c["Wtarget"], c["W0"], spec.eta, spec.C,
                                                starts, pad_mode, clip)
    O, W = _run(_target_state(cwl, x, spec.C, spec.eta, pad_mode), x["Z"], x["X0"], starts, clip)
    eo, ew = rel_err(O, O_ref), rel_err(W, W_ref)
    print(f"packed fused target pad {pad_mode} clip {clip}: O {eo:.3e}  W {ew:.3e}")
    assert eo <= TOL and ew <= TOL


@pytest.mark.parametrize("pad_mode", [0, 1])
def test_fused_target_one_document_equals_given_targets(cwl, pad_mode):
    """One document of whole chunks: the targets made inside the call are those of
    ttt_target_values_noalloc (the same kernels) and the scan then equals the packed scan with
    those targets given, bit for bit."""
    from chunked_weight_layers_b200 import abi
    spec = workloads.scaled(workloads.INPLACE_128K_TARGET, T=512, C=128, d=256, f=384, seed=95)
    x = workloads.inplace_inputs(spec, device="cuda")
    V = torch.empty((spec.T, spec.d), device="cuda", dtype=torch.bfloat16)
    lib = abi.load()
    r = lib.ttt_target_values_noalloc(x["X0"].data_ptr(), x["convw"].data_ptr(), x["Wtarget"].data_ptr(), spec.T,
                                      spec.d, spec.C, 3, pad_mode, V.data_ptr(), None,
                                      torch.cuda.current_stream().cuda_stream or None)
    assert r == abi.TTT_OK
    O1, W1 = _run(_target_state(cwl, x, spec.C, spec.eta, pad_mode), x["Z"], x["X0"], [0])
    O2, W2 = _run(new_state(cwl, x["W0"], spec.C, spec.eta), x["Z"], V, [0])
    assert torch.equal(O1, O2) and torch.equal(W1, W2)


ROWS = [0, 1, 127, 128, 1000, 2047, 2048, 2559]


@pytest.mark.slow
def test_inplace_4b_shapes_packed_sampled(cwl):
    """The 4B-class widths (d=2560, f=9728) over T=8192 packed as five documents of ragged
    lengths: sampled Wdown rows against the oracle (without clipping rows evolve independently,
    so the oracle needs only the sampled rows)."""
    spec = workloads.scaled(workloads.INPLACE_4B, T=8192)
    x = workloads.inplace_inputs(spec, device="cuda")
    starts = [0, 1500, 3100, 5000, 7777]
    O, W = run_docs(cwl, x, spec.C, spec.eta, starts)
    Z = x["Z"].cpu()
    Oref, Wref = opk.inplace_scan_docs(Z, x["Vhat"][:, ROWS].cpu(), x["W0"][ROWS].cpu(), spec.eta, spec.C, starts)
    eo, ew = rel_err(O[:, ROWS], Oref), rel_err(W[ROWS], Wref)
    print(f"4B-class widths, packed: O {eo:.3e}  W {ew:.3e}")
    assert eo <= TOL and ew <= TOL
