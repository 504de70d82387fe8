"""GPU parity of the In-Place scan, fp32 path (SIMT FFMA kernels) against the oracle."""

import numpy as np
import pytest
import torch

from gen import workloads
from oracle import inplace as ora
from tests._util import rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cwl():
    from chunked_weight_layers_b200 import build
    build.build()
    import chunked_weight_layers_b200 as cwl
    return cwl


def _state(cwl, W0, C, eta):
    d, f = W0.shape
    cfg = cwl.config("inplace", io_dtype=0, d_key=f, d_val=d, chunk=C, eta=eta)
    return cwl.FastWeightState(cfg, W0)


def _scan(cwl, Z, V, W0, C, eta):
    st = _state(cwl, W0, C, eta)
    O = torch.empty((Z.shape[0], W0.shape[0]), device="cuda", dtype=torch.float32)
    st.chunk_scan(Z, V, out=O)
    W = torch.empty_like(W0)
    st.get_weights(W)
    torch.cuda.synchronize()
    st.poll()
    return O, W, st


def test_exact_integers_bit_exact(cwl):
    """Small integers with η = 2^-4 keep every product and sum exact in fp32 and float64."""
    g = torch.Generator().manual_seed(5)
    T, C, d, f = 96, 32, 70, 100
    Z = torch.randint(-2, 3, (T, f), generator=g).float()
    V = torch.randint(-2, 3, (T, d), generator=g).float()
    W0 = torch.randint(-4, 5, (d, f), generator=g).float()
    O, W, _ = _scan(cwl, Z.cuda(), V.cuda(), W0.cuda(), C, 0.0625)
    Oref, Wref = ora.inplace_scan(Z, V, W0, 0.0625, C)
    assert np.array_equal(to_np(O), Oref)
    assert np.array_equal(to_np(W), Wref)


def test_fp32_workload_full_size(cwl):
    spec = workloads.INPLACE_FP32
    x = workloads.inplace_inputs(spec, device="cuda")
    O, W, st = _scan(cwl, x["Z"], x["Vhat"], x["W0"], spec.C, spec.eta)
    Oref, Wref = ora.inplace_scan(x["Z"].cpu(), x["Vhat"].cpu(), x["W0"].cpu(), spec.eta, spec.C)
    eo, ew = rel_err(O, Oref), rel_err(W, Wref)
    print(f"fp32 workload: O rel err {eo:.3e}, W rel err {ew:.3e}")
    assert eo <= 1e-4 and ew <= 1e-4
    assert st.launch_count() >= spec.T // spec.C  # one launch per chunk


def test_ragged_shapes(cwl):
    g = torch.Generator().manual_seed(6)
    T, C, d, f = 144, 48, 33, 45
    Z, V = torch.randn(T, f, generator=g), torch.randn(T, d, generator=g)
    W0 = 0.1 * torch.randn(d, f, generator=g)
    O, W, _ = _scan(cwl, Z.cuda(), V.cuda(), W0.cuda(), C, 0.05)
    Oref, Wref = ora.inplace_scan(Z, V, W0, 0.05, C)
    assert rel_err(O, Oref) <= 1e-5 and rel_err(W, Wref) <= 1e-5


def test_causality_streaming_and_reset(cwl):
    spec = workloads.scaled(workloads.INPLACE_FP32, T=512, C=128, d=96, f=160)
    x = workloads.inplace_inputs(spec, device="cuda")
    O1, W1, st = _scan(cwl, x["Z"], x["Vhat"], x["W0"], spec.C, spec.eta)
    # Perturb chunk 2: outputs of chunks 0 and 1 are unchanged bit for bit.
    Z2, V2 = x["Z"].clone(), x["Vhat"].clone()
    Z2[256:] += 1.0
    V2[256:] *= -1.0
    O2, _, _ = _scan(cwl, Z2, V2, x["W0"], spec.C, spec.eta)
    assert torch.equal(O1[:256], O2[:256]) and not torch.equal(O1[256:], O2[256:])
    # Two calls split at a chunk boundary equal one call.
    st.reset()
    O3 = torch.empty_like(O1)
    st.chunk_scan(x["Z"][:128], x["Vhat"][:128], out=O3[:128])
    st.chunk_scan(x["Z"][128:], x["Vhat"][128:], out=O3[128:])
    W3 = torch.empty_like(W1)
    st.get_weights(W3)
    torch.cuda.synchronize()
    assert torch.equal(O3, O1) and torch.equal(W3, W1)
    # Reset, then the same scan again, is bit-identical.
    st.reset()
    O4 = torch.empty_like(O1)
    st.chunk_scan(x["Z"], x["Vhat"], out=O4)
    torch.cuda.synchronize()
    assert torch.equal(O4, O1)


def test_invalid_arguments(cwl):
    from chunked_weight_layers_b200 import TTTError, abi
    W0 = torch.zeros(8, 16, device="cuda")
    st = _state(cwl, W0, 4, 0.1)
    Z, V, O = torch.zeros(6, 16, device="cuda"), torch.zeros(6, 8, device="cuda"), torch.zeros(6, 8, device="cuda")
    with pytest.raises(TTTError) as e:
        st.chunk_scan(Z, V, out=O)  # T = 6 is not a multiple of the chunk 4
    assert e.value.status == abi.TTT_ERR_INVALID_ARG
    with pytest.raises(TTTError) as e:
        st.chunk_scan(Z[:4], V[:4], out=None)
    assert e.value.status == abi.TTT_ERR_INVALID_ARG
    with pytest.raises(TTTError) as e:
        cwl.FastWeightState(cwl.config("inplace", io_dtype=0, d_key=16, d_val=8, chunk=4, batch=2), W0)
    assert e.value.status == abi.TTT_ERR_UNSUPPORTED
    # Misaligned pointer.
    raw = torch.zeros(6 * 16 + 1, device="cuda")
    with pytest.raises(TTTError) as e:
        st.chunk_scan(raw[1:65].view(4, 16), V[:4], out=O[:4])
    assert e.value.status == abi.TTT_ERR_INVALID_ARG


def test_injected_allocation_failure(cwl, monkeypatch):
    from chunked_weight_layers_b200 import TTTError, abi
    monkeypatch.setenv("TTT_INJECT_OOM", "1")
    with pytest.raises(TTTError) as e:
        _state(cwl, torch.zeros(8, 16, device="cuda"), 4, 0.1)
    assert e.value.status == abi.TTT_ERR_OOM
