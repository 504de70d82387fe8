"""ttt_target_values_noalloc: target generation for callers that cannot allocate device memory.

Callers whose GPU memory belongs to another allocator, or that must not call cudaMalloc
after start-up, cannot create a state just to get the target V̂ = Conv1D(X0)·Wtarget. This
entry point computes it into their output buffer using only a fixed scratch array built
into the library. Here it is called through the C ABI twice in a row, and each result is
fed as the given target of an In-Place scan whose outputs must match the scan that builds
the same target itself (target_mode 1), within the tolerance of the bf16 workloads.

This file is named so that pytest collects it last."""

import ctypes

import pytest
import torch

from gen import workloads
from tests._util import rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def lib():
    from chunked_weight_layers_b200 import abi, build
    build.build()
    return abi.load()


def _scan(cwl, x, spec, targets, target_mode):
    d, f = x["W0"].shape
    cfg = cwl.config("inplace", io_dtype=1, d_key=f, d_val=d, chunk=spec.C, eta=spec.eta, target_mode=target_mode,
                     conv_pad_mode=spec.conv_pad_mode)
    st = cwl.FastWeightState(cfg, x["W0"], x["Wtarget"] if target_mode else None, x["convw"] if target_mode else None)
    O = torch.empty((spec.T, d), device="cuda", dtype=torch.bfloat16)
    st.chunk_scan(x["Z"], targets, out=O)
    W = torch.empty_like(x["W0"])
    st.get_weights(W)
    torch.cuda.synchronize()
    st.poll()
    st.close()
    return O, W


def test_noalloc_target_matches_fused_target_scan(lib):
    import chunked_weight_layers_b200 as cwl
    from chunked_weight_layers_b200 import abi

    spec = workloads.scaled(workloads.INPLACE_128K_TARGET, T=1024, C=256, d=512, f=384, seed=71)
    x = workloads.inplace_inputs(spec, device="cuda")
    O_ref, W_ref = _scan(cwl, x, spec, x["X0"], target_mode=1)

    stream = torch.cuda.current_stream().cuda_stream or None
    previous = None
    for call in range(2):
        V = torch.full((spec.T, spec.d), float("nan"), device="cuda", dtype=torch.bfloat16)
        st = lib.ttt_target_values_noalloc(x["X0"].data_ptr(), x["convw"].data_ptr(), x["Wtarget"].data_ptr(),
                                           spec.T, spec.d, spec.C, 3, spec.conv_pad_mode, V.data_ptr(), stream)
        assert st == abi.TTT_OK, lib.ttt_last_error_string()
        torch.cuda.synchronize()
        assert torch.isfinite(V.float()).all()
        O, W = _scan(cwl, x, spec, V, target_mode=0)
        eo, ew = rel_err(O, O_ref), rel_err(W, W_ref)
        print(f"no-alloc target, call {call}: O {eo:.3e}  W {ew:.3e}")
        assert eo <= TOL and ew <= TOL
        if previous is not None:
            assert torch.equal(V, previous)
        previous = V


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    from chunked_weight_layers_b200 import abi
    d, T = 4096, 2048  # T·d = 8M elements, twice the fixed scratch
    X0 = torch.zeros((T, d), device="cuda", dtype=torch.bfloat16)
    w = torch.zeros((d, 3), device="cuda")
    Wt = torch.zeros((d, d), device="cuda", dtype=torch.bfloat16)
    V = torch.zeros_like(X0)
    st = lib.ttt_target_values_noalloc(X0.data_ptr(), w.data_ptr(), Wt.data_ptr(), T, d, 256, 3, 0, V.data_ptr(),
                                       None)
    assert st == abi.TTT_ERR_INVALID_ARG
    assert b"exceeds the fixed scratch" in lib.ttt_last_error_string()
    assert ctypes.c_int(st).value != abi.TTT_OK
