"""ttt_target_values_noalloc: target generation for callers that cannot allocate device memory.

Callers whose GPU memory belongs to another allocator, or that must not call cudaMalloc
after start-up, cannot create a state just to get the target V̂ = Conv1D(X0)·Wtarget. This
entry point computes it into their output buffer using only a fixed scratch array built
into the library. Here it is called through the C ABI twice in a row: each result is checked
against the oracle's targets (both padding modes), must not change device memory use after
the first call, must leave its status word at 0, and, fed as the given target of an In-Place
scan, must give the outputs of the scan that builds the same target itself (target_mode 1),
within the tolerance of the bf16 workloads.

This file is named so that pytest collects it last."""

import ctypes

import numpy as np
import pytest
import torch

from gen import workloads
from oracle import inplace as oinp
from tests._util import rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def lib():
    from chunked_weight_layers_b200 import abi, build
    build.build()
    return abi.load()


def _scan(cwl, x, spec, targets, target_mode, pad_mode):
    d, f = x["W0"].shape
    cfg = cwl.config("inplace", io_dtype=1, d_key=f, d_val=d, chunk=spec.C, eta=spec.eta, target_mode=target_mode,
                     conv_pad_mode=pad_mode)
    st = cwl.FastWeightState(cfg, x["W0"], x["Wtarget"] if target_mode else None, x["convw"] if target_mode else None)
    O = torch.empty((spec.T, d), device="cuda", dtype=torch.bfloat16)
    st.chunk_scan(x["Z"], targets, out=O)
    W = torch.empty_like(x["W0"])
    st.get_weights(W)
    torch.cuda.synchronize()
    st.poll()
    st.close()
    return O, W


@pytest.mark.parametrize("pad_mode", [0, 1])
def test_noalloc_target_matches_oracle_and_fused_target_scan(lib, pad_mode):
    import chunked_weight_layers_b200 as cwl
    from chunked_weight_layers_b200 import abi

    spec = workloads.scaled(workloads.INPLACE_128K_TARGET, T=1024, C=256, d=512, f=384, seed=71)
    x = workloads.inplace_inputs(spec, device="cuda")
    V_ref = oinp.target_values(x["X0"].cpu(), x["convw"].cpu(), x["Wtarget"].cpu(), spec.C, pad_mode)
    O_ref, W_ref = _scan(cwl, x, spec, x["X0"], target_mode=1, pad_mode=pad_mode)

    stream = torch.cuda.current_stream().cuda_stream or None
    status = torch.full((1,), -1, device="cuda", dtype=torch.int32)
    outs = [torch.full((spec.T, spec.d), float("nan"), device="cuda", dtype=torch.bfloat16) for _ in range(2)]
    torch.cuda.synchronize()
    for call, V in enumerate(outs):
        free_before = torch.cuda.mem_get_info()[0]
        st = lib.ttt_target_values_noalloc(x["X0"].data_ptr(), x["convw"].data_ptr(), x["Wtarget"].data_ptr(),
                                           spec.T, spec.d, spec.C, 3, pad_mode, V.data_ptr(), status.data_ptr(),
                                           stream)
        assert st == abi.TTT_OK, lib.ttt_last_error_string()
        torch.cuda.synchronize()
        if call > 0:
            # Only the first call on a device may bring the fixed array into device memory.
            assert torch.cuda.mem_get_info()[0] == free_before
        assert int(status.item()) == abi.TTT_OK
        ev = rel_err(V, V_ref)
        print(f"no-alloc target, pad mode {pad_mode}, call {call}: V̂ {ev:.3e}")
        assert ev <= TOL
    assert torch.equal(outs[0], outs[1])
    O, W = _scan(cwl, x, spec, outs[1], target_mode=0, pad_mode=pad_mode)
    eo, ew = rel_err(O, O_ref), rel_err(W, W_ref)
    print(f"no-alloc target, pad mode {pad_mode}, scan: O {eo:.3e}  W {ew:.3e}")
    assert eo <= TOL and ew <= TOL
    assert np.isfinite(O.float().cpu().numpy()).all()


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    from chunked_weight_layers_b200 import abi
    d, T = 4096, 2048  # T·d = 8M elements, twice the fixed scratch
    X0 = torch.zeros((T, d), device="cuda", dtype=torch.bfloat16)
    w = torch.zeros((d, 3), device="cuda")
    Wt = torch.zeros((d, d), device="cuda", dtype=torch.bfloat16)
    V = torch.zeros_like(X0)
    st = lib.ttt_target_values_noalloc(X0.data_ptr(), w.data_ptr(), Wt.data_ptr(), T, d, 256, 3, 0, V.data_ptr(),
                                       None, None)
    assert st == abi.TTT_ERR_INVALID_ARG
    assert b"exceeds the fixed scratch" in lib.ttt_last_error_string()
    assert ctypes.c_int(st).value != abi.TTT_OK
