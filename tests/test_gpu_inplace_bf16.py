"""GPU parity of the In-Place scan on the tcgen05 tensor-core path (bf16 in, fp32 state)."""

import numpy as np
import pytest
import torch

from gen import workloads
from oracle import inplace as ora
from tests._util import bf16_round, rel_err, to_np

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def cwl():
    from chunked_weight_layers_b200 import build
    build.build()
    import chunked_weight_layers_b200 as cwl
    return cwl


def scan(cwl, x, C, eta, target=False, pad_mode=0, T=None, pair=1, calls=1):
    """pair=1 (the default) runs on SM pairs wherever C and d are multiples of 256; 0 forces
    one CTA per tile."""
    from chunked_weight_layers_b200 import abi
    Z = x["Z"]
    T = Z.shape[0] if T is None else T
    d, f = x["W0"].shape
    cfg = cwl.config("inplace", io_dtype=1, d_key=f, d_val=d, chunk=C, eta=eta, target_mode=int(target),
                     conv_pad_mode=pad_mode)
    st = cwl.FastWeightState(cfg, x["W0"], x.get("Wtarget") if target else None, x.get("convw") if target else None)
    st.set_option(abi.TTT_OPT_SM_PAIR, pair)
    O = torch.empty((T, d), device="cuda", dtype=torch.bfloat16)
    V = x["X0"] if target else x["Vhat"]
    step = T // calls
    for a in range(0, T, step):
        st.chunk_scan(Z[a:a + step], V[a:a + step], out=O[a:a + step])
    W = torch.empty_like(x["W0"])
    st.get_weights(W)
    torch.cuda.synchronize()
    st.poll()
    return O, W, st


def test_exact_integers_bit_exact(cwl):
    """Sparse {-1,0,1} inputs, W0 in steps of 1/64 and η = 2^-6: every W_c is exact in bf16,
    every product and sum exact in fp32; O must equal bf16(oracle) bit for bit."""
    g = torch.Generator().manual_seed(9)
    T, C, d, f = 384, 128, 136, 200

    def sparse(shape, p):
        v = torch.randint(-1, 2, shape, generator=g).float()
        keep = torch.rand(shape, generator=g) < p
        return v * keep

    Z, V = sparse((T, f), 0.15), sparse((T, d), 0.15)
    W0 = torch.randint(-32, 33, (d, f), generator=g).float() / 64
    O_ref, W_ref = ora.inplace_scan(Z, V, W0, 2.0 ** -6, C)
    # Premise: every intermediate W is a multiple of 1/64 below 4 in magnitude (exact in bf16).
    Wc = W0.double().numpy()
    for c in range(T // C):
        assert np.all(np.abs(Wc) * 64 < 256) and np.all(Wc * 64 == np.round(Wc * 64))
        Wc = Wc + 2.0 ** -6 * (V[c * C:(c + 1) * C].double().numpy().T @ Z[c * C:(c + 1) * C].double().numpy())
    x = {"Z": Z.to(torch.bfloat16).cuda(), "Vhat": V.to(torch.bfloat16).cuda(), "W0": W0.cuda()}
    O, W, _ = scan(cwl, x, C, 2.0 ** -6)
    assert np.array_equal(to_np(O), bf16_round(O_ref))
    assert np.array_equal(to_np(W), W_ref)


def _sparse_case(seed, T, d, f):
    g = torch.Generator().manual_seed(seed)

    def sparse(shape, p):
        v = torch.randint(-1, 2, shape, generator=g).float()
        return v * (torch.rand(shape, generator=g) < p)

    Z, V = sparse((T, f), 0.12), sparse((T, d), 0.12)
    W0 = torch.randint(-32, 33, (d, f), generator=g).float() / 64
    return Z, V, W0


@pytest.mark.parametrize("pair", [1, 0])
def test_exact_integers_bit_exact_256_tiles(cwl, pair):
    """The same exact-integer premise on chunks of 256 tokens and d = 512, the shapes that run
    on SM pairs (tiles of 256 x 256, 128 rows per CTA), with f = 200 ragged against the pair's
    column halves; pair=0 runs the same shapes on single SMs. O and W bit-exact to the oracle."""
    T, C, d, f = 768, 256, 512, 200
    Z, V, W0 = _sparse_case(23, T, d, f)
    O_ref, W_ref = ora.inplace_scan(Z, V, W0, 2.0 ** -6, C)
    Wc = W0.double().numpy()
    for c in range(T // C):
        assert np.all(np.abs(Wc) * 64 < 256) and np.all(Wc * 64 == np.round(Wc * 64))
        Wc = Wc + 2.0 ** -6 * (V[c * C:(c + 1) * C].double().numpy().T @ Z[c * C:(c + 1) * C].double().numpy())
    x = {"Z": Z.to(torch.bfloat16).cuda(), "Vhat": V.to(torch.bfloat16).cuda(), "W0": W0.cuda()}
    O, W, _ = scan(cwl, x, C, 2.0 ** -6, pair=pair)
    assert np.array_equal(to_np(O), bf16_round(O_ref))
    assert np.array_equal(to_np(W), W_ref)


@pytest.mark.parametrize("d,f,calls", [(256, 384, 1), (512, 328, 1), (768, 520, 2)])
def test_sm_pairs_random(cwl, d, f, calls):
    """Random inputs on SM-pair shapes (C = 256, d a multiple of 256): against the oracle, and
    against the single-SM form of the same scan (same sums, tensor-core addition order aside)."""
    spec = workloads.scaled(workloads.INPLACE_4B, T=1024, C=256, d=d, f=f, seed=57 + d)
    x = workloads.inplace_inputs(spec, device="cuda")
    O, W, _ = scan(cwl, x, spec.C, spec.eta, calls=calls)
    O1, W1, _ = scan(cwl, x, spec.C, spec.eta, pair=0)
    Oref, Wref = ora.inplace_scan(x["Z"].cpu(), x["Vhat"].cpu(), x["W0"].cpu(), spec.eta, spec.C)
    eo, ew = rel_err(O, Oref), rel_err(W, Wref)
    print(f"SM pairs d={d} f={f}: O {eo:.3e}  W {ew:.3e}")
    assert eo <= TOL and ew <= TOL
    assert rel_err(O, O1.float()) <= 1e-2 and rel_err(W, W1) <= 1e-5


@pytest.mark.parametrize("pad_mode", [0, 1])
def test_sm_pairs_target(cwl, pad_mode):
    """Fused target generation on SM pairs (TARGET tiles of 256 tokens x 256 columns)."""
    spec = workloads.scaled(workloads.INPLACE_128K_TARGET, T=1024, C=256, d=512, f=384, seed=43,
                            conv_pad_mode=pad_mode)
    x = workloads.inplace_inputs(spec, device="cuda")
    O, W, _ = scan(cwl, x, spec.C, spec.eta, target=True, pad_mode=pad_mode)
    V = ora.target_values(x["X0"].cpu(), x["convw"].cpu(), x["Wtarget"].cpu(), spec.C, pad_mode)
    Oref, Wref = ora.inplace_scan(x["Z"].cpu(), V, x["W0"].cpu(), spec.eta, spec.C)
    eo, ew = rel_err(O, Oref), rel_err(W, Wref)
    print(f"SM pairs + target (pad {pad_mode}): O {eo:.3e}  W {ew:.3e}")
    assert eo <= TOL and ew <= TOL


@pytest.mark.parametrize("d,f", [(256, 256), (200, 328), (392, 520)])
def test_small_random(cwl, d, f):
    spec = workloads.scaled(workloads.INPLACE_4B, T=512, C=128, d=d, f=f, seed=31 + d)
    x = workloads.inplace_inputs(spec, device="cuda")
    O, W, _ = scan(cwl, x, spec.C, spec.eta)
    Oref, Wref = ora.inplace_scan(x["Z"].cpu(), x["Vhat"].cpu(), x["W0"].cpu(), spec.eta, spec.C)
    eo, ew = rel_err(O, Oref), rel_err(W, Wref)
    print(f"bf16 In-Place d={d} f={f}: O {eo:.3e}  W {ew:.3e}")
    assert eo <= TOL and ew <= TOL


def test_streaming_reset_causality(cwl):
    spec = workloads.scaled(workloads.INPLACE_4B, T=512, C=128, d=256, f=384, seed=5)
    x = workloads.inplace_inputs(spec, device="cuda")
    O1, W1, st = scan(cwl, x, spec.C, spec.eta)
    st.reset()
    O2 = torch.empty_like(O1)
    st.chunk_scan(x["Z"][:256], x["Vhat"][:256], out=O2[:256])
    st.chunk_scan(x["Z"][256:], x["Vhat"][256:], out=O2[256:])
    W2 = torch.empty_like(W1)
    st.get_weights(W2)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(W1, W2)
    x2 = dict(x)
    x2["Z"] = x["Z"].clone()
    x2["Z"][384:] = 0
    O3, _, _ = scan(cwl, x2, spec.C, spec.eta)
    assert torch.equal(O3[:384], O1[:384])


@pytest.mark.parametrize("pad_mode", [0, 1])
def test_target_small(cwl, pad_mode):
    spec = workloads.scaled(workloads.INPLACE_128K_TARGET, T=512, C=128, d=256, f=384, seed=41, conv_pad_mode=pad_mode)
    x = workloads.inplace_inputs(spec, device="cuda")
    O, W, _ = scan(cwl, x, spec.C, spec.eta, target=True, pad_mode=pad_mode)
    V = ora.target_values(x["X0"].cpu(), x["convw"].cpu(), x["Wtarget"].cpu(), spec.C, pad_mode)
    Oref, Wref = ora.inplace_scan(x["Z"].cpu(), V, x["W0"].cpu(), spec.eta, spec.C)
    eo, ew = rel_err(O, Oref), rel_err(W, Wref)
    print(f"bf16 In-Place + target (pad {pad_mode}): O {eo:.3e}  W {ew:.3e}")
    assert eo <= TOL and ew <= TOL


ROWS = [0, 1, 127, 128, 1000, 2047, 2048, 2559]


@pytest.mark.slow
def test_inplace_4b_workload_sampled(cwl):
    """Full 4B-class shape (T=32768, d=2560, f=9728): sampled Wdown rows against the oracle,
    whose rows evolve independently (O[:, i] and W[i] need only V̂[:, i], W0[i] and Z)."""
    spec = workloads.INPLACE_4B
    x = workloads.inplace_inputs(spec, device="cuda")
    O, W, _ = scan(cwl, x, spec.C, spec.eta)
    Z = x["Z"].cpu()
    Oref, Wref = ora.inplace_scan_rows(Z, x["Vhat"][:, ROWS].cpu(), x["W0"][ROWS].cpu(), spec.eta, spec.C)
    eo, ew = rel_err(O[:, ROWS], Oref), rel_err(W[ROWS], Wref)
    print(f"4B-class workload sampled rows: O {eo:.3e}  W {ew:.3e}")
    assert eo <= TOL and ew <= TOL
    assert torch.isfinite(O.float()).all()


@pytest.mark.slow
def test_inplace_128k_target_workload_sampled(cwl):
    spec = workloads.INPLACE_128K_TARGET
    x = workloads.inplace_inputs(spec, device="cuda")
    O, W, _ = scan(cwl, x, spec.C, spec.eta, target=True)
    V = ora.target_values(x["X0"].cpu(), x["convw"].cpu(), x["Wtarget"].cpu(), spec.C, 0, cols=ROWS)
    Oref, Wref = ora.inplace_scan_rows(x["Z"].cpu(), V, x["W0"][ROWS].cpu(), spec.eta, spec.C)
    eo, ew = rel_err(O[:, ROWS], Oref), rel_err(W[ROWS], Wref)
    print(f"128k + target workload sampled rows: O {eo:.3e}  W {ew:.3e}")
    assert eo <= TOL and ew <= TOL
