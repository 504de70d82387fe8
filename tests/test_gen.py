"""The seeded generator: vectorised SplitMix64 equals the scalar definition, normals have
the right moments, needles are distinct and deterministic."""

import math

import torch

from gen import rng, workloads


def test_splitmix64_matches_scalar_definition():
    key = 0x0123456789ABCDEF ^ rng.fnv1a64("K")
    ctr = torch.arange(0, 64, dtype=torch.int64)
    vec = rng.splitmix64(key, ctr)
    for i in range(64):
        expect = rng.splitmix64_scalar(key, i)
        got = int(vec[i]) & ((1 << 64) - 1)
        assert got == expect


def test_splitmix64_known_value():
    # The first output of SplitMix64 seeded with 0 (published test vector of the generator).
    assert rng.splitmix64_scalar(0, 0) == 0xE220A8397B1DCDAF


def test_fnv1a_known_value():
    assert rng.fnv1a64("") == 0xCBF29CE484222325
    assert rng.fnv1a64("a") == 0xAF63DC4C8601EC8C


def test_normal_moments_and_determinism():
    x = rng.normal("x", (200_000,), 7)
    assert abs(float(x.mean())) < 0.01
    assert abs(float(x.std()) - 1.0) < 0.01
    y = rng.normal("x", (200_000,), 7)
    assert torch.equal(x, y)
    z = rng.normal("y", (200_000,), 7)
    assert not torch.equal(x, z)


def test_needles_distinct_and_stable():
    spec = workloads.SR_TTT_GATE
    p0 = workloads.needle_positions(spec, 0)
    assert len(p0) == round(0.01 * spec.T) == 82
    assert len(set(p0)) == len(p0) and all(0 <= p < spec.T for p in p0)
    assert p0 == workloads.needle_positions(spec, 0)
    assert p0 != workloads.needle_positions(spec, 1)


def test_linear_inputs_small():
    spec = workloads.scaled(workloads.SR_TTT_GATE, B=2, H=3, T=256)
    x = workloads.linear_inputs(spec)
    assert x["K"].dtype == torch.bfloat16 and x["K"].shape == (2, 3, 256, 64)
    assert "Q" not in x
    assert torch.equal(x["W0"][1, 2], torch.eye(64))
    pos = workloads.needle_positions(spec, 1)
    ratio = (x["V"][1, :, pos].float().abs().mean() / x["V"][1].float().abs().mean()).item()
    assert ratio > 4.0


def test_inplace_inputs_small():
    spec = workloads.scaled(workloads.INPLACE_4B, T=64, C=32, d=32, f=48)
    x = workloads.inplace_inputs(spec)
    assert x["Z"].shape == (64, 48) and x["Z"].dtype == torch.bfloat16
    assert x["Vhat"].shape == (64, 32) and x["W0"].shape == (32, 48)
    assert abs(float(x["W0"].std()) - 0.02) < 0.004
    spec_t = workloads.scaled(workloads.INPLACE_128K_TARGET, T=64, C=32, d=32, f=48)
    xt = workloads.inplace_inputs(spec_t)
    assert xt["X0"].shape == (64, 32) and xt["Wtarget"].shape == (32, 32)
    assert xt["convw"].shape == (32, 3)
    assert math.isclose(float(xt["convw"].var()), 1 / 3, rel_tol=0.35)
