"""Pins of the In-Place oracle to things other than itself.

Each test would catch a plausible slip in oracle/inplace.py: a wrong sign of ΔW, a
transposed Wdown or V̂ᵀZ, an update applied before the chunk's own output, a dropped
prefix term, a mis-indexed convolution tap or boundary.
"""

import json
import os

import numpy as np
import pytest

from oracle import inplace

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "inplace_hand.json")))
    O, W = inplace.inplace_scan(np.array(g["Z"], float), np.array(g["Vhat"], float),
                                np.array(g["W0"], float), g["eta"], g["C"])
    np.testing.assert_array_equal(O, np.array(g["O"], float))
    np.testing.assert_array_equal(W, np.array(g["W_final"], float))


def test_prefix_sum_identity():
    """W_c = W0 + Σ_{j<c} ΔW_j and the parallel apply (context parallelism) equal the loop."""
    T, C, d, f = 48, 16, 5, 7
    Z, V, W0 = _rand((T, f), 1), _rand((T, d), 2), _rand((d, f), 3)
    O1, W1 = inplace.inplace_scan(Z, V, W0, 0.37, C)
    O2, W2 = inplace.inplace_scan_prefix(Z, V, W0, 0.37, C)
    np.testing.assert_allclose(O1, O2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(W1, W2, rtol=1e-12, atol=1e-12)


def test_dual_form():
    """O_c = Z_c W0ᵀ + η Σ_{j<c} (Z_c Z_jᵀ) V̂_j, written without any W state."""
    T, C, d, f = 40, 8, 3, 6
    eta = 0.25
    Z, V, W0 = _rand((T, f), 4), _rand((T, d), 5), _rand((d, f), 6)
    O, W = inplace.inplace_scan(Z, V, W0, eta, C)
    for c in range(T // C):
        Zc = Z[c * C:(c + 1) * C]
        ref = Zc @ W0.T
        for j in range(c):
            Zj, Vj = Z[j * C:(j + 1) * C], V[j * C:(j + 1) * C]
            ref = ref + eta * (Zc @ Zj.T) @ Vj
        np.testing.assert_allclose(O[c * C:(c + 1) * C], ref, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(W, W0 + eta * V.T @ Z, rtol=1e-12, atol=1e-12)


def test_eta_zero_is_plain_projection():
    """η = 0 leaves Wdown untouched: O[t,i] = Σ_j Z[t,j] W0[i,j] by a textbook triple loop."""
    T, C, d, f = 6, 2, 3, 4
    Z, V, W0 = _rand((T, f), 7), _rand((T, d), 8), _rand((d, f), 9)
    O, W = inplace.inplace_scan(Z, V, W0, 0.0, C)
    for t in range(T):
        for i in range(d):
            s = 0.0
            for j in range(f):
                s += Z[t, j] * W0[i, j]
            assert abs(O[t, i] - s) < 1e-12
    np.testing.assert_array_equal(W, W0)


def test_brute_force_token_loop():
    """Scalar token-by-token restatement: outputs from the frozen W, deltas pending until
    the chunk ends, then W[i,j] += η Σ_t V̂[t,i] Z[t,j]."""
    T, C, d, f = 9, 3, 2, 3
    eta = 0.5
    Z, V, W0 = _rand((T, f), 10), _rand((T, d), 11), _rand((d, f), 12)
    W = [[W0[i, j] for j in range(f)] for i in range(d)]
    pend = [[0.0] * f for _ in range(d)]
    O = [[0.0] * d for _ in range(T)]
    for t in range(T):
        for i in range(d):
            O[t][i] = sum(Z[t, j] * W[i][j] for j in range(f))
            for j in range(f):
                pend[i][j] += eta * V[t, i] * Z[t, j]
        if (t + 1) % C == 0:
            for i in range(d):
                for j in range(f):
                    W[i][j] += pend[i][j]
                    pend[i][j] = 0.0
    O2, W2 = inplace.inplace_scan(Z, V, W0, eta, C)
    np.testing.assert_allclose(O2, np.array(O), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(W2, np.array(W), rtol=1e-12, atol=1e-12)


def test_single_chunk_closed_form():
    T = C = 5
    d, f = 3, 4
    Z, V, W0 = _rand((T, f), 13), _rand((T, d), 14), _rand((d, f), 15)
    O, W = inplace.inplace_scan(Z, V, W0, 0.125, C)
    np.testing.assert_allclose(O, Z @ W0.T, rtol=1e-13)
    np.testing.assert_allclose(W, W0 + 0.125 * V.T @ Z, rtol=1e-13)


def test_causality():
    """Perturbing chunk k changes nothing produced before chunk k (bit for bit)."""
    T, C, d, f = 32, 8, 4, 5
    Z, V, W0 = _rand((T, f), 16), _rand((T, d), 17), _rand((d, f), 18)
    O, _ = inplace.inplace_scan(Z, V, W0, 0.3, C)
    k = 2
    Z2, V2 = Z.copy(), V.copy()
    Z2[k * C:] += _rand((T - k * C, f), 19)
    V2[k * C:] -= 1.0
    O2, _ = inplace.inplace_scan(Z2, V2, W0, 0.3, C)
    assert np.array_equal(O[:k * C], O2[:k * C])
    assert not np.array_equal(O[k * C:], O2[k * C:])


def test_rows_are_independent():
    T, C, d, f = 24, 8, 6, 5
    Z, V, W0 = _rand((T, f), 20), _rand((T, d), 21), _rand((d, f), 22)
    O, W = inplace.inplace_scan(Z, V, W0, 0.2, C)
    rows = [4, 1]
    Or, Wr = inplace.inplace_scan_rows(Z, V[:, rows], W0[rows], 0.2, C)
    np.testing.assert_array_equal(Or, O[:, rows])
    np.testing.assert_array_equal(Wr, W[rows])


def test_rejects_ragged_chunks():
    with pytest.raises(ValueError):
        inplace.inplace_scan(np.zeros((10, 2)), np.zeros((10, 2)), np.zeros((2, 2)), 0.1, 4)


def test_target_conv_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "target_conv_hand.json")))
    X0, w = np.array(g["X0"], float), np.array(g["convw"], float)
    np.testing.assert_array_equal(inplace.target_conv(X0, w, g["C"], 0), np.array(g["conv_mode0"], float))
    np.testing.assert_array_equal(inplace.target_conv(X0, w, g["C"], 1), np.array(g["conv_mode1"], float))
    conv = np.array(g["proj_conv"], float)
    Wt = np.array(g["proj_Wtarget"], float)
    # V̂ = conv · Wtarget, through target_values with identity taps (w = [1, 0, 0]).
    V = inplace.target_values(conv, np.array([[1.0, 0, 0], [1.0, 0, 0]]), Wt, 1, 0)
    np.testing.assert_array_equal(V, np.array(g["proj_Vhat"], float))


def test_target_conv_impulse():
    """A unit impulse at token s, channel i reaches conv[t,i] for t = s, s-1, s-2 inside s's chunk."""
    T, C, d = 12, 4, 3
    w = _rand((d, 3), 23)
    for s in range(T):
        X0 = np.zeros((T, d))
        X0[s, 1] = 1.0
        conv = inplace.target_conv(X0, w, C, 0)
        expect = np.zeros((T, d))
        for k in range(3):
            t = s - k
            if t >= 0 and t // C == s // C:
                expect[t, 1] = w[1, k]
        np.testing.assert_array_equal(conv, expect)
