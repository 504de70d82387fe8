"""Pins of the TTT-Linear oracle: finite differences, the delta rule, fixed points,
projection, affine composition and a hand-derived example."""

import json
import os

import numpy as np

from oracle import linear

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return scale * np.random.default_rng(seed).standard_normal(shape)


def _single(x):
    return np.asarray(x, float)[None, None]


def test_hand_examples():
    g = json.load(open(os.path.join(GOLDEN, "linear_hand.json")))
    for case in ("scalar_case", "matrix_case"):
        c = g[case]
        O, W, L = linear.ttt_linear_scan(_single(c["K"]), _single(c["V"]), _single(c["Q"]),
                                         _single(c["W0"]), c["eta"], c["b"])
        np.testing.assert_array_equal(O[0, 0], np.array(c["O"], float))
        np.testing.assert_array_equal(L[0, 0], np.array(c["loss"], float))
        np.testing.assert_array_equal(W[0, 0], np.array(c["W_final"], float))


def test_step_is_gradient_descent_by_finite_differences():
    """One mini-batch step equals W − η·∇ℓ(W) with ℓ = 1/(2b)‖KW − V‖², gradient by
    central differences in float64."""
    D, b, eta = 4, 2, 0.7
    K, V, W0 = _rand((b, D), 1), _rand((b, D), 2), _rand((D, D), 3)
    h = 1e-6
    grad = np.zeros((D, D))
    for i in range(D):
        for j in range(D):
            Wp, Wm = W0.copy(), W0.copy()
            Wp[i, j] += h
            Wm[i, j] -= h
            grad[i, j] = (linear.inner_loss(K, V, Wp) - linear.inner_loss(K, V, Wm)) / (2 * h)
    _, W1, _ = linear.ttt_linear_scan(_single(K), _single(V), None, _single(W0), eta, b)
    np.testing.assert_allclose(W1[0, 0], W0 - eta * grad, rtol=0, atol=1e-8)


def test_batch_one_is_delta_rule():
    """Inner mini-batch 1 without LayerNorm/residual is DeltaNet's delta rule:
    w ← w − η·kᵀ(k·w − v), token by token (written here with plain loops)."""
    T, D, eta = 12, 3, 0.3
    K, V, W0 = _rand((T, D), 4), _rand((T, D), 5), _rand((D, D), 6)
    W = [[W0[i, j] for j in range(D)] for i in range(D)]
    for t in range(T):
        r = [sum(K[t, i] * W[i][j] for i in range(D)) - V[t, j] for j in range(D)]
        for i in range(D):
            for j in range(D):
                W[i][j] -= eta * K[t, i] * r[j]
    _, W2, _ = linear.ttt_linear_scan(_single(K), _single(V), None, _single(W0), eta, 1)
    np.testing.assert_allclose(W2[0, 0], np.array(W), rtol=1e-12, atol=1e-12)


def test_identity_is_fixed_point_when_values_equal_keys():
    B, H, T, D = 2, 3, 32, 8
    K = _rand((B, H, T, D), 7)
    Q = _rand((B, H, T, D), 8)
    W0 = np.broadcast_to(np.eye(D), (B, H, D, D)).copy()
    O, W, L = linear.ttt_linear_scan(K, K, Q, W0, 1.0, 4)
    assert np.array_equal(W, W0)
    assert np.array_equal(L, np.zeros_like(L))
    np.testing.assert_array_equal(O, Q)


def test_unit_key_step_projects_onto_value():
    """b = 1, ‖k‖ = 1, η = 1: after the step the inner model maps k exactly to v."""
    D = 5
    k = _rand((1, D), 9)
    k /= np.linalg.norm(k)
    v, W0 = _rand((1, D), 10), _rand((D, D), 11)
    _, W1, _ = linear.ttt_linear_scan(_single(k), _single(v), None, _single(W0), 1.0, 1)
    np.testing.assert_allclose(k @ W1[0, 0], v, rtol=0, atol=1e-12)


def test_affine_composition():
    """W_{i+1} = A_i W_i + B_i with A_i = I − (η/b)K_iᵀK_i and B_i = (η/b)K_iᵀV_i."""
    T, D, b, eta = 48, 6, 8, 0.9
    K, V, W0 = _rand((T, D), 12), _rand((T, D), 13), _rand((D, D), 14)
    W = W0.copy()
    for i in range(T // b):
        Ki, Vi = K[i * b:(i + 1) * b], V[i * b:(i + 1) * b]
        A = np.eye(D) - (eta / b) * Ki.T @ Ki
        Bm = (eta / b) * Ki.T @ Vi
        W = A @ W + Bm
    _, W2, _ = linear.ttt_linear_scan(_single(K), _single(V), None, _single(W0), eta, b)
    np.testing.assert_allclose(W2[0, 0], W, rtol=1e-11, atol=1e-11)


def test_outputs_and_losses_use_weight_at_start_of_minibatch():
    """Every row of mini-batch i sees W_i; the loss is ‖k_t W_i − v_t‖² for all b rows."""
    T, D, b, eta = 16, 4, 4, 0.5
    K, V, Q, W0 = _rand((T, D), 15), _rand((T, D), 16), _rand((T, D), 17), _rand((D, D), 18)
    O, _, L = linear.ttt_linear_scan(_single(K), _single(V), _single(Q), _single(W0), eta, b)
    W = W0.copy()
    for i in range(T // b):
        s = slice(i * b, (i + 1) * b)
        for t in range(i * b, (i + 1) * b):
            np.testing.assert_allclose(O[0, 0, t], Q[t] @ W, rtol=1e-12, atol=1e-12)
            r = K[t] @ W - V[t]
            assert abs(L[0, 0, t] - float(r @ r)) < 1e-12
        W = W - (eta / b) * K[s].T @ (K[s] @ W - V[s])


def test_heads_are_independent():
    B, H, T, D = 2, 2, 16, 4
    K, V, Q = _rand((B, H, T, D), 19), _rand((B, H, T, D), 20), _rand((B, H, T, D), 21)
    W0 = _rand((B, H, D, D), 22)
    O, W, L = linear.ttt_linear_scan(K, V, Q, W0, 0.4, 4)
    O1, W1, L1 = linear.ttt_linear_scan(K[1:2, 0:1], V[1:2, 0:1], Q[1:2, 0:1], W0[1:2, 0:1], 0.4, 4)
    np.testing.assert_array_equal(O[1, 0], O1[0, 0])
    np.testing.assert_array_equal(W[1, 0], W1[0, 0])
    np.testing.assert_array_equal(L[1, 0], L1[0, 0])


def test_token_weights_last_and_first_token():
    """Per-token weights: the last token of a mini-batch gives the plain scan's output at the next
    mini-batch's first token (weight W_{i+1}); the first token the output of a plain scan with
    mini-batch 1 and step η/b after that token alone (the delta rule's step)."""
    T, D, b, eta = 24, 5, 4, 0.4
    K, V, Q, W0 = _rand((T, D), 30), _rand((T, D), 31), _rand((T, D), 32), _rand((D, D), 33)
    O_tw, W_tw, L_tw = linear.ttt_linear_scan(_single(K), _single(V), _single(Q), _single(W0), eta, b,
                                              token_weights=True)
    last = np.arange(b - 1, T - b, b)
    Q2 = Q.copy()
    Q2[last + 1] = Q[last]
    O_pl, W_pl, L_pl = linear.ttt_linear_scan(_single(K), _single(V), _single(Q2), _single(W0), eta, b)
    np.testing.assert_allclose(O_tw[0, 0, last], O_pl[0, 0, last + 1], rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(W_tw, W_pl)
    np.testing.assert_array_equal(L_tw, L_pl)
    K2, V2, Q3 = (np.stack([x[0], x[0]]) for x in (K, V, Q))
    O_one = linear.ttt_linear_scan(_single(K2), _single(V2), _single(Q3), _single(W0), eta / b, 1)[0]
    np.testing.assert_allclose(O_tw[0, 0, 0], O_one[0, 0, 1], rtol=1e-12, atol=1e-12)
