"""Pins of the richer inner-model oracle (TTT-Linear with LayerNorm and residual, TTT-MLP):
a hand-derived example, LayerNorm's closed forms and invariances, tabulated GELU values,
finite differences of the loss, and special cases that reduce to simpler models."""

import json
import os

import numpy as np

from oracle import inner

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return scale * np.random.default_rng(seed).standard_normal(shape)


def _single(x):
    return np.asarray(x, float)[None, None]


def test_hand_example_ln_linear():
    c = json.load(open(os.path.join(GOLDEN, "inner_ln_hand.json")))["ln_linear_case"]
    O, W, L = inner.ttt_linear_ln_scan(_single(c["K"]), _single(c["V"]), _single(c["Q"]), _single(c["W0"]),
                                       [c["gamma"]], [c["beta"]], c["eta"], c["b"], c["eps"])
    np.testing.assert_array_equal(O[0, 0], np.array(c["O"], float))
    np.testing.assert_array_equal(L[0, 0], np.array(c["loss"], float))
    np.testing.assert_array_equal(W[0, 0], np.array(c["W_final"], float))


def test_gelu_tabulated_values_and_odd_part():
    c = json.load(open(os.path.join(GOLDEN, "inner_ln_hand.json")))["gelu_values"]
    np.testing.assert_allclose(inner.gelu(np.array(c["x"])), c["gelu"], rtol=0, atol=1e-15)
    x = _rand(1000, 1, 3.0)
    # x·Φ(x) − (−x)·Φ(−x) = x·(Φ(x) + 1 − Φ(x)) = x
    np.testing.assert_allclose(inner.gelu(x) - inner.gelu(-x), x, rtol=0, atol=1e-13)
    assert abs(inner.gelu(np.array(12.0)) - 12.0) < 1e-15 and abs(inner.gelu(np.array(-12.0))) < 1e-15


def test_gelu_grad_by_finite_differences():
    x = _rand(200, 2, 3.0)
    h = 1e-6
    np.testing.assert_allclose(inner.gelu_grad(x), (inner.gelu(x + h) - inner.gelu(x - h)) / (2 * h),
                               rtol=0, atol=1e-8)


def test_layer_norm_closed_forms():
    """γ = 1, β = 0: every row has mean 0 and mean square σ²/(σ² + ε) with σ² the population
    variance; γ and β act as y = γ·ẑ + β."""
    Z = _rand((50, 64), 3, 2.0) + 5.0
    eps = 0.3
    one, zero = np.ones(64), np.zeros(64)
    Y, _, _ = inner.layer_norm(Z, one, zero, eps)
    np.testing.assert_allclose(Y.mean(axis=1), 0.0, atol=1e-12)
    var = np.var(Z, axis=1)
    np.testing.assert_allclose((Y * Y).mean(axis=1), var / (var + eps), rtol=1e-12)
    gamma, beta = _rand(64, 4), _rand(64, 5)
    Yg, _, _ = inner.layer_norm(Z, gamma, beta, eps)
    np.testing.assert_allclose((Yg - beta) / gamma, Y, rtol=1e-10, atol=1e-12)


def test_layer_norm_shift_and_scale_invariance():
    Z = _rand((20, 16), 6)
    one, zero = np.ones(16), np.zeros(16)
    shift = _rand((20, 1), 7, 10.0)
    np.testing.assert_allclose(inner.layer_norm(Z + shift, one, zero, 0.1)[0],
                               inner.layer_norm(Z, one, zero, 0.1)[0], rtol=0, atol=1e-11)
    np.testing.assert_allclose(inner.layer_norm(7.5 * Z, one, zero, 0.0)[0],
                               inner.layer_norm(Z, one, zero, 0.0)[0], rtol=0, atol=1e-12)


def test_ln_linear_step_is_gradient_descent_by_finite_differences():
    D, b, eta, eps = 4, 3, 0.7, 0.05
    K, V, W0 = _rand((b, D), 8), _rand((b, D), 9), _rand((D, D), 10)
    gamma, beta = _rand(D, 11) + 1.0, _rand(D, 12)
    h = 1e-6
    grad = np.zeros((D, D))
    for i in range(D):
        for j in range(D):
            Wp, Wm = W0.copy(), W0.copy()
            Wp[i, j] += h
            Wm[i, j] -= h
            grad[i, j] = (inner.inner_loss_ln(K, V, Wp, gamma, beta, eps)
                          - inner.inner_loss_ln(K, V, Wm, gamma, beta, eps)) / (2 * h)
    _, W1, _ = inner.ttt_linear_ln_scan(_single(K), _single(V), None, _single(W0), [gamma], [beta], eta, b, eps)
    np.testing.assert_allclose(W1[0, 0], W0 - eta * grad, rtol=0, atol=1e-8)


def test_mlp_step_is_gradient_descent_by_finite_differences():
    D, Dh, b, eta, eps = 3, 12, 2, 0.6, 0.05
    K, V = _rand((b, D), 13), _rand((b, D), 14)
    W1, W2 = _rand((D, Dh), 15), _rand((Dh, D), 16, 0.5)
    gamma, beta = _rand(D, 17) + 1.0, _rand(D, 18)
    h = 1e-6

    def loss(a, c):
        return inner.inner_loss_mlp(K, V, a, c, gamma, beta, eps)

    g1, g2 = np.zeros_like(W1), np.zeros_like(W2)
    for idx in np.ndindex(W1.shape):
        p, m = W1.copy(), W1.copy()
        p[idx] += h
        m[idx] -= h
        g1[idx] = (loss(p, W2) - loss(m, W2)) / (2 * h)
    for idx in np.ndindex(W2.shape):
        p, m = W2.copy(), W2.copy()
        p[idx] += h
        m[idx] -= h
        g2[idx] = (loss(W1, p) - loss(W1, m)) / (2 * h)
    _, A, B_, _ = inner.ttt_mlp_scan(_single(K), _single(V), None, _single(W1), _single(W2), [gamma], [beta],
                                     eta, b, eps)
    np.testing.assert_allclose(A[0, 0], W1 - eta * g1, rtol=0, atol=1e-8)
    np.testing.assert_allclose(B_[0, 0], W2 - eta * g2, rtol=0, atol=1e-8)


def test_zero_gain_leaves_only_the_residual():
    """γ = β = 0: the LayerNorm branch is zero, so f(x) = x: outputs are the queries, the loss is
    ‖k − v‖², and no gradient reaches the weights."""
    B, H, T, D = 1, 2, 32, 8
    K, V, Q = _rand((B, H, T, D), 19), _rand((B, H, T, D), 20), _rand((B, H, T, D), 21)
    W0 = _rand((B, H, D, D), 22)
    z = np.zeros((H, D))
    O, W, L = inner.ttt_linear_ln_scan(K, V, Q, W0, z, z, 0.5, 4, 1e-6)
    np.testing.assert_array_equal(O, Q)
    np.testing.assert_array_equal(W, W0)
    np.testing.assert_allclose(L, np.sum((K - V) ** 2, axis=3), rtol=1e-14)
    W1, W2 = _rand((B, H, D, 4 * D), 23), _rand((B, H, 4 * D, D), 24)
    O, A, C, L = inner.ttt_mlp_scan(K, V, Q, W1, W2, z, z, 0.5, 4, 1e-6)
    np.testing.assert_array_equal(O, Q)
    np.testing.assert_array_equal(A, W1)
    np.testing.assert_array_equal(C, W2)


def test_mlp_with_zero_second_layer():
    """W2 = 0: every token's LayerNorm input is zero, so LN gives β and o = q + β; the first
    layer gets no gradient (it reaches W1 only through W2), the second does."""
    T, D, b = 8, 4, 4
    K, V, Q = _rand((T, D), 25), _rand((T, D), 26), _rand((T, D), 27)
    W1, W2 = _rand((D, 4 * D), 28), np.zeros((4 * D, D))
    gamma, beta = _rand(D, 29) + 1.0, _rand(D, 30)
    O, A, C, _ = inner.ttt_mlp_scan(_single(K[:b]), _single(V[:b]), _single(Q[:b]), _single(W1), _single(W2),
                                    [gamma], [beta], 0.5, b, 1e-3)
    np.testing.assert_array_equal(O[0, 0], Q[:b] + beta)
    np.testing.assert_array_equal(A[0, 0], W1)
    assert np.abs(C[0, 0]).max() > 1e-3


def test_mlp_with_identity_activation_is_linear_in_the_product():
    """With the activation replaced by the identity, the MLP computes x·(W1·W2): its outputs and
    losses over the first mini-batch equal the LayerNorm TTT-Linear's with W = W1·W2."""
    B, H, T, D, b = 1, 2, 8, 6, 8
    K, V, Q = _rand((B, H, T, D), 31), _rand((B, H, T, D), 32), _rand((B, H, T, D), 33)
    W1, W2 = _rand((B, H, D, 4 * D), 34), _rand((B, H, 4 * D, D), 35, 0.3)
    gamma, beta = _rand((H, D), 36) + 1.0, _rand((H, D), 37)
    O1, _, _, L1 = inner.ttt_mlp_scan(K, V, Q, W1, W2, gamma, beta, 0.5, b, 1e-4, activation="identity")
    O2, _, L2 = inner.ttt_linear_ln_scan(K, V, Q, W1 @ W2, gamma, beta, 0.5, b, 1e-4)
    np.testing.assert_allclose(O1, O2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(L1, L2, rtol=1e-12, atol=1e-12)


def test_ln_linear_scale_of_the_weight():
    """ε = 0: LN(k·cW) = LN(k·W) for c > 0, so the first mini-batch's outputs and losses do not
    change, and the gradient through LN's 1/σ scales as 1/c: c·(W'(cW) − cW) = W'(W) − W."""
    T, D, b, c = 4, 5, 4, 3.0
    K, V, Q, W0 = _rand((T, D), 38), _rand((T, D), 39), _rand((T, D), 40), _rand((D, D), 41)
    gamma, beta = _rand(D, 42) + 1.0, _rand(D, 43)
    Oa, Wa, La = inner.ttt_linear_ln_scan(_single(K), _single(V), _single(Q), _single(W0), [gamma], [beta], 0.4, b, 0.0)
    Ob, Wb, Lb = inner.ttt_linear_ln_scan(_single(K), _single(V), _single(Q), _single(c * W0), [gamma], [beta], 0.4,
                                          b, 0.0)
    np.testing.assert_allclose(Ob, Oa, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Lb, La, rtol=1e-12)
    np.testing.assert_allclose(c * (Wb[0, 0] - c * W0), Wa[0, 0] - W0, rtol=0, atol=1e-12)


def test_causality_and_weight_at_start_of_minibatch():
    """Changing mini-batch i's keys and values changes no output of mini-batches 0..i (they use
    the weights from before its step) and changes the outputs after it."""
    B, H, T, D, b = 1, 1, 32, 8, 8
    K, V, Q = _rand((B, H, T, D), 44), _rand((B, H, T, D), 45), _rand((B, H, T, D), 46)
    W0 = _rand((B, H, D, D), 47, 0.5)
    W1, W2 = _rand((B, H, D, 4 * D), 48, 0.5), _rand((B, H, 4 * D, D), 49, 0.5)
    g, be = _rand((H, D), 50) + 1.0, _rand((H, D), 51)
    K2, V2 = K.copy(), V.copy()
    K2[..., 8:16, :] += 0.5
    V2[..., 8:16, :] -= 0.5
    for run in (lambda k, v: inner.ttt_linear_ln_scan(k, v, Q, W0, g, be, 0.5, b, 1e-5)[0],
                lambda k, v: inner.ttt_mlp_scan(k, v, Q, W1, W2, g, be, 0.5, b, 1e-5)[0]):
        Oa, Ob = run(K, V), run(K2, V2)
        np.testing.assert_array_equal(Oa[..., :16, :], Ob[..., :16, :])
        assert np.abs(Oa[..., 16:, :] - Ob[..., 16:, :]).max() > 1e-6


def test_heads_take_their_own_gain_and_bias():
    B, H, T, D, b = 2, 2, 16, 4, 4
    K, V, Q = _rand((B, H, T, D), 52), _rand((B, H, T, D), 53), _rand((B, H, T, D), 54)
    W0 = _rand((B, H, D, D), 55)
    W1, W2 = _rand((B, H, D, 4 * D), 56), _rand((B, H, 4 * D, D), 57, 0.5)
    g, be = _rand((H, D), 58) + 1.0, _rand((H, D), 59)
    O, W, L = inner.ttt_linear_ln_scan(K, V, Q, W0, g, be, 0.4, b, 1e-5)
    o, w, l = inner.ttt_linear_ln_scan(K[1:, 1:], V[1:, 1:], Q[1:, 1:], W0[1:, 1:], g[1:], be[1:], 0.4, b, 1e-5)
    np.testing.assert_array_equal(O[1, 1], o[0, 0])
    np.testing.assert_array_equal(W[1, 1], w[0, 0])
    np.testing.assert_array_equal(L[1, 1], l[0, 0])
    O, A, C, L = inner.ttt_mlp_scan(K, V, Q, W1, W2, g, be, 0.4, b, 1e-5)
    o, a, c, l = inner.ttt_mlp_scan(K[1:, 1:], V[1:, 1:], Q[1:, 1:], W1[1:, 1:], W2[1:, 1:], g[1:], be[1:], 0.4, b,
                                    1e-5)
    np.testing.assert_array_equal(O[1, 1], o[0, 0])
    np.testing.assert_array_equal(A[1, 1], a[0, 0])
    np.testing.assert_array_equal(C[1, 1], c[0, 0])
    np.testing.assert_array_equal(L[1, 1], l[0, 0])


def test_outputs_and_losses_evaluate_the_same_model():
    """With the queries equal to the keys, o_t = f(k_t; θ_i), so ‖o_t − v_t‖² is the token's loss;
    and the first mini-batch's losses sum to 2b·ℓ(θ_0), the loss the step descends."""
    B, H, T, D, b = 1, 1, 16, 6, 8
    K, V = _rand((B, H, T, D), 60), _rand((B, H, T, D), 61)
    W0 = _rand((B, H, D, D), 62, 0.5)
    W1, W2 = _rand((B, H, D, 4 * D), 63, 0.5), _rand((B, H, 4 * D, D), 64, 0.5)
    g, be = _rand((H, D), 65) + 1.0, _rand((H, D), 66)
    O, _, L = inner.ttt_linear_ln_scan(K, V, K, W0, g, be, 0.5, b, 1e-5)
    np.testing.assert_allclose(np.sum((O - V) ** 2, axis=3), L, rtol=1e-12)
    assert abs(L[0, 0, :b].sum() - 2 * b * inner.inner_loss_ln(K[0, 0, :b], V[0, 0, :b], W0[0, 0], g[0], be[0],
                                                               1e-5)) < 1e-10
    O, _, _, L = inner.ttt_mlp_scan(K, V, K, W1, W2, g, be, 0.5, b, 1e-5)
    np.testing.assert_allclose(np.sum((O - V) ** 2, axis=3), L, rtol=1e-12)
    assert abs(L[0, 0, :b].sum() - 2 * b * inner.inner_loss_mlp(K[0, 0, :b], V[0, 0, :b], W1[0, 0], W2[0, 0], g[0],
                                                                be[0], 1e-5)) < 1e-10


def _shifted_queries(Q, positions, sources):
    """Q with the rows at ``positions`` replaced by the rows at ``sources``."""
    Q2 = Q.copy()
    Q2[..., positions, :] = Q[..., sources, :]
    return Q2


def test_token_weights_last_token_sees_the_next_minibatch_weight():
    """With per-token weights the last token of mini-batch i has taken every step of it, so its
    output is the output the plain scan gives a query equal to it at the first token of
    mini-batch i + 1 (whose weight is θ_{i+1})."""
    B, H, T, D, b = 1, 2, 24, 6, 4
    K, V, Q = _rand((B, H, T, D), 67), _rand((B, H, T, D), 68), _rand((B, H, T, D), 69)
    W0 = _rand((B, H, D, D), 70, 0.5)
    W1, W2 = _rand((B, H, D, 4 * D), 71, 0.5), _rand((B, H, 4 * D, D), 72, 0.5)
    g, be = _rand((H, D), 73) + 1.0, _rand((H, D), 74)
    last = np.arange(b - 1, T - b, b)
    Q2 = _shifted_queries(Q, last + 1, last)
    O_tw = inner.ttt_linear_ln_scan(K, V, Q, W0, g, be, 0.3, b, 1e-4, token_weights=True)[0]
    O_pl = inner.ttt_linear_ln_scan(K, V, Q2, W0, g, be, 0.3, b, 1e-4)[0]
    np.testing.assert_allclose(O_tw[..., last, :], O_pl[..., last + 1, :], rtol=1e-11, atol=1e-11)
    O_tw = inner.ttt_mlp_scan(K, V, Q, W1, W2, g, be, 0.3, b, 1e-4, token_weights=True)[0]
    O_pl = inner.ttt_mlp_scan(K, V, Q2, W1, W2, g, be, 0.3, b, 1e-4)[0]
    np.testing.assert_allclose(O_tw[..., last, :], O_pl[..., last + 1, :], rtol=1e-11, atol=1e-11)


def test_token_weights_first_token_takes_only_its_own_step():
    """The first token of a mini-batch sees θ_i − (η/b)·∇ of its own loss alone: the weight a
    plain scan with mini-batch 1 and step η/b reaches after that one token."""
    B, H, D, b, eta = 1, 2, 6, 4, 0.3
    K, V, Q = _rand((B, H, b, D), 75), _rand((B, H, b, D), 76), _rand((B, H, b, D), 77)
    W0 = _rand((B, H, D, D), 78, 0.5)
    W1, W2 = _rand((B, H, D, 4 * D), 79, 0.5), _rand((B, H, 4 * D, D), 80, 0.5)
    g, be = _rand((H, D), 81) + 1.0, _rand((H, D), 82)
    # Two-token plain scans with mini-batch 1: token 0 steps, token 1 carries the query.
    K2 = np.concatenate([K[..., :1, :], K[..., :1, :]], axis=2)
    V2 = np.concatenate([V[..., :1, :], V[..., :1, :]], axis=2)
    Q2 = np.concatenate([Q[..., :1, :], Q[..., :1, :]], axis=2)
    O_tw = inner.ttt_linear_ln_scan(K, V, Q, W0, g, be, eta, b, 1e-4, token_weights=True)[0]
    O_pl = inner.ttt_linear_ln_scan(K2, V2, Q2, W0, g, be, eta / b, 1, 1e-4)[0]
    np.testing.assert_allclose(O_tw[..., 0, :], O_pl[..., 1, :], rtol=1e-11, atol=1e-11)
    O_tw = inner.ttt_mlp_scan(K, V, Q, W1, W2, g, be, eta, b, 1e-4, token_weights=True)[0]
    O_pl = inner.ttt_mlp_scan(K2, V2, Q2, W1, W2, g, be, eta / b, 1, 1e-4)[0]
    np.testing.assert_allclose(O_tw[..., 0, :], O_pl[..., 1, :], rtol=1e-11, atol=1e-11)


def test_token_weights_change_only_the_outputs():
    """Losses and the final weights do not depend on how the outputs are taken; with mini-batch
    1 the two forms differ by exactly one step (checked above), with larger ones the middle
    tokens differ from both ends."""
    B, H, T, D, b = 1, 1, 16, 5, 8
    K, V, Q = _rand((B, H, T, D), 83), _rand((B, H, T, D), 84), _rand((B, H, T, D), 85)
    W0 = _rand((B, H, D, D), 86, 0.5)
    g, be = _rand((H, D), 87) + 1.0, _rand((H, D), 88)
    Oa, Wa, La = inner.ttt_linear_ln_scan(K, V, Q, W0, g, be, 0.3, b, 1e-4)
    Ob, Wb, Lb = inner.ttt_linear_ln_scan(K, V, Q, W0, g, be, 0.3, b, 1e-4, token_weights=True)
    np.testing.assert_array_equal(Wa, Wb)
    np.testing.assert_array_equal(La, Lb)
    assert np.abs(Oa - Ob).max() > 1e-3
