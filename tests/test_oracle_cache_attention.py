"""Pins of the residual-cache read path oracle: a hand-derived example, softmax special cases
with exact answers, a dense masked-attention formulation, causality, order invariance and
the clamp of α."""

import json
import os

import numpy as np

from oracle import cache_attention

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _one(x):
    return np.asarray(x, float)[None, None]


def _cache(tokens, capacity, B=1, H=1, routed=None):
    """Entries [B, H, capacity, 3] and counts [B, H, 2] holding ``tokens`` for every (b, h)."""
    E = np.full((B, H, capacity, 3), -1, np.int32)
    C = np.zeros((B, H, 2), np.int32)
    n = min(len(tokens), capacity)
    for b in range(B):
        for h in range(H):
            for j, t in enumerate(tokens[:n]):
                E[b, h, j] = (b, h, t)
            r = len(tokens) if routed is None else routed
            C[b, h] = (r, max(0, r - capacity))
    return E, C


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "cache_attention_hand.json")))
    E = np.asarray(g["entries"], np.int32)[None, None]
    C = np.asarray(g["counts"], np.int32)[None, None]
    A = cache_attention.cache_attention(_one(g["Q"]), _one(g["K"]), _one(g["V"]), E, C, g["gate_chunk"])
    np.testing.assert_allclose(A[0, 0], np.asarray(g["A"], float), rtol=0, atol=1e-14)
    T = len(g["Q"])
    O_ttt = np.repeat(np.arange(T, dtype=float)[:, None], 4, axis=1)
    O = cache_attention.alpha_fusion(_one(O_ttt), A, np.asarray(g["alpha"], float)[None])
    np.testing.assert_allclose(O[0, 0], np.asarray(g["O"], float), rtol=0, atol=1e-14)


def test_single_visible_entry_returns_its_value_exactly():
    """A softmax over one score is exactly 1, so every query after the entry's chunk returns
    that entry's value bit for bit, and every query up to its chunk returns zero."""
    T, D, gc = 40, 8, 8
    Q, K, V = _rand((1, 1, T, D), 1), _rand((1, 1, T, D), 2), _rand((1, 1, T, D), 3)
    E, C = _cache([13], 4)
    A = cache_attention.cache_attention(Q, K, V, E, C, gc)
    for t in range(T):
        want = V[0, 0, 13] if t // gc > 13 // gc else np.zeros(D)
        assert np.array_equal(A[0, 0, t], want), t


def test_identical_keys_average_the_values():
    T, D, gc = 32, 4, 4
    Q, V = _rand((1, 1, T, D), 4), _rand((1, 1, T, D), 5)
    K = np.tile(_rand((1, 1, 1, D), 6), (1, 1, T, 1))
    cached = [1, 6, 9, 14, 22]
    E, C = _cache(cached, 8)
    A = cache_attention.cache_attention(Q, K, V, E, C, gc)
    for t in range(T):
        vis = [c for c in cached if c // gc < t // gc]
        want = np.mean(V[0, 0, vis], axis=0) if vis else np.zeros(D)
        np.testing.assert_allclose(A[0, 0, t], want, rtol=0, atol=1e-14)


def test_two_entries_follow_the_logistic_weight():
    """With two visible entries the weight of the second is σ(s₂ − s₁), s = q·k/√D."""
    D = 16
    q, k1, k2, v1, v2 = (_rand(D, s) for s in (7, 8, 9, 10, 11))
    Q = np.zeros((1, 1, 3, D))
    Q[0, 0, 2] = q
    K = np.stack([k1, k2, np.zeros(D)])[None, None]
    V = np.stack([v1, v2, np.zeros(D)])[None, None]
    E, C = _cache([0, 1], 2)
    A = cache_attention.cache_attention(Q, K, V, E, C, gate_chunk=2)
    s1, s2 = q @ k1 / 4.0, q @ k2 / 4.0
    w2 = 1.0 / (1.0 + np.exp(s1 - s2))
    np.testing.assert_allclose(A[0, 0, 2], (1 - w2) * v1 + w2 * v2, rtol=1e-13, atol=1e-14)


def test_equals_dense_masked_attention():
    """The same attention as a dense softmax over all T tokens with every token masked out
    that is not cached or whose gate chunk is not before the query's."""
    B, H, T, D, gc = 2, 3, 96, 16, 16
    Q, K, V = (_rand((B, H, T, D), s) for s in (12, 13, 14))
    rng = np.random.default_rng(15)
    E = np.full((B, H, 12, 3), -1, np.int32)
    Cn = np.zeros((B, H, 2), np.int32)
    for b in range(B):
        for h in range(H):
            toks = np.sort(rng.choice(T, size=15, replace=False))
            for j, t in enumerate(toks[:12]):
                E[b, h, j] = (b, h, t)
            Cn[b, h] = (15, 3)
    A = cache_attention.cache_attention(Q, K, V, E, Cn, gc)
    for b in range(B):
        for h in range(H):
            cached = np.zeros(T, bool)
            cached[E[b, h, :12, 2]] = True
            S = (Q[b, h] @ K[b, h].T) / np.sqrt(D)
            chunk = np.arange(T) // gc
            mask = cached[None, :] & (chunk[None, :] < chunk[:, None])
            S = np.where(mask, S, -np.inf)
            has = mask.any(axis=1)
            P = np.zeros_like(S)
            P[has] = np.exp(S[has] - S[has].max(axis=1, keepdims=True))
            P[has] /= P[has].sum(axis=1, keepdims=True)
            np.testing.assert_allclose(A[b, h], P @ V[b, h], rtol=0, atol=1e-12)


def test_causal_bit_exact():
    """Changing the keys and values of gate chunks ≥ g leaves every output of chunks ≤ g
    unchanged bit for bit (those queries read only entries of earlier chunks), and changing
    the queries of chunks ≥ g leaves the outputs of chunks < g unchanged."""
    T, D, gc, g = 64, 8, 8, 4
    Q, K, V = (_rand((1, 1, T, D), s) for s in (16, 17, 18))
    E, C = _cache([2, 9, 17, 30, 33, 41, 50, 60], 8)
    A = cache_attention.cache_attention(Q, K, V, E, C, gc)
    K2, V2 = K.copy(), V.copy()
    K2[0, 0, g * gc:] += 5.0
    V2[0, 0, g * gc:] -= 3.0
    A2 = cache_attention.cache_attention(Q, K2, V2, E, C, gc)
    assert np.array_equal(A[0, 0, :(g + 1) * gc], A2[0, 0, :(g + 1) * gc])
    assert not np.array_equal(A[0, 0, (g + 1) * gc:], A2[0, 0, (g + 1) * gc:])
    Q3 = Q.copy()
    Q3[0, 0, g * gc:] *= -2.0
    A3 = cache_attention.cache_attention(Q3, K, V, E, C, gc)
    assert np.array_equal(A[0, 0, :g * gc], A3[0, 0, :g * gc])


def test_order_of_entries_does_not_matter():
    T, D, gc = 48, 8, 8
    Q, K, V = (_rand((1, 1, T, D), s) for s in (19, 20, 21))
    toks = [3, 11, 12, 20, 27, 35]
    E1, C1 = _cache(toks, 6)
    E2, C2 = _cache(toks[::-1], 6)
    A1 = cache_attention.cache_attention(Q, K, V, E1, C1, gc)
    A2 = cache_attention.cache_attention(Q, K, V, E2, C2, gc)
    np.testing.assert_allclose(A1, A2, rtol=0, atol=1e-13)


def test_only_stored_entries_are_read():
    """Entries past min(routed, capacity) are never read, whatever they hold: an unused -1 row
    (which as an index would wrap to the last token) and a full cache that dropped tokens."""
    T, D, gc = 32, 4, 4
    Q, K, V = (_rand((1, 1, T, D), s) for s in (22, 23, 24))
    E, C = _cache([1, 5], 4)
    A = cache_attention.cache_attention(Q, K, V, E, C, gc)
    E_one, C_one = _cache([1], 4)
    E_one[0, 0, 1] = (0, 0, 5)      # a stale row past the count
    C_one[0, 0] = (1, 0)
    A_one = cache_attention.cache_attention(Q, K, V, E_one, C_one, gc)
    assert np.array_equal(A_one[0, 0, 4:], np.tile(V[0, 0, 1], (T - 4, 1)))
    assert not np.array_equal(A, A_one)
    # Routed beyond capacity: the first `capacity` stored tokens only.
    E_full, C_full = _cache([1, 5, 9, 13, 17, 21], 2)
    assert C_full[0, 0, 0] == 6 and C_full[0, 0, 1] == 4
    E_two, C_two = _cache([1, 5], 2)
    assert np.array_equal(cache_attention.cache_attention(Q, K, V, E_full, C_full, gc),
                          cache_attention.cache_attention(Q, K, V, E_two, C_two, gc))


def test_alpha_is_clamped_to_the_unit_interval():
    B, H, T, D = 1, 2, 4, 3
    O, A = _rand((B, H, T, D), 25), _rand((B, H, T, D), 26)
    zero = np.zeros((H, D))
    assert np.array_equal(cache_attention.alpha_fusion(O, A, zero), O)
    assert np.array_equal(cache_attention.alpha_fusion(O, A, zero - 3.0), O)
    one = cache_attention.alpha_fusion(O, A, zero + 1.0)
    assert np.array_equal(one, O + A)
    assert np.array_equal(cache_attention.alpha_fusion(O, A, zero + 7.0), one)
    alpha = np.array([[0.25, 2.0, -1.0], [0.5, 0.0, 1.0]])
    got = cache_attention.alpha_fusion(O, A, alpha)
    for h in range(H):
        for c in range(D):
            w = min(1.0, max(0.0, alpha[h, c]))
            assert np.array_equal(got[0, h, :, c], O[0, h, :, c] + w * A[0, h, :, c])
