"""Pins of the packed-sequence oracle (per-document resets, update-norm clipping): a single
document is the plain scan, every document restarts from W0 as if alone, a ragged last chunk
equals its zero-padded chunk, a short last mini-batch is the gradient step of its own loss,
and a clipped chunk delta keeps its direction at exactly the threshold's norm."""

import numpy as np
import pytest

from oracle import inplace, linear, packed


def _rand(shape, seed, scale=1.0):
    return scale * np.random.default_rng(seed).standard_normal(shape)


def test_one_document_is_the_plain_scan():
    T, C, d, f = 96, 32, 6, 10
    Z, V, W0 = _rand((T, f), 1), _rand((T, d), 2), _rand((d, f), 3, 0.1)
    O, W = packed.inplace_scan_docs(Z, V, W0, 0.05, C, [0])
    O_ref, W_ref = inplace.inplace_scan(Z, V, W0, 0.05, C)
    assert np.array_equal(O, O_ref) and np.array_equal(W, W_ref)
    B, H, T, D, b = 2, 2, 64, 4, 8
    K, Vl, Q = _rand((B, H, T, D), 4, 0.5), _rand((B, H, T, D), 5, 0.5), _rand((B, H, T, D), 6)
    W0l = np.broadcast_to(np.eye(D), (B, H, D, D)).copy()
    O, W, L = packed.ttt_linear_scan_docs(K, Vl, Q, W0l, 0.3, b, [[0], [0]])
    O_ref, W_ref, L_ref = linear.ttt_linear_scan(K, Vl, Q, W0l, 0.3, b)
    for got, want in ((O, O_ref), (W, W_ref), (L, L_ref)):
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_every_document_restarts_from_the_pretrained_weight():
    T, C, d, f, eta = 160, 32, 5, 9, 0.07
    Z, V, W0 = _rand((T, f), 7), _rand((T, d), 8), _rand((d, f), 9, 0.1)
    starts = [0, 64, 96]
    O, W = packed.inplace_scan_docs(Z, V, W0, eta, C, starts)
    for a, e in zip(starts, starts[1:] + [T]):
        O_doc, W_doc = inplace.inplace_scan(Z[a:e], V[a:e], W0, eta, C)
        np.testing.assert_allclose(O[a:e], O_doc, rtol=0, atol=1e-13)
    np.testing.assert_allclose(W, W_doc, rtol=0, atol=1e-13)
    # Without the boundaries the later documents would see the earlier ones.
    O_flat, _ = inplace.inplace_scan(Z, V, W0, eta, C)
    assert not np.allclose(O[64:], O_flat[64:])


def test_ragged_last_chunk_equals_its_zero_padded_chunk():
    """A document of 75 tokens with C = 32 ends in an 11-token chunk; padding its Z and V̂
    rows with zeros to 96 tokens changes nothing (zero rows add nothing to V̂ᵀZ)."""
    C, d, f, eta = 32, 4, 6, 0.1
    Z, V, W0 = _rand((75, f), 10), _rand((75, d), 11), _rand((d, f), 12, 0.1)
    O, W = packed.inplace_scan_docs(Z, V, W0, eta, C, [0])
    Zp, Vp = np.zeros((96, f)), np.zeros((96, d))
    Zp[:75], Vp[:75] = Z, V
    O_pad, W_pad = inplace.inplace_scan(Zp, Vp, W0, eta, C)
    np.testing.assert_allclose(O, O_pad[:75], rtol=0, atol=1e-13)
    np.testing.assert_allclose(W, W_pad, rtol=0, atol=1e-13)


def test_clipped_delta_keeps_its_direction_at_the_threshold():
    T, C, d, f, eta = 128, 32, 6, 8, 0.2
    Z, V, W0 = _rand((T, f), 13), _rand((T, d), 14), _rand((d, f), 15, 0.1)
    O_none, W_none = packed.inplace_scan_docs(Z, V, W0, eta, C, [0])
    O_big, W_big = packed.inplace_scan_docs(Z, V, W0, eta, C, [0], clip=1e9)
    assert np.array_equal(O_none, O_big) and np.array_equal(W_none, W_big)
    clip = 1e-5
    Ws = [packed.inplace_scan_docs(Z[:k * C], V[:k * C], W0, eta, C, [0], clip=clip)[1] for k in range(1, 5)]
    Ws = [np.asarray(W0, float)] + Ws
    for k in range(4):
        step = Ws[k + 1] - Ws[k]
        raw = V[k * C:(k + 1) * C].T @ Z[k * C:(k + 1) * C]   # direction of the unclipped delta
        assert abs(np.linalg.norm(step) / clip - 1.0) < 1e-6
        cos = np.sum(step * raw) / (np.linalg.norm(step) * np.linalg.norm(raw))
        assert abs(cos - 1.0) < 1e-9
    O, _ = packed.inplace_scan_docs(Z, V, W0, eta, C, [0], clip=clip)
    for k in range(4):
        np.testing.assert_allclose(O[k * C:(k + 1) * C], Z[k * C:(k + 1) * C] @ Ws[k].T, rtol=0, atol=1e-12)


def test_linear_documents_per_sequence():
    """Each sequence has its own document starts; every document equals a scan from W0."""
    B, H, T, D, b, eta = 2, 3, 96, 4, 8, 0.4
    K, V, Q = _rand((B, H, T, D), 16, 0.5), _rand((B, H, T, D), 17, 0.5), _rand((B, H, T, D), 18)
    W0 = _rand((B, H, D, D), 19, 0.3)
    starts = [[0, 32], [0, 48, 64]]
    O, W, L = packed.ttt_linear_scan_docs(K, V, Q, W0, eta, b, starts)
    for s in range(B):
        bounds = list(zip(starts[s], starts[s][1:] + [T]))
        for a, e in bounds:
            O_d, W_d, L_d = linear.ttt_linear_scan(K[s:s + 1, :, a:e], V[s:s + 1, :, a:e], Q[s:s + 1, :, a:e],
                                                   W0[s:s + 1], eta, b)
            np.testing.assert_allclose(O[s, :, a:e], O_d[0], rtol=0, atol=1e-12)
            np.testing.assert_allclose(L[s, :, a:e], L_d[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(W[s], W_d[0], rtol=0, atol=1e-12)


def test_short_last_mini_batch_is_the_step_of_its_own_loss():
    """A 29-token document with b = 8 ends in a 5-token mini-batch: from the weight after the
    three full mini-batches it takes W ← W − (η/5)·Kᵀ(KW − V), as a 5-token scan with b = 5."""
    D, b, eta = 4, 8, 0.3
    K, V, Q = _rand((1, 1, 29, D), 20, 0.5), _rand((1, 1, 29, D), 21, 0.5), _rand((1, 1, 29, D), 22)
    W0 = _rand((1, 1, D, D), 23, 0.3)
    O, W, L = packed.ttt_linear_scan_docs(K, V, Q, W0, eta, b, [[0]])
    _, W24, _ = linear.ttt_linear_scan(K[:, :, :24], V[:, :, :24], Q[:, :, :24], W0, eta, b)
    O5, W5, L5 = linear.ttt_linear_scan(K[:, :, 24:], V[:, :, 24:], Q[:, :, 24:], W24, eta, 5)
    np.testing.assert_allclose(W, W5, rtol=0, atol=1e-12)
    np.testing.assert_allclose(O[:, :, 24:], O5, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L[:, :, 24:], L5, rtol=0, atol=1e-12)


def test_rejects_bad_document_starts():
    Z, V, W0 = np.zeros((8, 2)), np.zeros((8, 2)), np.zeros((2, 2))
    for starts in ([], [1], [0, 0], [0, 5, 3], [0, 8]):
        with pytest.raises(ValueError):
            packed.inplace_scan_docs(Z, V, W0, 0.1, 4, starts)


def test_linear_token_weights_per_document():
    """Per-token weights over packed sequences: one document of whole mini-batches equals the
    per-token scan, and the final weight and losses do not depend on the outputs' form."""
    B, H, T, D, b, eta = 1, 2, 32, 4, 8, 0.3
    K, V, Q = _rand((B, H, T, D), 40, 0.5), _rand((B, H, T, D), 41, 0.5), _rand((B, H, T, D), 42)
    W0 = _rand((B, H, D, D), 43, 0.3)
    O, W, L = packed.ttt_linear_scan_docs(K, V, Q, W0, eta, b, [[0]], token_weights=True)
    O_r, W_r, L_r = linear.ttt_linear_scan(K, V, Q, W0, eta, b, token_weights=True)
    for got, want in ((O, O_r), (W, W_r), (L, L_r)):
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    O2, W2, L2 = packed.ttt_linear_scan_docs(K, V, Q, W0, eta, b, [[0, 13]], token_weights=True)
    O3, W3, L3 = packed.ttt_linear_scan_docs(K, V, Q, W0, eta, b, [[0, 13]])
    np.testing.assert_array_equal(W2, W3)
    np.testing.assert_array_equal(L2, L3)
    # The first document's 5-token last mini-batch: the per-token scan with b = 5 from the weight
    # after its first 8 tokens.
    _, W8, _ = linear.ttt_linear_scan(K[:, :, :8], V[:, :, :8], Q[:, :, :8], W0, eta, b)
    O5 = linear.ttt_linear_scan(K[:, :, 8:13], V[:, :, 8:13], Q[:, :, 8:13], W8, eta, 5, token_weights=True)[0]
    np.testing.assert_allclose(O2[:, :, 8:13], O5, rtol=0, atol=1e-12)


def test_layernorm_model_per_document():
    _inner_per_document("linear_ln")


def test_mlp_model_per_document():
    _inner_per_document("mlp")


def _inner_per_document(model):
    """The LayerNorm and MLP models over packed sequences: one document of whole mini-batches is
    the inner scan; every document restarts from the pretrained weights; a short last mini-batch
    is one step of the inner scan with mini-batch n."""
    from oracle import inner
    B, H, T, D, b, eta, eps = 2, 2, 40, 4, 8, 0.3, 1e-3
    K, V, Q = _rand((B, H, T, D), 44, 0.5), _rand((B, H, T, D), 45, 0.5), _rand((B, H, T, D), 46)
    g, be = _rand((H, D), 47) + 1.0, _rand((H, D), 48)
    if model == "mlp":
        W0 = (_rand((B, H, D, 4 * D), 49, 0.5), _rand((B, H, 4 * D, D), 50, 0.5))
        scan = lambda k, v, q, w, bb: inner.ttt_mlp_scan(k, v, q, w[0], w[1], g, be, eta, bb, eps)  # noqa: E731
        weights = lambda r: (r[1], r[2])  # noqa: E731
    else:
        W0 = _rand((B, H, D, D), 49, 0.5)
        scan = lambda k, v, q, w, bb: inner.ttt_linear_ln_scan(k, v, q, w, g, be, eta, bb, eps)  # noqa: E731
        weights = lambda r: r[1]  # noqa: E731
    O, W, L = packed.inner_scan_docs(model, K, V, Q, W0, g, be, eta, b, eps, [[0], [0]])
    ref = scan(K, V, Q, W0, b)
    np.testing.assert_allclose(O, ref[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, ref[-1], rtol=0, atol=1e-12)
    # Sequence 1 as two documents, [0, 24) and [24, 40): 24 = 3 mini-batches, then 16 = 2.
    O, W, L = packed.inner_scan_docs(model, K, V, Q, W0, g, be, eta, b, eps, [[0], [0, 24]])
    sl = lambda x, a, e: x[1:2, :, a:e]  # noqa: E731
    w1 = (W0[0][1:2], W0[1][1:2]) if model == "mlp" else W0[1:2]
    r1 = scan(sl(K, 0, 24), sl(V, 0, 24), sl(Q, 0, 24), w1, b)
    r2 = scan(sl(K, 24, 40), sl(V, 24, 40), sl(Q, 24, 40), w1, b)
    np.testing.assert_allclose(O[1:2, :, :24], r1[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(O[1:2, :, 24:], r2[0], rtol=0, atol=1e-12)
    # A 13-token document with b = 8: one full mini-batch, then one step with mini-batch 5.
    O, W, L = packed.inner_scan_docs(model, K[:, :, :13], V[:, :, :13], Q[:, :, :13], W0, g, be, eta, b, eps,
                                     [[0], [0]])
    full = scan(K[:, :, :8], V[:, :, :8], Q[:, :, :8], W0, b)
    tail = scan(K[:, :, 8:13], V[:, :, 8:13], Q[:, :, 8:13], weights(full), 5)
    np.testing.assert_allclose(O[:, :, 8:13], tail[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(L[:, :, 8:13], tail[-1], rtol=0, atol=1e-12)
    for got, want in zip(W if model == "mlp" else (W,), weights(tail) if model == "mlp" else (weights(tail),)):
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def _target_inputs(T, C, d, f, seed):
    Z, X0 = _rand((T, f), seed), _rand((T, d), seed + 1)
    w, Wt, W0 = _rand((d, 3), seed + 2, 0.6), _rand((d, d), seed + 3, 0.3), _rand((d, f), seed + 4, 0.1)
    return Z, X0, w, Wt, W0


def test_fused_target_one_document_is_the_fused_target_scan():
    """One document: the scan with the targets Conv1D(X0)·Wtarget of the whole sequence (both
    padding modes)."""
    T, C, d, f, eta = 96, 32, 5, 7, 0.05
    Z, X0, w, Wt, W0 = _target_inputs(T, C, d, f, 30)
    for pad_mode in (0, 1):
        O, W = packed.inplace_scan_docs_target(Z, X0, w, Wt, W0, eta, C, [0], pad_mode)
        O_ref, W_ref = inplace.inplace_scan(Z, inplace.target_values(X0, w, Wt, C, pad_mode), W0, eta, C)
        np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-13)
        np.testing.assert_allclose(W, W_ref, rtol=0, atol=1e-13)


def test_fused_target_documents_read_only_their_own_rows():
    for pad_mode in (0, 1):
        _documents_read_only_their_own_rows(pad_mode)


def _documents_read_only_their_own_rows(pad_mode):
    """Documents of 64 (two whole chunks: its last taps sit right before the next document),
    37 and 59 tokens: each document's outputs are those of the same call on that document
    alone, and changing another document's X0 changes none of them."""
    T, C, d, f, eta = 160, 32, 4, 6, 0.08
    Z, X0, w, Wt, W0 = _target_inputs(T, C, d, f, 40)
    starts = [0, 64, 101]
    O, W = packed.inplace_scan_docs_target(Z, X0, w, Wt, W0, eta, C, starts, pad_mode)
    bounds = list(zip(starts, starts[1:] + [T]))
    for a, e in bounds:
        O_doc, W_doc = packed.inplace_scan_docs_target(Z[a:e], X0[a:e], w, Wt, W0, eta, C, [0], pad_mode)
        np.testing.assert_allclose(O[a:e], O_doc, rtol=0, atol=1e-13)
    np.testing.assert_allclose(W, W_doc, rtol=0, atol=1e-13)
    for k, (a, e) in enumerate(bounds):
        X1 = X0.copy()
        X1[a:e] += 5.0
        O1, _ = packed.inplace_scan_docs_target(Z, X1, w, Wt, W0, eta, C, starts, pad_mode)
        for j, (a2, e2) in enumerate(bounds):
            if j != k:
                np.testing.assert_array_equal(O1[a2:e2], O[a2:e2])
        assert not np.allclose(O1[a:e], O[a:e])
