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
