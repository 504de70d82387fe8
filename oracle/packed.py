"""Oracle of packed sequences: per-document resets and update-norm clipping (float64) — test
infrastructure only.

Source: "In-Place Test-Time Training" (blog summary of arXiv 2604.06169), §6 "context
parallelism" and the implementation notes that follow it:

* when an independent document ends, the fast weight goes back to its pretrained state, so
  nothing leaks from one document into the next;
* the Frobenius norm of the update delta is clipped (the page's threshold reads 1e-5), so a
  long run of updates cannot flood the weight.

The TTT layers page gives the same boundary for TTT-Linear: the recurrent state is the inner
model's weight, restarted for a new sequence.

Readings taken where the pages leave it open (a CUDA path must apply the same ones):

* a packed sequence is documents laid end to end; ``doc_starts`` lists each document's first
  token (the first is 0). Every document is scanned as if alone: the weight starts from W0,
  chunks (In-Place) or inner mini-batches (TTT-Linear) are counted from the document's first
  token, and a document's last chunk or mini-batch may be shorter;
* a shorter last TTT-Linear mini-batch of b' tokens takes the gradient step of its own loss
  1/(2b')·‖K·W − V‖², i.e. W ← W − (η/b')·Kᵀ(K·W − V);
* clipping acts on each chunk's delta ΔW_c = η·V̂_cᵀ·Z_c on its own: if ‖ΔW_c‖_F exceeds the
  threshold, ΔW_c is scaled to that norm; the threshold is a parameter (None: no clipping).
* with the target made inside the scan (V̂ = Conv1D(X0)·Wtarget, §4), each document's targets
  are its own: the future taps stop at the document's end as they stop at the sequence's end
  (and, in pad mode 0, at the end of each of its chunks, counted from its first token), so a
  document's targets read nothing of the next document.
"""

from __future__ import annotations

import numpy as np

from . import inner, inplace
from ._util import f64


def _documents(doc_starts, T: int):
    starts = [int(s) for s in doc_starts]
    if not starts or starts[0] != 0 or any(b <= a for a, b in zip(starts, starts[1:])) or starts[-1] >= T:
        raise ValueError("doc_starts must start at 0, increase strictly and lie below T")
    return list(zip(starts, starts[1:] + [T]))


def clip_delta(dW, clip):
    """ΔW scaled to Frobenius norm ``clip`` when it is larger (unchanged otherwise)."""
    if clip is None:
        return dW
    n = float(np.sqrt(np.sum(dW * dW)))
    return dW * (clip / n) if n > clip else dW


def inplace_scan_docs(Z, Vhat, W0, eta: float, C: int, doc_starts, clip=None):
    """Apply-then-update over each document of a packed sequence, W reset to W0 at each start.

    Z [T, f], Vhat [T, d], W0 [d, f]. Returns (O [T, d], W after the last document [d, f])."""
    Zd, Vd, W0d = f64(Z), f64(Vhat), f64(W0)
    T = Zd.shape[0]
    O = np.empty((T, W0d.shape[0]))
    W = W0d
    for a, e in _documents(doc_starts, T):
        W = W0d.copy()                                   # document boundary: pretrained weight
        for c0 in range(a, e, C):
            rows = slice(c0, min(c0 + C, e))
            O[rows] = Zd[rows] @ W.T                     # apply first
            W = W + clip_delta(eta * (Vd[rows].T @ Zd[rows]), clip)   # then update
    return O, W


def inplace_scan_docs_target(Z, X0, convw, Wtarget, W0, eta: float, C: int, doc_starts, pad_mode: int = 0,
                             clip=None):
    """inplace_scan_docs with each document's targets V̂ = Conv1D(X0)·Wtarget computed from
    that document alone (X0 [T, d], convw [d, taps], Wtarget [d, d])."""
    X = f64(X0)
    T = X.shape[0]
    V = np.empty((T, f64(Wtarget).shape[1]))
    for a, e in _documents(doc_starts, T):
        V[a:e] = inplace.target_values(X[a:e], convw, Wtarget, C, pad_mode)
    return inplace_scan_docs(Z, V, W0, eta, C, doc_starts, clip)


def ttt_linear_scan_docs(K, V, Q, W0, eta: float, b: int, doc_starts, token_weights: bool = False):
    """TTT-Linear over packed sequences; ``doc_starts[s]`` lists sequence s's document starts.

    K, V, Q [B, H, T, D] (Q may be None), W0 [B, H, D, D]. Returns (O or None, W after each
    sequence's last document [B, H, D, D], loss [B, H, T])."""
    Kd, Vd = f64(K), f64(V)
    Qd = None if Q is None else f64(Q)
    W0d = f64(W0)
    B, H, T, D = Kd.shape
    O = None if Qd is None else np.empty((B, H, T, D))
    loss = np.empty((B, H, T))
    Wout = np.empty((B, H, D, D))
    for s in range(B):
        docs = _documents(doc_starts[s], T)
        for h in range(H):
            W = W0d[s, h]
            for a, e in docs:
                W = W0d[s, h].copy()                     # document boundary: W ← W0
                for i0 in range(a, e, b):
                    r = slice(i0, min(i0 + b, e))
                    n = r.stop - r.start                 # b, or fewer for the last mini-batch
                    if Qd is not None and not token_weights:
                        O[s, h, r] = Qd[s, h, r] @ W     # outputs with the mini-batch's start W
                    R = Kd[s, h, r] @ W - Vd[s, h, r]
                    loss[s, h, r] = np.sum(R * R, axis=1)
                    if Qd is not None and token_weights:  # token j sees the steps of tokens 0..j
                        for j in range(n):
                            Wt = W - (eta / n) * (Kd[s, h, i0:i0 + j + 1].T @ R[:j + 1])
                            O[s, h, i0 + j] = Qd[s, h, i0 + j] @ Wt
                    W = W - (eta / n) * (Kd[s, h, r].T @ R)
            Wout[s, h] = W
    return O, Wout, loss


def inner_scan_docs(model: str, K, V, Q, W0, gamma, beta, eta: float, b: int, eps: float, doc_starts,
                    token_weights: bool = False):
    """The richer inner models (``model`` "linear_ln" or "mlp", oracle.inner) over packed
    sequences, by the same reading: every document of sequence s (``doc_starts[s]``) restarts
    every head from W0 (LayerNorm TTT-Linear: [B,H,D,D]; TTT-MLP: the pair (W1 [B,H,D,Dh],
    W2 [B,H,Dh,D])), mini-batches count from its first token, and a last mini-batch of n < b
    tokens takes the step of its own loss (one step of the inner scan with mini-batch n).

    Returns (O or None, the weights after each sequence's last document, loss [B, H, T])."""
    Kd, Vd = f64(K), f64(V)
    Qd = None if Q is None else f64(Q)
    B, H, T, D = Kd.shape
    mlp = model == "mlp"
    W0s = (f64(W0[0]), f64(W0[1])) if mlp else f64(W0)
    O = None if Qd is None else np.empty((B, H, T, D))
    loss = np.empty((B, H, T))
    Wout = ([np.empty_like(W0s[0]), np.empty_like(W0s[1])] if mlp else np.empty_like(W0s))
    for s in range(B):
        docs = _documents(doc_starts[s], T)
        for h in range(H):
            g, be = f64(gamma)[h:h + 1], f64(beta)[h:h + 1]
            for a, e in docs:
                W = (W0s[0][s, h], W0s[1][s, h]) if mlp else W0s[s, h]   # document boundary: θ ← θ0
                for i0 in range(a, e, b):
                    r = slice(i0, min(i0 + b, e))
                    n = r.stop - r.start
                    one = lambda x: None if x is None else x[s, h, r][None, None]  # noqa: E731
                    if mlp:
                        o, W1n, W2n, l = inner.ttt_mlp_scan(one(Kd), one(Vd), one(Qd), W[0][None, None], W[1][None, None],
                                                            g, be, eta, n, eps, token_weights=token_weights)
                        W = (W1n[0, 0], W2n[0, 0])
                    else:
                        o, Wn, l = inner.ttt_linear_ln_scan(one(Kd), one(Vd), one(Qd), W[None, None], g, be, eta, n, eps,
                                                            token_weights=token_weights)
                        W = Wn[0, 0]
                    if O is not None:
                        O[s, h, r] = o[0, 0]
                    loss[s, h, r] = l[0, 0]
            if mlp:
                Wout[0][s, h], Wout[1][s, h] = W
            else:
                Wout[s, h] = W
    return O, (tuple(Wout) if mlp else Wout), loss
