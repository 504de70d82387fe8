"""Oracle of the In-Place TTT chunk scan (float64) — test infrastructure only.

Source: "In-Place Test-Time Training" (blog summary of arXiv 2604.06169, Feng et al.).

* §2 "Wdown as fast weight": the gated MLP's final projection Wdown [d_model x d_ff] is
  the fast weight; the block output for intermediate activations Z is O = Z Wdownᵀ and the
  simplified update is ΔWdown = η·V̂ᵀ·Z.
* §3 "apply first, update later": the sequence is split into chunks; each chunk's output
  is produced with the current Wdown, then Wdown is updated from that same chunk; chunk 0
  uses the pretrained Wdown.
* §4 "predict the next token": the target is V̂ = Conv1D(X0)·Wtarget.
* §6 "context parallelism": the per-chunk deltas are additive, so W_c = W0 + Σ_{j<c} ΔW_j
  (exclusive prefix sum); chunk-boundary padding stops the target convolution from
  reading another chunk's future tokens.

Reading taken where the page is silent: the final W includes the last chunk's update; the
convolution taps sit at offsets 0, +1, +2 (depthwise) and are zero past the end of the
token's chunk (pad mode 0) or past the sequence end only (pad mode 1); Wtarget is
[in, out] with V̂[t, j] = Σ_i conv[t, i]·Wtarget[i, j].
"""

from __future__ import annotations

import numpy as np

from ._util import f64


def inplace_scan(Z, Vhat, W0, eta: float, C: int):
    """Sequential apply-then-update scan.

    Z [T, f], Vhat [T, d], W0 [d, f]; T must be a multiple of the chunk C.
    Returns (O [T, d], W_final [d, f]) in float64. Chunks are widened to float64 one at a
    time, so the full-size inputs never exist in float64 at once.
    """
    T = Z.shape[0]
    if T % C != 0:
        raise ValueError("T must be a multiple of the chunk size")
    W = f64(W0).copy()
    O = np.empty((T, W.shape[0]), dtype=np.float64)
    for c in range(T // C):
        rows = slice(c * C, (c + 1) * C)
        Zc = f64(Z[rows])
        Vc = f64(Vhat[rows])
        O[rows] = Zc @ W.T                 # apply with W before this chunk's update (§3)
        W = W + eta * (Vc.T @ Zc)          # ΔW = η·V̂ᵀ·Z (§2)
    return O, W


def inplace_scan_prefix(Z, Vhat, W0, eta: float, C: int):
    """Context-parallel form (§6): all ΔW_j first, exclusive prefix sum, then every output."""
    Zd, Vd, W0d = f64(Z), f64(Vhat), f64(W0)
    T = Zd.shape[0]
    n = T // C
    deltas = [eta * (Vd[j * C:(j + 1) * C].T @ Zd[j * C:(j + 1) * C]) for j in range(n)]
    prefix = [np.zeros_like(W0d)]
    for j in range(n):
        prefix.append(prefix[-1] + deltas[j])
    O = np.empty((T, W0d.shape[0]))
    for c in range(n):
        O[c * C:(c + 1) * C] = Zd[c * C:(c + 1) * C] @ (W0d + prefix[c]).T
    return O, W0d + prefix[n]


def target_conv(X0, convw, C: int, pad_mode: int = 0):
    """Depthwise future-tap convolution conv[t, i] = Σ_k w[i, k]·X0[t + k, i], k = 0..taps-1.

    A tap that would read past the boundary contributes zero; the boundary is the end of
    token t's chunk (pad_mode 0) or the end of the sequence (pad_mode 1), and never lies past
    the sequence's end (a shorter last chunk has no tokens beyond T).
    """
    X = f64(X0)
    w = f64(convw)
    T, d = X.shape
    taps = w.shape[1]
    t = np.arange(T)
    end = np.minimum((t // C + 1) * C, T) if pad_mode == 0 else np.full(T, T)
    out = np.zeros((T, d))
    for k in range(taps):
        src = t + k
        ok = src < end
        out[ok] += X[src[ok]] * w[:, k]
    return out


def target_values(X0, convw, Wtarget, C: int, pad_mode: int = 0, cols=None):
    """LM-aligned target V̂ = Conv1D(X0)·Wtarget (§4); ``cols`` restricts the output columns."""
    conv = target_conv(X0, convw, C, pad_mode)
    Wt = f64(Wtarget)
    if cols is not None:
        Wt = Wt[:, cols]
    return conv @ Wt


def inplace_scan_rows(Z, Vhat_cols, W0_rows, eta: float, C: int):
    """The scan restricted to a subset of Wdown's rows.

    Row i of W only ever receives η·V̂[:, i]ᵀ·Z, so the rows evolve independently: passing
    V̂'s columns for rows R and W0[R] yields exactly O[:, R] and W_final[R]. This is how the
    full-size workloads are checked on sampled outputs.
    """
    return inplace_scan(Z, Vhat_cols, W0_rows, eta, C)
