"""Oracle of the SR-TTT residual-cache read path and α fusion (float64) — test infrastructure only.

Source: "SR-TTT: Surprisal-Aware Residual Test-Time Training" (technical summary), §2.1,
"Residual Cache" and "Alpha Fusion":

* the cache holds the keys and values of the tokens the surprisal filter routed, as a
  fixed-capacity memory track that runs beside the fast weight;
* the layer's output is the TTT output plus the cache's attention output weighted by a
  learned gate vector α (Output = TTT(x) + α·CacheAttention(x));
* α is parameterised by a direct clamp rather than a sigmoid, so the gate can open without
  its gradient dying.

Readings taken where the page leaves the computation open (a CUDA read path must apply the
same ones):

* keys, values and queries are the scan's own K, V and Q of the same (sequence, head); the
  cache of a (sequence, head) is the first min(routed, capacity) triples (sequence, head, t)
  the gate stored, t counted from the last reset;
* causality: a token's routing is decided once its whole 64-token gate chunk has been seen,
  so a query at token t reads only the entries whose gate chunk lies before t's
  (⌊t'/64⌋ < ⌊t/64⌋); a query with no such entry has a zero attention output;
* the attention is the standard scaled dot product, one softmax per query over its visible
  entries: A_t = Σ_j softmax_j(q_t·k_j / √D)·v_j;
* α is one vector of D channels per head, clamped elementwise to [0, 1]:
  O_t = O_TTT,t + clamp(α, 0, 1) ⊙ A_t.

This covers one call from a reset (the cached keys and values are gathered from the same
K and V); a streaming read path would keep copies of the cached rows across calls.
"""

from __future__ import annotations

import numpy as np

from ._util import f64


def cached_tokens(entries, counts, bi: int, hi: int) -> np.ndarray:
    """Token indices held by the cache of (sequence bi, head hi), in stored order."""
    E = np.asarray(entries)
    n = min(int(np.asarray(counts)[bi, hi, 0]), E.shape[2])
    rows = E[bi, hi, :n]
    if n and not (np.all(rows[:, 0] == bi) and np.all(rows[:, 1] == hi)):
        raise ValueError("cache entries name another (sequence, head)")
    return rows[:, 2].astype(np.int64)


def cache_attention(Q, K, V, entries, counts, gate_chunk: int = 64) -> np.ndarray:
    """A [B, H, T, D]: each query's softmax attention over the cache entries it may see."""
    Qd, Kd, Vd = f64(Q), f64(K), f64(V)
    B, H, T, D = Qd.shape
    scale = 1.0 / np.sqrt(D)
    A = np.zeros((B, H, T, D))
    for bi in range(B):
        for hi in range(H):
            ts = cached_tokens(entries, counts, bi, hi)
            kc, vc, gc = Kd[bi, hi, ts], Vd[bi, hi, ts], ts // gate_chunk
            for t in range(T):
                visible = gc < t // gate_chunk
                if not visible.any():
                    continue
                s = (kc[visible] @ Qd[bi, hi, t]) * scale
                w = np.exp(s - s.max())
                A[bi, hi, t] = (w / w.sum()) @ vc[visible]
    return A


def alpha_fusion(O_ttt, A, alpha) -> np.ndarray:
    """O = O_TTT + clamp(α, 0, 1) ⊙ A, with α [H, D] broadcast over sequences and tokens."""
    a = np.clip(f64(alpha), 0.0, 1.0)
    return f64(O_ttt) + a[None, :, None, :] * f64(A)
