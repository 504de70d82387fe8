"""Oracle of the TTT-Linear mini-batch gradient scan (float64) — test infrastructure only.

Source: "テスト時学習（Test-Time Training）とは" (TTT layers page, arXiv 2407.04620):

* the layer's recurrent state is the weight W of an inner model, and the update rule is
  one step of self-supervised learning on the sequence; TTT-Linear is the instance with a
  linear inner model.
* the related-work remark: DeltaNet is TTT-Linear with inner mini-batch 1 and without
  LayerNorm and the residual connection.

Reading taken where the page prints no formula: the self-supervised loss of mini-batch i
is ℓ_i(W) = 1/(2b)·‖K_i·W − V_i‖²_F, so one gradient step is
W ← W − (η/b)·K_iᵀ(K_i·W − V_i); the b outputs of mini-batch i all use the W in effect at
its start (O_i = Q_i·W_i); there is no LayerNorm or residual inside the inner model; the
per-token loss (SR-TTT §2.1, inner-loop forward pass) is L_t = ‖k_t·W_i − v_t‖².

Per-token weights (``token_weights=True``; the same page: with mini-batch 1 the rule is the
delta rule, in which each token trains before the next is read): output t of mini-batch i uses
W_t = W_i − (η/b)·Σ_{s ≤ t} k_sᵀ(k_s·W_i − v_s), the gradients of the mini-batch's tokens up
to t, all at W_i; the last token sees W_{i+1}. Losses and the update are unchanged.
"""

from __future__ import annotations

import numpy as np

from ._util import f64


def ttt_linear_scan(K, V, Q, W0, eta: float, b: int, token_weights: bool = False):
    """Scan every (sequence, head) of [B, H, T, D] inputs.

    Returns (O [B,H,T,D] or None when Q is None, W_final [B,H,D,D], loss [B,H,T]).
    Heads are independent problems and are stacked into one batched matmul per
    mini-batch; within a head the steps run in order.
    """
    Kd, Vd = f64(K), f64(V)
    Qd = None if Q is None else f64(Q)
    B, H, T, D = Kd.shape
    if T % b != 0:
        raise ValueError("T must be a multiple of the inner mini-batch b")
    W = f64(W0).reshape(B * H, D, D).copy()
    Kf, Vf = Kd.reshape(B * H, T, D), Vd.reshape(B * H, T, D)
    Qf = None if Qd is None else Qd.reshape(B * H, T, D)
    O = None if Qf is None else np.empty((B * H, T, D))
    loss = np.empty((B * H, T))
    for i in range(T // b):
        s = slice(i * b, (i + 1) * b)
        Ki, Vi = Kf[:, s], Vf[:, s]
        if Qf is not None and not token_weights:
            O[:, s] = Qf[:, s] @ W                       # output with W_i (start of mini-batch)
        R = Ki @ W - Vi                                  # residual of the inner model
        if Qf is not None and token_weights:
            for j in range(b):                           # token j sees the steps of tokens 0..j
                t = i * b + j
                O[:, t:t + 1] = Qf[:, t:t + 1] @ (W - (eta / b) * (np.swapaxes(Ki[:, :j + 1], 1, 2) @ R[:, :j + 1]))
        loss[:, s] = np.sum(R * R, axis=2)               # L_t = ‖k_t W_i − v_t‖²
        W = W - (eta / b) * (np.swapaxes(Ki, 1, 2) @ R)  # one gradient step on ℓ_i
    O = None if O is None else O.reshape(B, H, T, D)
    return O, W.reshape(B, H, D, D), loss.reshape(B, H, T)


def inner_loss(K_i, V_i, W) -> float:
    """ℓ(W) = 1/(2b)·‖K_i·W − V_i‖²_F for one mini-batch (used by the gradient pin)."""
    K_i, V_i, W = f64(K_i), f64(V_i), f64(W)
    R = K_i @ W - V_i
    return float(np.sum(R * R) / (2.0 * K_i.shape[0]))
