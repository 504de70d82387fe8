"""Oracle of the richer TTT inner models (float64) — test infrastructure only.

Source: "テスト時学習（Test-Time Training）とは" (TTT layers page, arXiv 2407.04620):

* the layer's hidden state is itself a model, and its update rule is one step of
  self-supervised learning on the sequence; the page's two instances are TTT-Linear (a
  linear model) and TTT-MLP (a two-layer MLP).
* the related-work remark: DeltaNet is TTT-Linear with inner mini-batch 1 once its
  LayerNorm and residual connection are removed, so the full TTT-Linear's inner model has
  both.
* the conclusion: TTT-MLP is efficient in FLOPs, but its memory I/O remains a challenge.

Readings taken where the page prints no formula (the plainest ones the rest supports):

* inner model f(x) = x + LN(g(x)): g(x) = x·W for TTT-Linear and g(x) = GELU(x·W1)·W2 for
  TTT-MLP (hidden width 4·D, no biases). LN normalises each token's D values with their mean
  and population variance (ε added under the square root), then scales by γ and shifts by β:
  per-head [D] vectors that belong to the outer model, so the inner step leaves them alone.
* GELU(x) = x·Φ(x), Φ the standard normal distribution function (the erf form).
* the self-supervised loss of mini-batch i is ℓ_i = 1/(2b)·Σ_t ‖f(k_t) − v_t‖², and one
  gradient step moves every inner weight at once, from the weights in effect at the start of
  the mini-batch: θ_{i+1} = θ_i − η·∇ℓ_i(θ_i).
* as for the plain TTT-Linear scan, the b outputs of mini-batch i are o_t = f(q_t; θ_i) and
  the per-token loss is L_t = ‖f(k_t; θ_i) − v_t‖².
* per-token weights (``token_weights=True``, the TTT layer's mini-batch form in which each token
  sees the gradient steps of the tokens before it and its own): output t of mini-batch i uses
  θ_t = θ_i − (η/b)·Σ_{s ≤ t} ∇(½‖f(k_s; θ_i) − v_s‖²), every gradient taken at θ_i, so the
  last token of the mini-batch sees θ_{i+1}; losses and the weight update are unchanged.

The gradients are written out by the chain rule, one layer at a time; the pins check them
against central differences of the loss.
"""

from __future__ import annotations

import numpy as np
from scipy.special import erf

from ._util import f64


def layer_norm(Z, gamma, beta, eps: float):
    """LN over the last axis. Returns (γ·ẑ + β, ẑ, 1/sqrt(σ² + ε))."""
    mu = Z.mean(axis=-1, keepdims=True)
    var = ((Z - mu) ** 2).mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    zhat = (Z - mu) * rstd
    return gamma * zhat + beta, zhat, rstd


def layer_norm_backward(dY, zhat, rstd, gamma):
    """∂/∂Z of a loss whose gradient with respect to LN's output is dY."""
    g = dY * gamma
    return rstd * (g - g.mean(axis=-1, keepdims=True) - zhat * (g * zhat).mean(axis=-1, keepdims=True))


def gelu(x):
    """x·Φ(x)."""
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def gelu_grad(x):
    """d/dx of x·Φ(x) = Φ(x) + x·φ(x)."""
    return 0.5 * (1.0 + erf(x / np.sqrt(2.0))) + x * np.exp(-0.5 * x * x) / np.sqrt(2.0 * np.pi)


def _act(name: str):
    # "identity" exists only so that the pins can compare the MLP with a linear model.
    if name == "gelu":
        return gelu, gelu_grad
    if name == "identity":
        return (lambda x: x), (lambda x: np.ones_like(x))
    raise ValueError(name)


def _per_head(p, B: int, H: int, D: int):
    """γ or β given per head [H, D] → [B·H, 1, D]."""
    p = f64(p).reshape(H, D)
    return np.broadcast_to(p[None], (B, H, D)).reshape(B * H, 1, D)


def _check(Kd, b):
    if Kd.shape[2] % b != 0:
        raise ValueError("T must be a multiple of the inner mini-batch b")


def ttt_linear_ln_scan(K, V, Q, W0, gamma, beta, eta: float, b: int, eps: float, token_weights: bool = False):
    """TTT-Linear with LayerNorm and residual over every (sequence, head) of [B, H, T, D]
    inputs; W0 [B, H, D, D], gamma and beta [H, D].

    Returns (O [B,H,T,D] or None when Q is None, W_final [B,H,D,D], loss [B,H,T]).
    """
    Kd, Vd = f64(K), f64(V)
    B, H, T, D = Kd.shape
    _check(Kd, b)
    Kf, Vf = Kd.reshape(B * H, T, D), Vd.reshape(B * H, T, D)
    Qf = None if Q is None else f64(Q).reshape(B * H, T, D)
    gam, bet = _per_head(gamma, B, H, D), _per_head(beta, B, H, D)
    W = f64(W0).reshape(B * H, D, D).copy()
    O = None if Qf is None else np.empty((B * H, T, D))
    loss = np.empty((B * H, T))
    for i in range(T // b):
        s = slice(i * b, (i + 1) * b)
        Ki, Vi = Kf[:, s], Vf[:, s]
        if Qf is not None and not token_weights:
            O[:, s] = Qf[:, s] + layer_norm(Qf[:, s] @ W, gam, bet, eps)[0]  # f(q; W_i)
        Y, zhat, rstd = layer_norm(Ki @ W, gam, bet, eps)
        E = Ki + Y - Vi                                    # f(k) − v
        loss[:, s] = np.sum(E * E, axis=2)
        dZ = layer_norm_backward(E, zhat, rstd, gam)       # ∂(½‖f(k) − v‖²)/∂(k·W)
        if Qf is not None and token_weights:
            for j in range(b):                             # token j sees the steps of tokens 0..j
                Wt = W - (eta / b) * (np.swapaxes(Ki[:, :j + 1], 1, 2) @ dZ[:, :j + 1])
                t = i * b + j
                O[:, t:t + 1] = Qf[:, t:t + 1] + layer_norm(Qf[:, t:t + 1] @ Wt, gam, bet, eps)[0]
        W = W - (eta / b) * (np.swapaxes(Ki, 1, 2) @ dZ)   # one gradient step on ℓ_i
    O = None if O is None else O.reshape(B, H, T, D)
    return O, W.reshape(B, H, D, D), loss.reshape(B, H, T)


def ttt_mlp_scan(K, V, Q, W1_0, W2_0, gamma, beta, eta: float, b: int, eps: float, activation: str = "gelu",
                 token_weights: bool = False):
    """TTT-MLP over every (sequence, head) of [B, H, T, D] inputs; W1_0 [B, H, D, Dh],
    W2_0 [B, H, Dh, D], gamma and beta [H, D].

    Returns (O or None, W1_final, W2_final, loss [B,H,T]).
    """
    act, act_grad = _act(activation)
    Kd, Vd = f64(K), f64(V)
    B, H, T, D = Kd.shape
    _check(Kd, b)
    Dh = f64(W1_0).shape[-1]
    Kf, Vf = Kd.reshape(B * H, T, D), Vd.reshape(B * H, T, D)
    Qf = None if Q is None else f64(Q).reshape(B * H, T, D)
    gam, bet = _per_head(gamma, B, H, D), _per_head(beta, B, H, D)
    W1 = f64(W1_0).reshape(B * H, D, Dh).copy()
    W2 = f64(W2_0).reshape(B * H, Dh, D).copy()
    O = None if Qf is None else np.empty((B * H, T, D))
    loss = np.empty((B * H, T))
    for i in range(T // b):
        s = slice(i * b, (i + 1) * b)
        Ki, Vi = Kf[:, s], Vf[:, s]
        if Qf is not None and not token_weights:
            O[:, s] = Qf[:, s] + layer_norm(act(Qf[:, s] @ W1) @ W2, gam, bet, eps)[0]
        Hpre = Ki @ W1                                     # hidden pre-activation [b, Dh]
        A = act(Hpre)
        Y, zhat, rstd = layer_norm(A @ W2, gam, bet, eps)
        E = Ki + Y - Vi
        loss[:, s] = np.sum(E * E, axis=2)
        dZ = layer_norm_backward(E, zhat, rstd, gam)       # at the second layer's output
        dW2 = np.swapaxes(A, 1, 2) @ dZ
        dH = (dZ @ np.swapaxes(W2, 1, 2)) * act_grad(Hpre)  # back through W2 and the activation
        dW1 = np.swapaxes(Ki, 1, 2) @ dH
        if Qf is not None and token_weights:
            for j in range(b):                             # token j sees the steps of tokens 0..j
                W1t = W1 - (eta / b) * (np.swapaxes(Ki[:, :j + 1], 1, 2) @ dH[:, :j + 1])
                W2t = W2 - (eta / b) * (np.swapaxes(A[:, :j + 1], 1, 2) @ dZ[:, :j + 1])
                t = i * b + j
                O[:, t:t + 1] = Qf[:, t:t + 1] + layer_norm(act(Qf[:, t:t + 1] @ W1t) @ W2t, gam, bet, eps)[0]
        W1 = W1 - (eta / b) * dW1
        W2 = W2 - (eta / b) * dW2
    O = None if O is None else O.reshape(B, H, T, D)
    return O, W1.reshape(B, H, D, Dh), W2.reshape(B, H, Dh, D), loss.reshape(B, H, T)


def inner_loss_ln(K_i, V_i, W, gamma, beta, eps: float) -> float:
    """ℓ(W) = 1/(2b)·Σ_t ‖k_t + LN(k_t·W) − v_t‖² for one mini-batch [b, D] (gradient pins)."""
    K_i, V_i = f64(K_i), f64(V_i)
    E = K_i + layer_norm(K_i @ f64(W), f64(gamma), f64(beta), eps)[0] - V_i
    return float(np.sum(E * E) / (2.0 * K_i.shape[0]))


def inner_loss_mlp(K_i, V_i, W1, W2, gamma, beta, eps: float) -> float:
    """ℓ(W1, W2) = 1/(2b)·Σ_t ‖k_t + LN(GELU(k_t·W1)·W2) − v_t‖² for one mini-batch."""
    K_i, V_i = f64(K_i), f64(V_i)
    E = K_i + layer_norm(gelu(K_i @ f64(W1)) @ f64(W2), f64(gamma), f64(beta), eps)[0] - V_i
    return float(np.sum(E * E) / (2.0 * K_i.shape[0]))
