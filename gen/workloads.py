"""The five synthetic fast-weight workloads and their scaled-down parity variants.

Only numbers are drawn here; the fast-weight method itself (apply, update, gradient
step, gate) lives elsewhere. Shapes and distributions follow the In-Place TTT page
(gated-MLP intermediate Z, Wdown of shape d_model x d_ff, chunks of 512-1024 tokens,
Qwen3-4B-class widths 2560/9728), the TTT-layers page (TTT-Linear with 64-wide
heads and inner mini-batches) and the SR-TTT page (needle tokens inside a haystack).

Every tensor is drawn by :func:`gen.rng.normal` under the workload's seed and a fixed
name, then rounded (round-to-nearest-even) to its storage type.
"""

from __future__ import annotations

from dataclasses import dataclass, replace

import torch

from . import rng


@dataclass(frozen=True)
class InplaceSpec:
    """In-Place TTT scan over one sequence: Z[T,f], V̂[T,d], Wdown[d,f]."""

    name: str
    T: int
    C: int
    d: int          # d_model (rows of Wdown)
    f: int          # d_ff (columns of Wdown)
    eta: float
    dtype: str      # "f32" or "bf16" storage of Z, V̂ (or X0) and O
    target: bool = False       # V̂ produced from X0 by conv + Wtarget inside the scan
    conv_pad_mode: int = 0     # 0: zero past each chunk end, 1: past the sequence end only
    seed: int = 1000

    @property
    def flops(self) -> float:
        f = 4.0 * self.T * self.d * self.f
        if self.target:
            f += 2.0 * self.T * self.d * self.d
        return f


@dataclass(frozen=True)
class LinearSpec:
    """TTT-Linear mini-batch gradient scan over B sequences x H heads of width 64."""

    name: str
    B: int
    H: int
    T: int
    b: int
    eta: float
    with_queries: bool = True
    needle_frac: float = 0.0
    needle_scale: float = 8.0
    gate: bool = False
    seed: int = 1000
    D: int = 64

    @property
    def flops(self) -> float:
        per = 6.0 if self.with_queries else 4.0
        return per * self.D * self.D * self.T * self.B * self.H


@dataclass(frozen=True)
class InnerSpec:
    """TTT-Linear with LayerNorm and residual ("linear_ln") or TTT-MLP ("mlp") over B sequences x
    H heads of width 64, inner mini-batch b."""

    name: str
    model: str
    B: int
    H: int
    T: int
    b: int = 16
    eta: float = 0.1
    eps: float = 1e-6
    with_queries: bool = True
    seed: int = 1000
    D: int = 64
    hidden: int = 256
    token_weights: bool = False   # outputs with per-token weights within the mini-batch

    @property
    def flops(self) -> float:
        """Products per (token, head) (the per-token form's extra products are not counted): LayerNorm TTT-Linear k·W, q·W and Kᵀ·dZ (2·D² each);
        TTT-MLP two layers forward for keys and queries and three gradient products (2·D·Dh each)."""
        if self.model == "linear_ln":
            per = (6.0 if self.with_queries else 4.0) * self.D * self.D
        else:
            per = (14.0 if self.with_queries else 10.0) * self.D * self.hidden
        return per * self.T * self.B * self.H


# The five workloads, by what they are.
INPLACE_FP32 = InplaceSpec("inplace_fp32_T2048_C512_d256_f512", T=2048, C=512, d=256, f=512,
                           eta=0.01, dtype="f32", seed=1001)
LINEAR_GD = LinearSpec("ttt_linear_B8_H12_T2048_b16", B=8, H=12, T=2048, b=16, eta=1.0, seed=1002)
INPLACE_4B = InplaceSpec("inplace_bf16_T32768_C1024_d2560_f9728", T=32768, C=1024, d=2560, f=9728,
                         eta=1e-3, dtype="bf16", seed=1003)
INPLACE_128K_TARGET = InplaceSpec("inplace_bf16_target_T131072_C1024_d2560_f9728", T=131072, C=1024,
                                  d=2560, f=9728, eta=1e-3, dtype="bf16", target=True, seed=1004)
SR_TTT_GATE = LinearSpec("srttt_gate_B4_H16_T8192_b16", B=4, H=16, T=8192, b=16, eta=1.0,
                         with_queries=False, needle_frac=0.01, gate=True, seed=1005)

WORKLOADS = {w.name: w for w in (INPLACE_FP32, LINEAR_GD, INPLACE_4B, INPLACE_128K_TARGET, SR_TTT_GATE)}

# The richer inner models at the TTT-Linear workload's shapes (the TTT layers page's two
# instances, with LayerNorm and residual).
LINEAR_LN = InnerSpec("ttt_linear_ln_B8_H12_T2048_b16", model="linear_ln", B=8, H=12, T=2048, seed=1007)
MLP = InnerSpec("ttt_mlp_B8_H12_T2048_b16", model="mlp", B=8, H=12, T=2048, seed=1008)
LINEAR_LN_TW = InnerSpec("ttt_linear_ln_B8_H12_T2048_b16_token_weights", model="linear_ln", B=8, H=12, T=2048,
                         seed=1007, token_weights=True)
MLP_TW = InnerSpec("ttt_mlp_B8_H12_T2048_b16_token_weights", model="mlp", B=8, H=12, T=2048, seed=1008,
                   token_weights=True)
INNER_WORKLOADS = {w.name: w for w in (LINEAR_LN, MLP, LINEAR_LN_TW, MLP_TW)}


def document_starts(T: int, n_docs: int, seed: int, min_len: int = 64) -> list[int]:
    """First tokens of ``n_docs`` documents packed end to end in T tokens (0 first): the n_docs − 1
    interior boundaries are drawn uniformly without replacement from the positions that leave
    every document at least ``min_len`` tokens (a seeded draw; lengths then vary widely and
    almost never fall on chunk boundaries, like packed pretraining text)."""
    g = torch.Generator().manual_seed(seed)
    cuts = set()
    while len(cuts) < n_docs - 1:
        c = int(torch.randint(min_len, T - min_len + 1, (1,), generator=g))
        if all(abs(c - o) >= min_len for o in cuts):
            cuts.add(c)
    return [0] + sorted(cuts)


def scaled(spec, **changes):
    """A variant of ``spec`` with some sizes changed (parity cases at oracle-friendly sizes)."""
    return replace(spec, **changes)


# ----------------------------------------------------------------------------------------------
# In-Place inputs
# ----------------------------------------------------------------------------------------------

def _silu_times(a: torch.Tensor, b: torch.Tensor) -> torch.Tensor:
    """Gated-MLP intermediate silu(a) * b, elementwise in the dtype of ``a``."""
    return a * torch.sigmoid(a) * b


def inplace_inputs(spec: InplaceSpec, device="cpu") -> dict:
    """Draw the inputs of an In-Place scan.

    Returns a dict with ``Z`` [T,f], ``W0`` [d,f] fp32 and either ``Vhat`` [T,d] or, for the
    fused-target workloads, ``X0`` [T,d] (bf16), ``convw`` [d,3] fp32 and ``Wtarget`` [d,d] bf16.
    The fp32 workload draws Z = silu(a)*b from a, b ~ N(0,1) in float64; the bf16 workloads
    compute Z = silu(X Wg) * (X Wu) in fp32 (X ~ N(0,1), Wg, Wu ~ N(0, 0.02^2)) and round it.
    """
    s, T, d, f = spec.seed, spec.T, spec.d, spec.f
    out = {"eta": spec.eta}
    out["W0"] = (0.02 * rng.normal("W0", (d, f), s, device)).to(torch.float32)
    if spec.dtype == "f32":
        a = rng.normal("a", (T, f), s, device)
        b = rng.normal("b", (T, f), s, device)
        out["Z"] = _silu_times(a, b).to(torch.float32)
        out["Vhat"] = rng.normal("Vhat", (T, d), s, device).to(torch.float32)
        return out
    out["Z"] = mlp_intermediate(spec, device)
    if spec.target:
        out["X0"] = rng.normal("X0", (T, d), s, device).to(torch.bfloat16)
        out["convw"] = (rng.normal("convw", (d, 3), s, device) * (1.0 / 3.0) ** 0.5).to(torch.float32)
        out["Wtarget"] = (0.02 * rng.normal("Wtarget", (d, d), s, device)).to(torch.bfloat16)
    else:
        out["Vhat"] = rng.normal("Vhat", (T, d), s, device).to(torch.bfloat16)
    return out


def mlp_intermediate(spec: InplaceSpec, device="cpu", rows_per_block: int = 4096) -> torch.Tensor:
    """Z = silu(X Wg) * (X Wu) in fp32, rounded to bf16, drawn block by block of rows."""
    s, T, d, f = spec.seed, spec.T, spec.d, spec.f
    Wg = (0.02 * rng.normal("Wg", (d, f), s, device)).to(torch.float32)
    Wu = (0.02 * rng.normal("Wu", (d, f), s, device)).to(torch.float32)
    Z = torch.empty((T, f), dtype=torch.bfloat16, device=device)
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        key = (s ^ rng.fnv1a64("X")) & ((1 << 64) - 1)
        for r0 in range(0, T, rows_per_block):
            r1 = min(T, r0 + rows_per_block)
            X = _normal_rows(key, r0, r1, d, device).to(torch.float32)
            Z[r0:r1] = _silu_times(X @ Wg, X @ Wu).to(torch.bfloat16)
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    return Z


def _normal_rows(key: int, r0: int, r1: int, width: int, device) -> torch.Tensor:
    """Rows [r0, r1) of the normal tensor whose element i uses counters 2i and 2i+1."""
    import math
    idx = torch.arange(r0 * width, r1 * width, dtype=torch.int64, device=device)
    u1 = rng._uniform53(rng.splitmix64(key, 2 * idx), open_zero=True)
    u2 = rng._uniform53(rng.splitmix64(key, 2 * idx + 1), open_zero=False)
    n = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)
    return n.reshape(r1 - r0, width)


# ----------------------------------------------------------------------------------------------
# TTT-Linear / SR-TTT inputs
# ----------------------------------------------------------------------------------------------

def needle_positions(spec: LinearSpec, batch_index: int) -> list[int]:
    """Needle token positions of one sequence: round(frac*T) distinct, the same for all heads."""
    count = int(round(spec.needle_frac * spec.T))
    return rng.distinct_positions(f"needles/{batch_index}", count, spec.T, spec.seed)


def linear_inputs(spec: LinearSpec, device="cpu") -> dict:
    """K, V (and Q) [B,H,T,64] bf16 ~ N(0,1)/8, W0 = I [B,H,64,64] fp32, needle V rows x scale."""
    s, shape = spec.seed, (spec.B, spec.H, spec.T, spec.D)
    out = {"eta": spec.eta}
    out["K"] = (rng.normal("K", shape, s, device) / 8.0).to(torch.bfloat16)
    V = (rng.normal("V", shape, s, device) / 8.0).to(torch.bfloat16)
    if spec.needle_frac > 0.0:
        for bi in range(spec.B):
            pos = torch.tensor(needle_positions(spec, bi), dtype=torch.int64, device=device)
            # Scaling a bf16 value by a power of two is exact.
            V[bi, :, pos, :] = V[bi, :, pos, :] * spec.needle_scale
    out["V"] = V
    if spec.with_queries:
        out["Q"] = (rng.normal("Q", shape, s, device) / 8.0).to(torch.bfloat16)
    eye = torch.eye(spec.D, dtype=torch.float32, device=device)
    out["W0"] = eye.expand(spec.B, spec.H, spec.D, spec.D).contiguous()
    return out


# ----------------------------------------------------------------------------------------------
# Richer inner models
# ----------------------------------------------------------------------------------------------

def inner_inputs(spec: InnerSpec, device="cpu") -> dict:
    """K, V (and Q) [B,H,T,64] bf16 ~ N(0,1)/8 as for TTT-Linear; LayerNorm gain 1 + 0.1·N(0,1)
    and bias 0.1·N(0,1) per head [H, 64] fp32. LayerNorm TTT-Linear: W0 = I [B,H,64,64].
    TTT-MLP: W1 ~ N(0,1) [B,H,64,256] (so k·W1 ~ N(0,1)) and W2 ~ N(0,1)/16 [B,H,256,64],
    packed per (sequence, head) as W1 then W2."""
    s, shape = spec.seed, (spec.B, spec.H, spec.T, spec.D)
    out = {"eta": spec.eta, "eps": spec.eps}
    out["K"] = (rng.normal("K", shape, s, device) / 8.0).to(torch.bfloat16)
    out["V"] = (rng.normal("V", shape, s, device) / 8.0).to(torch.bfloat16)
    if spec.with_queries:
        out["Q"] = (rng.normal("Q", shape, s, device) / 8.0).to(torch.bfloat16)
    out["gamma"] = (1.0 + 0.1 * rng.normal("ln_gamma", (spec.H, spec.D), s, device)).to(torch.float32)
    out["beta"] = (0.1 * rng.normal("ln_beta", (spec.H, spec.D), s, device)).to(torch.float32)
    if spec.model == "linear_ln":
        eye = torch.eye(spec.D, dtype=torch.float32, device=device)
        out["W0"] = eye.expand(spec.B, spec.H, spec.D, spec.D).contiguous()
    else:
        W1 = rng.normal("W1", (spec.B, spec.H, spec.D, spec.hidden), s, device).to(torch.float32)
        W2 = (rng.normal("W2", (spec.B, spec.H, spec.hidden, spec.D), s, device) / 16.0).to(torch.float32)
        out["W1"], out["W2"] = W1, W2
        out["W0"] = torch.cat([W1.reshape(spec.B, spec.H, -1), W2.reshape(spec.B, spec.H, -1)], dim=2).contiguous()
    return out
