"""Planted mistakes: every plausible slip in the oracle fails at least one committed pin.

For each mutation below, one oracle module's source is edited in one place (on the CPU;
nothing here touches the CUDA path), loaded as a separate module, and the pin tests of
tests/test_oracle_<module>.py are run with it in place of the real module. The unmutated
oracle passes all of them; each mutant must fail at least one. This is the evidence that
the pins constrain the oracle's arithmetic rather than restate it.
"""

from __future__ import annotations

import importlib
import inspect
import os
import types

import pytest

ORACLE = os.path.join(os.path.dirname(__file__), "..", "oracle")

# (module, description, [(text, replacement), ...]); each text occurs exactly once.
MUTANTS = [
    ("inplace", "wrong sign of the update",
     [("W = W + eta * (Vc.T @ Zc)", "W = W - eta * (Vc.T @ Zc)")]),
    ("inplace", "step size dropped from the update",
     [("W = W + eta * (Vc.T @ Zc)", "W = W + (Vc.T @ Zc)")]),
    ("inplace", "update applied before the chunk's own output",
     [("        O[rows] = Zc @ W.T                 # apply with W before this chunk's update (§3)\n"
       "        W = W + eta * (Vc.T @ Zc)          # ΔW = η·V̂ᵀ·Z (§2)",
       "        W = W + eta * (Vc.T @ Zc)\n"
       "        O[rows] = Zc @ W.T")]),
    ("inplace", "every chunk applied with the initial weight",
     [("O[rows] = Zc @ W.T ", "O[rows] = Zc @ f64(W0).T ")]),
    ("inplace", "convolution tap shifted by one token",
     [("        src = t + k\n", "        src = t + k + 1\n")]),
    ("inplace", "convolution ignores the chunk boundary",
     [("end = np.minimum((t // C + 1) * C, T) if pad_mode == 0 else np.full(T, T)", "end = np.full(T, T)")]),
    ("inplace", "convolution weights of the wrong tap",
     [("out[ok] += X[src[ok]] * w[:, k]", "out[ok] += X[src[ok]] * w[:, taps - 1 - k]")]),
    ("linear", "wrong sign of the gradient step",
     [("W = W - (eta / b) * (np.swapaxes(Ki, 1, 2) @ R)", "W = W + (eta / b) * (np.swapaxes(Ki, 1, 2) @ R)")]),
    ("linear", "step size not divided by the mini-batch",
     [("W = W - (eta / b) * (np.swapaxes(Ki, 1, 2) @ R)", "W = W - eta * (np.swapaxes(Ki, 1, 2) @ R)")]),
    ("linear", "residual with the wrong sign",
     [("R = Ki @ W - Vi ", "R = Vi - Ki @ W ")]),
    ("linear", "transposed gradient",
     [("W = W - (eta / b) * (np.swapaxes(Ki, 1, 2) @ R)", "W = W - (eta / b) * (np.swapaxes(R, 1, 2) @ Ki)")]),
    ("linear", "outputs from the weight after the mini-batch's update",
     [("        if Qf is not None and not token_weights:\n"
       "            O[:, s] = Qf[:, s] @ W                       # output with W_i (start of mini-batch)\n",
       ""),
      ("        W = W - (eta / b) * (np.swapaxes(Ki, 1, 2) @ R)  # one gradient step on ℓ_i\n",
       "        W = W - (eta / b) * (np.swapaxes(Ki, 1, 2) @ R)\n"
       "        if Qf is not None and not token_weights:\n"
       "            O[:, s] = Qf[:, s] @ W\n")]),
    ("linear", "per-token weights without the token's own step",
     [("(np.swapaxes(Ki[:, :j + 1], 1, 2) @ R[:, :j + 1])", "(np.swapaxes(Ki[:, :j], 1, 2) @ R[:, :j])")]),
    ("packed", "per-document per-token weights from the wrong step size",
     [("Wt = W - (eta / n) * (Kd[s, h, i0:i0 + j + 1].T @ R[:j + 1])", "Wt = W - (eta / b) * (Kd[s, h, i0:i0 + j + 1].T @ R[:j + 1])")]),
    ("packed", "LayerNorm and MLP documents not restarted from the pretrained weights",
     [("                W = (W0s[0][s, h], W0s[1][s, h]) if mlp else W0s[s, h]   # document boundary: θ ← θ0\n",
       "                W = W if a > 0 else ((W0s[0][s, h], W0s[1][s, h]) if mlp else W0s[s, h])\n")]),
    ("packed", "short last LayerNorm or MLP mini-batch stepped as a full one",
     [("                                                            g, be, eta, n, eps, token_weights=token_weights)",
       "                                                            g, be, eta * n / b, n, eps, token_weights=token_weights)"),
      ("        o, Wn, l = inner.ttt_linear_ln_scan(one(Kd), one(Vd), one(Qd), W[None, None], g, be, eta, n, eps,",
       "        o, Wn, l = inner.ttt_linear_ln_scan(one(Kd), one(Vd), one(Qd), W[None, None], g, be, eta * n / b, n, eps,")]),
    ("linear", "loss not squared per element",
     [("loss[:, s] = np.sum(R * R, axis=2)", "loss[:, s] = np.sum(R, axis=2) ** 2")]),
    ("gate", "percentile one rank too high",
     [("p = np.sort(x)[rank - 1]", "p = np.sort(x)[min(rank, len(x) - 1)]")]),
    ("gate", "EMA weights swapped",
     [("tau = np.float32(np.float32(ema_old * tau) + np.float32(ema_new * p))",
       "tau = np.float32(np.float32(ema_new * tau) + np.float32(ema_old * p))")]),
    ("gate", "threshold not carried from chunk to chunk",
     [("                if state.tau_set[bi, hi]:\n", "                if False:\n")]),
    ("gate", "comparison with the threshold not strict",
     [("if x[j] > tau:", "if x[j] >= tau:")]),
    ("gate", "mean test with numerator and denominator swapped",
     [("passed = mean_den * S >= float(mean_num * gate_chunk) * float(tau)",
       "passed = mean_num * S >= float(mean_den * gate_chunk) * float(tau)")]),
    ("gate", "mean test skipped",
     [("                if not passed:\n                    continue\n", "")]),
    ("gate", "dropped tokens not counted",
     [("                            state.dropped[bi, hi] += 1\n", "                            pass\n")]),
    ("gate", "token index ignores the stream position",
     [("(bi, hi, state.t_offset + g * gate_chunk + j)", "(bi, hi, g * gate_chunk + j)")]),
    ("cache_attention", "entries of the query's own gate chunk visible",
     [("visible = gc < t // gate_chunk", "visible = gc <= t // gate_chunk")]),
    ("cache_attention", "scores not scaled by 1/sqrt(D)",
     [("scale = 1.0 / np.sqrt(D)", "scale = 1.0")]),
    ("cache_attention", "softmax weights not normalised",
     [("A[bi, hi, t] = (w / w.sum()) @ vc[visible]", "A[bi, hi, t] = w @ vc[visible]")]),
    ("cache_attention", "alpha not clamped",
     [("a = np.clip(f64(alpha), 0.0, 1.0)", "a = f64(alpha)")]),
    ("cache_attention", "every cache slot read, not the stored entries",
     [("n = min(int(np.asarray(counts)[bi, hi, 0]), E.shape[2])", "n = E.shape[2]")]),
    ("cache_attention", "keys and values swapped",
     [("kc, vc, gc = Kd[bi, hi, ts], Vd[bi, hi, ts], ts // gate_chunk",
       "kc, vc, gc = Vd[bi, hi, ts], Kd[bi, hi, ts], ts // gate_chunk")]),
    ("cache_attention", "query of the previous token",
     [("s = (kc[visible] @ Qd[bi, hi, t]) * scale", "s = (kc[visible] @ Qd[bi, hi, t - 1]) * scale")]),
    ("packed", "fused targets of a document computed over the whole packed sequence",
     [("V[a:e] = inplace.target_values(X[a:e], convw, Wtarget, C, pad_mode)",
       "V[a:e] = inplace.target_values(X, convw, Wtarget, C, pad_mode)[a:e]")]),
    ("packed", "fused targets of packed documents always padded at chunk ends",
     [("V[a:e] = inplace.target_values(X[a:e], convw, Wtarget, C, pad_mode)",
       "V[a:e] = inplace.target_values(X[a:e], convw, Wtarget, C, 0)")]),
    ("packed", "In-Place weight not reset at a document start",
     [("        W = W0d.copy()                                   # document boundary: pretrained weight\n",
       "")]),
    ("packed", "TTT-Linear weight not reset at a document start",
     [("                W = W0d[s, h].copy()                     # document boundary: W ← W0\n", "")]),
    ("packed", "clipping enlarges small deltas instead of shrinking large ones",
     [("return dW * (clip / n) if n > clip else dW", "return dW * (clip / n) if n < clip else dW")]),
    ("packed", "short last mini-batch divided by b instead of its own size",
     [("W = W - (eta / n) * (Kd[s, h, r].T @ R)", "W = W - (eta / b) * (Kd[s, h, r].T @ R)")]),
    ("inner", "LayerNorm variance divided by D - 1",
     [("var = ((Z - mu) ** 2).mean(axis=-1, keepdims=True)",
       "var = ((Z - mu) ** 2).sum(axis=-1, keepdims=True) / (Z.shape[-1] - 1)")]),
    ("inner", "LayerNorm without the mean subtracted",
     [("zhat = (Z - mu) * rstd", "zhat = Z * rstd")]),
    ("inner", "epsilon outside the square root",
     [("rstd = 1.0 / np.sqrt(var + eps)", "rstd = 1.0 / (np.sqrt(var) + eps)")]),
    ("inner", "gain and bias in the wrong order",
     [("return gamma * zhat + beta, zhat, rstd", "return gamma * (zhat + beta), zhat, rstd")]),
    ("inner", "LayerNorm backward without the normalised-input term",
     [(" - zhat * (g * zhat).mean(axis=-1, keepdims=True))", ")")]),
    ("inner", "LayerNorm backward without the mean term",
     [("(g - g.mean(axis=-1, keepdims=True) - zhat", "(g - zhat")]),
    ("inner", "gain not applied in the backward",
     [("    g = dY * gamma\n", "    g = dY\n")]),
    ("inner", "residual missing from the TTT-Linear loss",
     [("        E = Ki + Y - Vi                                    # f(k) − v\n",
       "        E = Y - Vi\n")]),
    ("inner", "residual missing from the outputs",
     [("O[:, s] = Qf[:, s] + layer_norm(Qf[:, s] @ W, gam, bet, eps)[0]",
       "O[:, s] = layer_norm(Qf[:, s] @ W, gam, bet, eps)[0]")]),
    ("inner", "TTT-Linear step with the wrong sign",
     [("W = W - (eta / b) * (np.swapaxes(Ki, 1, 2) @ dZ)", "W = W + (eta / b) * (np.swapaxes(Ki, 1, 2) @ dZ)")]),
    ("inner", "TTT-Linear outputs from the weight after the step",
     [("        if Qf is not None and not token_weights:\n"
       "            O[:, s] = Qf[:, s] + layer_norm(Qf[:, s] @ W, gam, bet, eps)[0]  # f(q; W_i)\n", ""),
      ("        W = W - (eta / b) * (np.swapaxes(Ki, 1, 2) @ dZ)   # one gradient step on ℓ_i\n",
       "        W = W - (eta / b) * (np.swapaxes(Ki, 1, 2) @ dZ)\n"
       "        if Qf is not None and not token_weights:\n"
       "            O[:, s] = Qf[:, s] + layer_norm(Qf[:, s] @ W, gam, bet, eps)[0]\n")]),
    ("inner", "MLP first layer's gradient taken through the updated second layer",
     [("        W1 = W1 - (eta / b) * dW1\n        W2 = W2 - (eta / b) * dW2\n",
       "        W1 = W1 - (eta / b) * dW1\n"),
      ("        dH = (dZ @ np.swapaxes(W2, 1, 2)) * act_grad(Hpre)  # back through W2 and the activation\n",
       "        W2 = W2 - (eta / b) * dW2\n"
       "        dH = (dZ @ np.swapaxes(W2, 1, 2)) * act_grad(Hpre)\n")]),
    ("inner", "GELU derivative without the density term",
     [(" + x * np.exp(-0.5 * x * x) / np.sqrt(2.0 * np.pi)", "")]),
    ("inner", "second layer's gradient from the pre-activation",
     [("dW2 = np.swapaxes(A, 1, 2) @ dZ", "dW2 = np.swapaxes(Hpre, 1, 2) @ dZ")]),
    ("inner", "MLP outputs without the activation",
     [("O[:, s] = Qf[:, s] + layer_norm(act(Qf[:, s] @ W1) @ W2, gam, bet, eps)[0]",
       "O[:, s] = Qf[:, s] + layer_norm((Qf[:, s] @ W1) @ W2, gam, bet, eps)[0]")]),
    ("inner", "per-token weights without the token's own step",
     [("Wt = W - (eta / b) * (np.swapaxes(Ki[:, :j + 1], 1, 2) @ dZ[:, :j + 1])",
       "Wt = W - (eta / b) * (np.swapaxes(Ki[:, :j], 1, 2) @ dZ[:, :j])")]),
    ("inner", "per-token weights that see the next token's step",
     [("Wt = W - (eta / b) * (np.swapaxes(Ki[:, :j + 1], 1, 2) @ dZ[:, :j + 1])",
       "Wt = W - (eta / b) * (np.swapaxes(Ki[:, :j + 2], 1, 2) @ dZ[:, :j + 2])")]),
    ("inner", "MLP per-token weights with the second layer left at the mini-batch's start",
     [("W2t = W2 - (eta / b) * (np.swapaxes(A[:, :j + 1], 1, 2) @ dZ[:, :j + 1])", "W2t = W2")]),
    ("inner", "GELU from the wrong distribution scale",
     [("return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))", "return 0.5 * x * (1.0 + erf(x))")]),
]


def _load(module: str, edits) -> types.ModuleType:
    src = open(os.path.join(ORACLE, f"{module}.py"), encoding="utf-8").read()
    for text, replacement in edits:
        assert src.count(text) == 1, f"mutation text not found once in oracle/{module}.py: {text!r}"
        src = src.replace(text, replacement)
    mod = types.ModuleType(f"oracle.planted_{module}")
    mod.__package__ = "oracle"
    exec(compile(src, f"<oracle/{module}.py, planted>", "exec"), mod.__dict__)
    return mod


def _failing_pins(module: str, impl: types.ModuleType) -> list[str]:
    """Names of the pin tests of ``module`` that fail with ``impl`` swapped in."""
    pins = importlib.import_module(f"tests.test_oracle_{module}")
    real = getattr(pins, module)
    setattr(pins, module, impl)
    failed = []
    try:
        for name, fn in inspect.getmembers(pins, inspect.isfunction):
            if not name.startswith("test_") or fn.__module__ != pins.__name__:
                continue
            try:
                fn()
            except (KeyboardInterrupt, SystemExit):
                raise
            except BaseException:  # an assertion, a pytest failure, or an error the slip causes
                failed.append(name)
    finally:
        setattr(pins, module, real)
    return failed


@pytest.mark.parametrize("module", ["inplace", "linear", "gate", "cache_attention", "packed", "inner"])
def test_unmutated_oracle_passes_every_pin(module):
    assert _failing_pins(module, _load(module, [])) == []


@pytest.mark.parametrize("module,description,edits", MUTANTS, ids=[f"{m}: {d}" for m, d, _ in MUTANTS])
def test_planted_mistake_fails_a_pin(module, description, edits):
    failed = _failing_pins(module, _load(module, edits))
    assert failed, f"no pin of oracle/{module}.py catches: {description}"
