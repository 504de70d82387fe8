"""Pins of the surprisal-gate oracle: hand-built loss arrays with written-down answers,
the percentile against numpy's inverted-CDF definition, and the compaction against a
plain loop over a precomputed decision mask."""

import json
import os

import numpy as np

from oracle import gate

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _run(loss_1d, capacity=256):
    L = np.asarray(loss_1d, dtype=np.float32)[None, None]
    st = gate.GateState(1, 1, capacity)
    gate.surprisal_route(L, st)
    n = min(int(st.routed[0, 0]), capacity)
    return st, [int(e[2]) for e in st.entries[0, 0, :n]]


def test_hand_cases():
    g = json.load(open(os.path.join(GOLDEN, "gate_hand.json")))
    for name in ("needles", "all_equal", "mean_boundary", "mean_just_below", "ema"):
        c = g[name]
        loss = np.concatenate([np.asarray(x, np.float32) for x in c["loss"]])
        st, routed = _run(loss)
        assert routed == c["routed_t"], name
        assert st.tau[0, 0] == np.float32(c["tau"][-1]), name
        assert st.routed[0, 0] == len(c["routed_t"]) and st.dropped[0, 0] == 0


def test_capacity_drops_late_tokens():
    c = json.load(open(os.path.join(GOLDEN, "gate_hand.json")))["capacity"]
    loss = np.ones(64 * c["chunks"], np.float32)
    for g in range(c["chunks"]):
        for o in c["needle_offsets"]:
            loss[64 * g + o] = 100.0
    st, routed = _run(loss, c["capacity"])
    assert int(st.routed[0, 0]) == c["routed"] and int(st.dropped[0, 0]) == c["dropped"]
    assert len(routed) == c["capacity"] and routed[-1] == c["last_stored_t"]
    assert routed == sorted(routed)
    assert st.tau[0, 0] == np.float32(1.0)


def test_percentile_is_nearest_rank():
    """The 61st smallest of 64 equals numpy's inverted-CDF (nearest-rank) 95th percentile."""
    assert gate.nearest_rank(0.95, 64) == 61
    rng = np.random.default_rng(0)
    for trial in range(50):
        x = rng.standard_normal(64).astype(np.float32) ** 2
        p_np = np.percentile(x, 95, method="inverted_cdf")
        st = gate.GateState(1, 1)
        gate.surprisal_route(x[None, None], st)
        assert st.tau[0, 0] == np.float32(p_np)


def test_streaming_equals_one_call():
    rng = np.random.default_rng(1)
    L = (rng.standard_normal((2, 3, 64 * 12)) ** 2).astype(np.float32)
    L[:, :, ::17] *= 50
    one = gate.GateState(2, 3, 16)
    gate.surprisal_route(L, one)
    two = gate.GateState(2, 3, 16)
    gate.surprisal_route(L[:, :, :64 * 5], two)
    gate.surprisal_route(L[:, :, 64 * 5:], two)
    assert np.array_equal(one.entries, two.entries)
    assert np.array_equal(one.counts(), two.counts())
    assert np.array_equal(one.tau, two.tau)


def test_compaction_matches_mask_loop():
    """Recompute τ and the pass flags chunk by chunk, build the routed mask, and compact it
    with a plain loop; the oracle's cache must agree entry for entry."""
    rng = np.random.default_rng(2)
    B, H, T = 2, 2, 64 * 9
    L = (rng.standard_normal((B, H, T)) ** 2).astype(np.float32)
    L[:, :, rng.integers(0, T, 40)] = 30.0
    st = gate.GateState(B, H, 32)
    gate.surprisal_route(L, st)
    for bi in range(B):
        for hi in range(H):
            taus, mask = [], np.zeros(T, bool)
            for g in range(T // 64):
                x = L[bi, hi, 64 * g:64 * (g + 1)]
                p = np.float32(np.percentile(x, 95, method="inverted_cdf"))
                tau = p if not taus else np.float32(np.float32(np.float32(0.9) * taus[-1])
                                                     + np.float32(np.float32(0.1) * p))
                taus.append(tau)
                if np.sum(x.astype(np.float64)) * 5.0 >= 256.0 * float(tau):
                    mask[64 * g:64 * (g + 1)] = x > tau
            routed = [t for t in range(T) if mask[t]]
            kept = routed[:32]
            got = [int(e[2]) for e in st.entries[bi, hi, :len(kept)]]
            assert got == kept
            assert all((e == -1).all() for e in st.entries[bi, hi, len(kept):])
            assert int(st.routed[bi, hi]) == len(routed)
            assert int(st.dropped[bi, hi]) == max(0, len(routed) - 32)
            assert all(int(e[0]) == bi and int(e[1]) == hi for e in st.entries[bi, hi, :len(kept)])
