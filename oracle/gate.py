"""Oracle of the SR-TTT surprisal gate and residual cache — test infrastructure only.

Source: "SR-TTT: Surprisal-Aware Residual Test-Time Training" (technical summary),
§2.1 "Surprisal Filter" and "Residual Cache", and §5 (eviction at saturation):

* condition 1: the token's reconstruction loss L_t exceeds τ_EMA, an EMA-smoothed
  95th-percentile threshold of recent losses;
* condition 2: the mean loss of the token's local chunk is at least 80 % of τ;
* tokens meeting both are routed to a fixed-capacity residual cache that runs beside the
  fast weight.

Readings taken where the page leaves the arithmetic open (all applied identically by the
CUDA path): chunks of 64 tokens per (sequence, head), processed in order; p95 is the
nearest-rank percentile, i.e. the ceil(0.95·64) = 61st smallest value; τ starts as the
first chunk's p95 and then follows τ ← fl32(fl32(0.9·τ) + fl32(0.1·p95)) with the fp32
constants 0.9 and 0.1 and no fused multiply-add; the threshold is updated first and the
chunk is then gated with the updated τ; the mean test "S/64 ≥ (4/5)·τ" is evaluated as
5·S ≥ 256·τ in double, with S the double sum of the chunk's 64 fp32 losses in index
order; L_t > τ is a strict fp32 comparison; one cache per (sequence, head) receives the
routed (sequence, head, t) triples in increasing t until it is full, after which routed
tokens are dropped and counted. The gate does not alter the fast-weight update.
"""

from __future__ import annotations

import math

import numpy as np


class GateState:
    """Per-(sequence, head) gate state: τ, whether τ is set, the cache and its counters."""

    def __init__(self, B: int, H: int, capacity: int = 256):
        self.B, self.H, self.capacity = B, H, capacity
        self.tau = np.zeros((B, H), dtype=np.float32)
        self.tau_set = np.zeros((B, H), dtype=bool)
        self.entries = np.full((B, H, capacity, 3), -1, dtype=np.int32)
        self.routed = np.zeros((B, H), dtype=np.int64)
        self.dropped = np.zeros((B, H), dtype=np.int64)
        self.t_offset = 0

    def counts(self) -> np.ndarray:
        """[B, H, 2] int32: (tokens routed since reset, routed tokens dropped because full)."""
        return np.stack([self.routed, self.dropped], axis=-1).astype(np.int32)


def nearest_rank(pct: float, n: int) -> int:
    """1-based nearest rank ceil(pct·n) (61 for pct = 0.95, n = 64)."""
    return int(math.ceil(pct * n - 1e-12))


def surprisal_route(loss, state: GateState, gate_chunk: int = 64, pct: float = 0.95,
                    ema_old=np.float32(0.9), ema_new=np.float32(0.1),
                    mean_num: int = 4, mean_den: int = 5) -> GateState:
    """Run the gate over ``loss`` [B, H, T] (fp32) and append to ``state`` in place.

    T must be a multiple of ``gate_chunk``. Token indices stored in the cache count from the
    last reset, so successive calls continue one stream.
    """
    L = np.asarray(loss, dtype=np.float32)
    B, H, T = L.shape
    if T % gate_chunk != 0:
        raise ValueError("T must be a multiple of the gate chunk")
    rank = nearest_rank(pct, gate_chunk)
    ema_old, ema_new = np.float32(ema_old), np.float32(ema_new)
    for bi in range(B):
        for hi in range(H):
            tau = state.tau[bi, hi]
            for g in range(T // gate_chunk):
                x = L[bi, hi, g * gate_chunk:(g + 1) * gate_chunk]
                p = np.sort(x)[rank - 1]
                if state.tau_set[bi, hi]:
                    tau = np.float32(np.float32(ema_old * tau) + np.float32(ema_new * p))
                else:
                    tau = np.float32(p)
                    state.tau_set[bi, hi] = True
                S = 0.0
                for v in x:
                    S += float(v)
                passed = mean_den * S >= float(mean_num * gate_chunk) * float(tau)
                if not passed:
                    continue
                for j in range(gate_chunk):
                    if x[j] > tau:
                        n = state.routed[bi, hi]
                        if n < state.capacity:
                            state.entries[bi, hi, n] = (bi, hi, state.t_offset + g * gate_chunk + j)
                        else:
                            state.dropped[bi, hi] += 1
                        state.routed[bi, hi] = n + 1
            state.tau[bi, hi] = tau
    state.t_offset += T
    return state
