"""The arithmetic fact behind the gate's tree-order chunk sum (CPU, no GPU needed).

The GPU gate sums a chunk's 64 fp32 losses in a tree order when every value is finite and
non-negative and their exponent fields span at most 23 (the smallest counted as at least 1);
otherwise it adds them in index order as the definition says. The tree is used because then
every partial sum is an integer multiple of the smallest ulp and below 2^53 of it, so every
order of double additions is exact. These tests check that fact itself against the index-order
double sum of the definition, and check that it fails without the span condition, so the
condition is needed.
"""

import numpy as np

from oracle import gate as ogate


def _tree_sum(x: np.ndarray) -> float:
    """Pairwise sum in the order the GPU's xor butterfly adds: lane j starts with x[j] + x[j+32],
    then partners at distance 1, 2, 4, 8, 16."""
    s = [float(x[j]) + float(x[j + 32]) for j in range(32)]
    o = 1
    while o < 32:
        s = [s[j] + s[j ^ o] for j in range(32)]
        o <<= 1
    return s[0]


def _index_sum(x: np.ndarray) -> float:
    S = 0.0
    for v in x:
        S += float(v)
    return S


def _exact_condition(x: np.ndarray) -> bool:
    b = x.view(np.uint32)
    e = (b >> 23) & 0xFF
    if np.any(b >> 31) or np.any(e == 0xFF):
        return False
    nz = b != 0
    if not nz.any():
        return True
    emin = np.maximum(e[nz], 1).min()
    return int(e.max()) - int(emin) <= 23


def test_every_order_agrees_within_the_exponent_span():
    rng = np.random.default_rng(2024)
    checked = 0
    for trial in range(3000):
        span = int(rng.integers(0, 24))
        base = int(rng.integers(-60, 60))
        exps = base + rng.integers(0, span + 1, 64)
        mant = rng.integers(1 << 23, 1 << 24, 64).astype(np.float64) / float(1 << 23)
        x = (mant * np.exp2(exps.astype(np.float64))).astype(np.float32)
        x[rng.random(64) < 0.05] = 0.0
        if not _exact_condition(x):
            continue
        checked += 1
        seq = _index_sum(x)
        assert _tree_sum(x) == seq
        assert float(np.sum(x.astype(np.float64)[rng.permutation(64)])) == seq
        # the sum is the exact rational sum of the values
        assert np.float64(seq) == np.float64(sum(map(float, x)))
    assert checked > 2500


def test_the_span_condition_is_needed():
    # 2^53 and 63 ones: in index order every +1 is a tie that rounds back to 2^53; a tree adds
    # the ones among themselves first and keeps them.
    x = np.ones(64, np.float32)
    x[0] = np.float32(2.0 ** 53)
    assert not _exact_condition(x)
    assert _tree_sum(x) != _index_sum(x)


def test_the_oracle_gate_sum_is_the_index_order_sum():
    """The oracle's pass test uses the index-order double sum; the identity above is what makes
    a tree on the GPU equal to it."""
    x = np.linspace(0.5, 2.0, 64, dtype=np.float32)
    assert _exact_condition(x)
    assert _tree_sum(x) == _index_sum(x)
    st = ogate.GateState(1, 1, 8)
    ogate.surprisal_route(x[None, None, :], st)
    assert st.tau_set[0, 0]
