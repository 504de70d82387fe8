"""Plain, slow CPU oracle of the fast-weight chunk scan — TEST INFRASTRUCTURE ONLY.

This package is the reference the CUDA path is checked against. It is written from
the pages' descriptions of the method, in float64 with numpy, step by step in the
pages' order, with no blocking, fusion or reordering beyond the definitions:

* :mod:`oracle.inplace` — In-Place TTT apply-then-update scan with the Hebbian,
  LM-aligned update and the Conv1D + Wtarget target (In-Place Test-Time Training,
  §2 "Wdown as fast weight", §3 "apply first, update later", §4 "predict the next
  token", §6 "context parallelism").
* :mod:`oracle.linear` — TTT-Linear mini-batch gradient scan (TTT layers page: the
  recurrent state is an inner model's weight trained while the sequence is read; and its
  DeltaNet remark).
* :mod:`oracle.gate` — SR-TTT surprisal gate and residual cache (SR-TTT technical
  summary, §2.1 "Surprisal Filter" and "Residual Cache").
* :mod:`oracle.cache_attention` — the residual cache's read path, attention over the cached
  keys and values fused into the TTT output through the clamped gate α (SR-TTT technical
  summary, §2.1 "Residual Cache" and "Alpha Fusion").
* :mod:`oracle.packed` — packed sequences: the weight reset to its pretrained value at every
  document start, and the update delta's Frobenius norm clipped (In-Place Test-Time
  Training, §6 and its implementation notes).
* :mod:`oracle.inner` — the richer inner models of a TTT layer: TTT-Linear with LayerNorm
  and residual, and TTT-MLP (TTT layers page: its two instances, the DeltaNet remark on
  LayerNorm and residual, and the conclusion on TTT-MLP's memory I/O).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import it. The product path (the C-ABI library and its Python binding) never does;
it shares no code, header or constant with this package.

Every function here is pinned by ``tests/test_oracle_*.py`` to closed forms,
hand-derived worked examples (``tests/golden/``), special cases and brute force.
"""

from . import cache_attention, gate, inner, inplace, linear, packed  # noqa: F401
