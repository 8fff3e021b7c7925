"""CPU oracle for the mask-aware attention forward pass (test infrastructure).

This package is test infrastructure, not product code. Only the tests, the
smoke check and the benchmark's CPU-baseline / reference legs may import it.
The CUDA library never calls it, and it imports nothing from the CUDA side.

It is deliberately plain: numpy in float64, the mask expanded to a dense
boolean matrix, attention computed row by row from its definition.

* ``masks``     -- dense visibility from a compact mask description
* ``attention`` -- exact softmax(QK^T/sqrt(d) + mask) V and its log-sum-exp
* ``tilemap``   -- the per-tile SKIP / FULL / PARTIAL map and the compacted lists

Every function states the passage it follows. Parity of all three is pinned by
the ``-m "not gpu"`` tests (closed forms, library special cases, brute force).
"""
from . import masks, attention, tilemap  # noqa: F401
