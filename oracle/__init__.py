"""Float64 CPU oracle for the KDA recurrence.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by the smoke check and by the
benchmark's CPU-baseline leg, never by the product path. It shares no code
with the CUDA library and does not import it.

* ``ref.forward``         -- the plain C recurrence (``kda_ref.c``), threaded over (sequence, head).
* ``ref.forward_numpy``   -- the same definition restated in numpy (small cases).
* ``chunked.forward``     -- the chunkwise form derived from the definition (float64, test-only).
* ``brute``               -- exact rational arithmetic on explicit transition matrices (tiny cases).
* ``backward.backward``   -- gradients of the recurrence by a token-level reverse sweep (float64).
* ``chunked.backward``    -- the same gradients through the chunk form (float64, test-only).

Parity status: every function here is pinned by tests that do not go through
itself (closed forms, exact rational brute force, invariants); see
``tests/test_oracle_pins.py`` and ``tests/test_oracle_backward.py``.
"""
