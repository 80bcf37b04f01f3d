"""fp64 CPU oracle for the LoRAForge hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The CUDA path never does, and this package never
imports the CUDA path: the two share no code.  Inputs are plain numpy arrays
(the seeded generators that fill them live in their own module and hold none of
the method's arithmetic).

Everything here is computed in float64 from the exact fp32/bf16 input bytes,
written for a reader to check against the pages by eye:

* ``factor``   -- Delta W = B A, its truncated SVD (definition route) and the
                  factor-space route (QR of B and A^T, SVD of R_B R_A^T),
                  export of retained factors, reconstruction errors.
* ``allocate`` -- LoRAForge-U (uniform retention) and LoRAForge-S (spectral
                  energy budget with a per-module floor) rank allocation.
* ``apply``    -- adapter routing and the multi-LoRA side path
                  y += s * B' (A' x) by brute force.
* ``jd``       -- joint diagonalization (JD-Full) of a LoRA collection by
                  eigenvalue iteration with a QR orthogonalize.
* ``pool``     -- the pool-wide shared subspace of stacked LoRA factors that keeps
                  a fraction (99 %) of their energy (LoRASpace).

Every function names the passage it follows by page title and section.
Readings of passages the pages leave open are stated beside the code.
Pins: every function here is pinned by ``tests/test_oracle_*.py`` against
closed forms, library special cases, brute force or hand-worked fixtures
(``tests/golden``); none is "parity unpinned".
"""
from . import factor, allocate, apply, jd, pool  # noqa: F401
