"""Float64 CPU oracle of the Gated KalmaNet layer.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``.  The CUDA library never imports,
links or runs anything here.

Parity status: every function is pinned by ``tests/test_oracle_pins.py``
(closed forms, the exact ridge solve, the page's rate table, invariances).
"""
from .oracle import (  # noqa: F401
    backward,
    build,
    cheb_solve,
    chunked_norms,
    decode_step,
    forward,
    max_threads,
    omegas,
    solver_residuals,
    solver_study,
    SOLVERS,
)
