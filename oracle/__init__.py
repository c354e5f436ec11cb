"""fp64 CPU oracle for the Falcon fast-weight forward pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package. The product
path (``delta_rule_linear_falcon_b200``) never imports it and shares no code
with it.

Parity status (each pinned by CPU tests against facts other than the oracle
itself; see tests/test_oracle_pins.py):
  recurrent  -- pinned: hand-expanded T<=3 algebra, Kaczmarz interpolation,
                decay-only closed form, finite-difference gradient steps of the
                two objectives, Falcon-1A closed form, NLMS scale invariance,
                orthonormal-key recall, Kaczmarz convergence, segment split.
  chunk      -- pinned: agrees with the recurrent form for every chunk size.
  masked     -- pinned: agrees with the recurrent form (one block of T steps).
  backward   -- pinned: central finite differences of the recurrent form for every
                input (tests/test_oracle_backward.py).
"""
from .oracle import (  # noqa: F401
    RULE_1, RULE_1A, RULE_3, RULE_3A, RULE_2, RULE_2A, falcon2,
    build_oracle, oracle_lib_path, recurrent, chunk, masked, decode_step, max_threads, backward,
)
