"""Plain fp64 CPU oracle for the fused chunked forward-KL distillation loss.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never calls it, links it or falls back to it, and this package imports nothing
from the CUDA library: the two share only the seeded input generator
(``synth``), which holds no loss arithmetic.

Every function here is pinned by ``tests/test_oracle_pins.py`` to something
other than itself (library routines, closed forms, invariants, finite
differences, autograd of a dense library formulation).  No function is
"parity unpinned".
"""
from .kl import (  # noqa: F401
    log_softmax,
    teacher_distribution,
    student_log_probs,
    dense_teacher,
    fused_chunked_kl,
    widen_bf16,
    oracle_from_inputs,
)
from .selective import student_entropy, select_top_rows  # noqa: F401
