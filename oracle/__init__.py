"""CPU oracle for the OCTOPUS KV-cache codec (test infrastructure only).

This package is the slow, plain reference that the CUDA library is checked
against. It is NOT part of the product: only ``tests/``, the smoke check in
``__graft_entry__.py`` and the ``cpu_baseline`` / ``--impl reference`` legs
of ``bench.py`` may import it. It shares no code with the CUDA library
(``rotation_preconditioned_quantization_b200``) and does not import it; the
only module both sides use is ``rotation_preconditioned_quantization_b200.inputs``,
which draws seeded random inputs and contains none of the codec's arithmetic.

Everything is numpy float64 unless a step is integer by nature. Each function
cites the passage of the pages it follows, by page and section:

* [EXPL]  the Chinese explainer of the OCTOPUS paper (m.youleyou.com,
          wenzhang 3300010), sections "rotation", "octahedral folding",
          "triplet decomposition", "non-uniform bit allocation",
          "joint rounding", "experimental results",
          "optional residual correction", "engineering implementation";
* [SUMM]  the agents-report.net summary "OCTOPUS: octahedral parametrisation
          and joint triplet quantisation", sections "method overview",
          "bit allocation", "implementation", "OCTOPUS-QJL";
* [ABS]   the paper's abstract ("OCTOPUS: Optimized KV Cache for Transformers
          via Octahedral Parametrization Under optimal Squared error
          quantization", arxivlens / chatpaper pages).

Where the pages leave a step open, the reading taken is stated in the
function's docstring.

Parity status: every function here is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_*.py``. The QJL sketch is pinned three ways: a worked
case with a non-symmetric permutation as the projection (orientation of S,
the sign of a zero projection, the scale), the estimator's unbiasedness over
seeds, and its closed-form variance over seeds; the projection matrix itself
is pinned by the generator's published test vector and its moments.
"""

from . import tables, codec, attention, baselines  # noqa: F401
