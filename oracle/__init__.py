"""fp64 CPU oracle for the rotation -> group-quantisation -> W4A4 linear path.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this package: only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline leg and
its ``--impl reference`` arm) may use it. It shares no code with the CUDA library;
the only module both sides use is ``workloads`` (seeded random draws).

Every function is the plain definition of what it computes, written from the
pages it cites, in float64 unless the pages fix a precision:

* ``hadamard``  Sylvester Hadamard matrix, randomized Hadamard transform (dense
  O(K^2) products), and a page-2-style in-place FWHT used only as a pin.
* ``harp``      HARP block construction (Givens x Sylvester, QR fallback) and the
  stage-by-stage mixed-radix processor with stride permutations.
* ``quant``     per-group symmetric absmax quantisation, fp16 scales, packing,
  dequantisation, rounding-boundary flags.
* ``linear``    the W4A4 linear (exact int64 group sums, fp64 scaling) and the
  page-2 ``matmul_q_err`` RMS-relative-error metric.

Parity status of each function is listed in the module docstrings; every function
here is pinned by a ``-m "not gpu"`` test in ``tests/test_oracle_pins.py`` except
where a docstring says "parity unpinned".
"""
from . import hadamard, harp, quant, linear  # noqa: F401
