"""CPU oracle for the two-point ZO probe step -- TEST INFRASTRUCTURE ONLY.

Plain, slow and written to be read against the pages: numpy for the
counter-based direction stream (fp32 / uint64 arithmetic, one rounding per
operation) and PyTorch CPU float64 for the decoder forward, the objective,
the estimator and the factored bank update.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The library under
``zeroth_order_fine_b200`` never does: it shares no code with the oracle,
and the oracle shares none with it -- the only common module is
``zeroth_order_fine_b200.workload``, which holds shapes and seeded inputs and
none of the method's arithmetic.

Parts and what pins them (see tests/test_oracle_*.py):

* generator  -- splitmix64 stream checked against an independent pure-Python
  integer implementation and the published first outputs of splitmix64;
  the own ln/sin/cos against libm within stated ulp bounds; N(0,1) moments
  and a Kolmogorov-Smirnov test.
* model      -- OPT and Qwen3 forwards checked against the HuggingFace
  ``transformers`` implementations of the same architectures (a library
  routine), causality and packing invariants.
* fp8        -- the E4M3 cast against the format decoded bit by bit (all 256
  codes; nearest value, ties to even, saturation), the per-row quantiser's
  scale equivariance and error bound.
* generation -- greedy decoding (one full forward per token) against teacher-forced
  scoring of the generated tokens, eps = 0 symmetry, the dense brute force.
* zo         -- the estimator against its closed form and an exact quadratic
  toy, its epsilon -> 0 limit against autograd, the factored perturbation
  against a dense brute force with W +/- eps*U V^T materialised, the bank
  against the dense sum of its updates.

Parity unpinned: the pages print no worked example, so no absolute L or c
value is pinned to the pages themselves; only the invariants above are.
"""
