"""Plain fp64 CPU oracle for the per-matrix Muon and SOAP optimizer steps.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library (no headers, helpers, constants or tables); the
only thing both sides consume is the seeded input generators in ``workloads``,
which hold none of the method's arithmetic.

Everything here is written from the method's published description, restated
in our own code, and follows its steps in the order the pages give them:

* ``ns``    - Newton-Schulz orthogonalisation ("LLM Optimizers: From SGD and
              AdamW to SOAP, Muon, and Scalable Training", section 11.4
              equation; "Matrix optimizers: K-FAC, Shampoo and Muon",
              Lemma 3 and the three-step algorithm under it).
* ``muon``  - the Muon step ("Matrix optimizers: K-FAC, Shampoo and Muon",
              section "Muon", steps 1-4; "LLM Optimizers ...", sections
              11.3 and 11.5).
* ``soap``  - the SOAP step with a per-step power-iteration + QR basis
              refresh ("LLM Optimizers ...", section 11.1 equations;
              "Reading notes on SOAP, Muon, and Beyond", sections 1 and 4;
              "初探优化器（一）", section 6.2).
* ``qr``    - the QR factorisation with the positive-diagonal convention.
* ``bf16``  - round-to-nearest-even rounding to bfloat16, used by the
              emulation modes that reproduce the GPU path's declared
              rounding points in otherwise-fp64 arithmetic.

Pins (what this oracle is checked against, independently of itself) live in
``tests/test_oracle_*.py`` and ``tests/golden/``.  Every function here has at
least one pin; none is "parity unpinned".
"""

from . import bf16, ns, muon, qr, soap  # noqa: F401
