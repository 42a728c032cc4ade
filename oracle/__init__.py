"""CPU oracle for the BenQ and MDBF weight-only quantized linear layers.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.

It is a plain, slow, obviously correct restatement of what the two pages
define, written independently of the CUDA path (no shared code, tables or
constants).  Floating point is fp32 where the pages fix a stored type and fp64
for every contraction:

* ``oracle.benq``   -- "Qwen3.8-27B -- BenQ 6-bit", section "What BenQ stores":
  6-bit codes index a per-row 64-entry bf16 table; decode is a gather.
* ``oracle.mdbf``   -- "MDBF (Multi-Envelope Double Binary Factorization)",
  section "Algorithm": W ~= sum_p F_p G_p with envelope-scaled sign matrices.
* ``oracle.accounting`` -- the bits/weight table of the BenQ card and the
  MDBF "Bit-width and rank" / "The matrix shape caps the reachable BPW"
  formulas.

Every function is pinned by ``tests/test_oracle_*.py`` against facts the
pages or the mathematics fix (worked values, closed forms, library special
cases, exact rational brute force on tiny inputs).
"""
