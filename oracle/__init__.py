"""Plain, slow, fp64 CPU oracle for the Muon update.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import anything here.  The
CUDA library never calls, links or imports this package, and this package
imports nothing from the CUDA library.

Sources (web pages; quoted by title and section only):

* [Guide]  "NanoGPT Speedrun: The Ultimate Guide to Pushing LLM Training
  Efficiency to Its Limits" (kongchang.com), section "Optimizer and Training
  Strategy Tuning", paragraph on Muon: the gradient matrix is orthogonalised
  after a Nesterov-momentum update, by Newton-Schulz iteration; Muon is used
  for hidden matrices only.
* [Overview] "The NanoGPT speedrun" (sbabichenko.com, notes/speedrun),
  paragraph "Six records account for most of the speedup", record #3: each
  hidden matrix's momentum update is replaced by its nearest semi-orthogonal
  matrix through five Newton-Schulz steps, at most T*m/B ~ 0.7 % extra FLOPs
  with T = 5, m = 768, B = 524,288.

Where the pages are silent, the library's specification fixes the iteration
form X <- aX + (bA + cA^2)X with A = X X^T, the coefficient triple
(3.4445, -4.7750, 2.0315), Frobenius normalisation, the transpose to
rows <= cols, and "then scaled and applied".  The remaining open points are
read as documented in each function.

Modules
-------
``muon``      fp64 definitions: normalisation, Newton-Schulz, momentum,
              scale rule, apply, the full step, FLOP accounting.
``fp32_ref``  fp32 restatement of the memory-bound steps in the exact
              operation order the kernels use (for bit-exact checks).
``jacobi``    one-sided Jacobi SVD for tiny inputs (brute-force polar factor).

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
(closed forms, invariants, special cases, brute force); none is unpinned.
"""
