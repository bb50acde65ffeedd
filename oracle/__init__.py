"""CPU fp64 oracle for exact blockwise attention.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import or run anything in this
package.  The product path (the C-ABI library and its Python binding) never
touches it, and this package never touches the product path: the two share no
code, only the seeded input tensors from ``seeded_inputs``.

Sources (page title, then section):

* TokenRing review (pith.science, arXiv 2412.20501), "What carries the
  argument": the partial-output update rule
  ``out <- out - sigma(block_lse - lse) * (out - block_out)`` and
  ``lse <- lse - ln sigma(lse - block_lse)``.
* same page, "Core claim" and "Referee Report / Summary": Q, K, V are split
  along the token dimension into blocks; a flash-attention kernel returns
  ``(block_out, block_lse)`` per (Q block, KV block); the partials are merged.
* same page, "Assumptions & free parameters" (standard math) and "Referee
  Report / Significance": the merge reproduces standard attention exactly.
* same page, "If this is right": zigzag causal partition for load balance;
  grouped / multi-query attention.
* same page, "Referee Report / major comments, Algorithm 1 (section 3.2)": the
  TokenRing step index t = (j - step + 1) mod N.
* Anthology of the SOTA, SOTA-181 (Liu et al. 2023, ring attention): blocks on
  a ring, each device keeps its query block and passes its key/value block to
  its neighbour; the attention is unchanged and exact.

Modules:

* ``attention``  - plain full softmax attention (the definition), fp64.
* ``blockwise``  - partitions, ring / TokenRing schedules, per-block partials
  and the pages' merge rule, fp64.  Shares no code with ``attention``.
* ``backward``   - gradients (dq, dk, dv): the definition over whole rows and
  the same gradient as sums over block pairs rebuilt from the full-row lse.

Every function here is pinned by ``tests/test_oracle.py`` against brute force,
closed forms, a library routine or an invariant the pages fix.  The timing
columns of the pages (7.6 ms / 3.5 ms on four A10s) are "parity unpinned": they
need hardware and a model shape the pages do not give.
"""
from . import attention, backward, blockwise  # noqa: F401
