"""CPU oracle for load-balanced split-KV decode attention. This is TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` may import it. The product path (``load_balanced_split_step_b200``) never
imports or calls anything here. This package shares no code with the CUDA library:
no kernels, headers, helpers, tables or constants. Both sides receive the same inputs
from ``load_balanced_split_step_b200.workloads``, which holds only random draws and
data layout.

Everything here is plain, slow, fp64 numpy that a reader can check against the
definitions by eye:

* ``attention.decode_attention``: softmax(scale * q K^T) V for every request and query
  head over the request's paged cache. This is the exact result that the split-KV method
  reaches up to rounding order.
* ``planner.plan_dynamic`` / ``planner.plan_static``: the per-step tile planner, unit by
  unit, and the static split-k plan it replaces.
* ``merge``: per-split softmax states and their log-sum-exp merge.
* ``prologue``: RMSNorm, NeoX RoPE and the KV-page write of the new token.
* ``fp8``: OCP E4M3 decode and encode (round to nearest even, saturating).

Pins (tests/test_oracle_*.py) tie each function to something other than itself:
library routines, closed forms, brute force on tiny inputs, invariants, and planted
mistakes that the pins must catch. The pages print no worked numerical example for the
attention value, so its pins are the definition's own: fp64 SDPA, brute force and closed
forms.
"""
