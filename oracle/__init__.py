"""fp64 CPU oracle for the KATA causal forward (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg (including its ``--impl reference`` arm) import this package. The CUDA
library under ``kernelized_linear_attention_kata_b200/`` shares no code with it
and never imports it.

Parity status per function (what pins it is listed in tests/test_oracle_pins.py):

* forward_brute_force, forward_rows      -- pinned (closed forms, hand-worked
  fixtures, invariances, convex hull).
* forward_recurrent_unpacked / forward_recurrent / forward_chunked /
  forward_chunked_scanned / forward_gated / decode_step(_batched)
                                         -- pinned against the brute force and
  against each other on tiny inputs, plus the same closed forms.
* exclusive_tree_scan                    -- pinned against a running sum.
* backward_brute_force, backward_rows (oracle/backward.py)
                                         -- pinned by central finite
  differences of forward_brute_force and by closed forms (T = 1, the
  normalisation identity, PSD homogeneity, equal keys, q = 0).
* the first-order feature phi_1(u) = [1, u] -- the arithmetic is pinned (hand
  fixture, forms agreement), but the READING that this is the pages'
  "first-order feature" is not fixed by the pages: parity of that reading is
  unpinned.
* KATA-Mg, KATA-Sigma-g and DeltaKATA (oracle/variants.py) -- the pages only
  name them; the arithmetic of each reading is pinned
  (tests/test_oracle_variants.py: reductions to the rank-one oracle, closed
  forms, invariances, an unpacked delta rule), parity of the readings is
  unpinned.
"""

from .kata import *  # noqa: F401,F403
from .kata import (  # noqa: F401
    FEATURES, FIRST_ORDER, PSD, chunk_deltas, decode_step, decode_step_batched,
    exclusive_tree_scan, final_state, first_order_feature, forward_brute_force,
    forward_chunked, forward_chunked_scanned, forward_gated, forward_recurrent,
    forward_recurrent_unpacked, forward_rows, key_feature, per_head, psd_key_feature,
    psd_pairs, psd_query_feature, query_feature, state_dim, weights,
)
from .backward import backward_brute_force, backward_rows  # noqa: F401
from . import variants  # noqa: F401
