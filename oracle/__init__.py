"""Oracle for the activation-sparse FFN decode path: TEST INFRASTRUCTURE ONLY.

A plain fp64 CPU statement of what the path computes (numpy, no blocking or fusion).
Only `tests/`, `__graft_entry__.smoke()` and the benchmark's CPU-baseline leg may
import it.  It never imports the library and the library never imports it; the two
share only the seeded input generators in `pi_synth`.

Parity status per function (pins live in tests/test_oracle_*.py):
  q4_0_unpack, predictor_logits, fire_bits, pack_mask/unpack_mask, compact,
  activations, sparse_ffn, dense_ffn, true_mask, down_accumulate, stack_glue,
  hot_order, permute_layer, hot_prefix_len, hot_fraction_for_mass: pinned.
  decode_stack, layer_step: compositions of pinned functions (pinned through them).
"""
from .ffn import *  # noqa: F401,F403
from . import ffn  # noqa: F401
