"""CPU oracle of the DSA forward path (fp64) -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s ``cpu_baseline`` / ``--impl reference`` legs
may import this package.  The product path (``sparse_attention_long_05_b200``) never does.

Parity status of each function (what pins it is in ``tests/test_oracle.py``):
  e4m3_table, bf16_to_f64      pinned: format definition values + torch's float8/bfloat16 conversions
  indexer_scores_row           pinned: hand-worked golden example, |x| identity route, int64 exactness,
                               invariants (w >= 0, head / dim permutations, q_I = 0)
  topk_row                     pinned: golden example, pairwise dominance brute force, q_I = 0 case,
                               argpartition on distinct values, n <= k case
  attention_row                pinned: golden example, torch scaled_dot_product_attention (fp64) on dense
                               causal rows, q = 0 closed form, k = 1, permutation invariance, logsumexp
  prefill_rows, decode_row     pinned: pure-Python brute force on micro sequences, t < k dense invariant
  indexer_kl_row               pinned: hand-worked closed form (two heads, three keys), zero divergence when
                               I = log p + const, invariance to a constant shift of I, non-negativity,
                               pure-Python brute force
"""
from .dsa_oracle import *  # noqa: F401,F403
from .dsa_oracle import __all__  # noqa: F401
