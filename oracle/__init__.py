"""fp64 CPU oracle for exact grouped-query attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
anything in this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it.  It shares
no code, tables or constants with the CUDA library in ``exact_attention_137_b200``.

What it computes, and where the pages define it (page titles abbreviated):

* ``attention_ref`` / ``attention_rows_ref`` -- softmax(Q K^T * scale) V per head with
  K/V heads repeated to the query heads (CSDN interview article «注意力变体深挖»,
  §五 ``grouped_query_attention``; gocoding blog «different attention mechanisms»,
  §1 and §3), plus the row log-sum-exp of the scaled scores.
* ``flash_blockwise_ref`` -- the tiled online-softmax forward of the same CSDN
  article, §6.2, which the pages say equals one-shot softmax exactly.
* ``brute_force_attention`` -- scalar-loop restatement for tiny inputs.
* ``decode_ref`` -- one new query token against a contiguous or paged KV cache
  (CSDN §七 KV cache; gocoding §5 PagedAttention page table).
* ``kv_cache_bytes_ref`` / ``paged_pool_blocks_ref`` -- the KV-cache size formula
  (kongchang course summary, "MHA、GQA与MQA"; CSDN §七).
* ``decode_plan_ref`` -- restatement of the library's split-KV plan formula (a
  scheduling choice of this library, not of the pages), for bit-exact checks.

Readings of points the pages leave open are listed in the module docstrings.
Every function here is pinned by ``tests/test_oracle.py`` against closed forms,
invariants, scalar brute force, the pages' printed KV-cache sizes and torch's
float64 CPU ``scaled_dot_product_attention``.
"""

from .attention import (
    attention_ref,
    attention_rows_ref,
    brute_force_attention,
    decode_ref,
    flash_blockwise_ref,
    allowed_mask,
)
from .backward import attention_bwd_ref
from .kvcache import e4m3_decode, e4m3_value, kv_cache_bytes_ref, paged_pool_blocks_ref
from .plan import decode_plan_ref, decode_heads_per_cta_ref, decode_schedule_ref

__all__ = [
    "attention_ref",
    "attention_bwd_ref",
    "attention_rows_ref",
    "brute_force_attention",
    "decode_ref",
    "flash_blockwise_ref",
    "allowed_mask",
    "kv_cache_bytes_ref",
    "paged_pool_blocks_ref",
    "e4m3_value",
    "e4m3_decode",
    "decode_plan_ref",
    "decode_schedule_ref",
    "decode_heads_per_cta_ref",
]
