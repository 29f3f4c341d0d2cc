"""KV-cache sizing, written out from the pages' formulas.

TEST INFRASTRUCTURE ONLY (see the package docstring).

* kongchang course summary, section "MHA、GQA与MQA": cache size is about
  ``2 x L x H_kv x d_head x b x bytes`` with L the sequence length and b the batch.
* CSDN interview article «注意力变体深挖», §七: ``2 x num_kv_heads x d_head x seq_len
  x num_layers x bytes_per_element``.

The two agree once both the layer and the batch factor are kept; the factor 2 counts
K and V.  Worked numbers printed on the pages live in ``tests/golden`` and pin this.
"""

from __future__ import annotations

__all__ = ["kv_cache_bytes_ref", "paged_pool_blocks_ref"]


def kv_cache_bytes_ref(layers: int, kv_heads: int, head_dim: int, seq_len: int,
                       batch: int, elem_bytes: int) -> int:
    """Bytes of a dense K+V cache: 2 * layers * kv_heads * head_dim * seq_len * batch * elem_bytes."""
    for x in (layers, kv_heads, head_dim, seq_len, batch, elem_bytes):
        if int(x) < 0:
            raise ValueError("sizes must be non-negative")
    return 2 * int(layers) * int(kv_heads) * int(head_dim) * int(seq_len) * int(batch) * int(elem_bytes)


def paged_pool_blocks_ref(seqlens, block_size: int) -> int:
    """Blocks a paged pool needs when every sequence gets ceil(len / block_size) blocks.

    gocoding blog §5 (PagedAttention): the cache is split into fixed-size blocks that are
    allocated on demand, so a sequence of ``len`` tokens holds ``ceil(len / block_size)``.
    """
    bs = int(block_size)
    if bs <= 0:
        raise ValueError("block_size must be positive")
    total = 0
    for n in seqlens:
        n = int(n)
        if n < 0:
            raise ValueError("sequence lengths must be non-negative")
        total += (n + bs - 1) // bs
    return total
