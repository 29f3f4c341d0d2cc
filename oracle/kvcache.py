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

__all__ = ["kv_cache_bytes_ref", "paged_pool_blocks_ref", "e4m3_value", "e4m3_decode"]


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


# ---------------------------------------------------------------- fp8 KV cache
#
# The CSDN page («注意力变体深挖», 追问4) lists quantising the KV cache to fp8/int4 among
# the long-context optimisations without fixing a format.  Reading: K and V are stored as
# OCP FP8 E4M3 codes (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent
# field 0 is subnormal; no infinities; S.1111.111 is NaN; largest finite value 448), and
# the cached value is the code's value times one fp32 scale per tensor (one for K, one for
# V).  The decoder below is that definition written out.


def e4m3_value(code: int) -> float:
    """Value of one E4M3 code (0..255) as a Python float (NaN for S.1111.111)."""
    code = int(code)
    if not 0 <= code <= 255:
        raise ValueError("an E4M3 code is one byte")
    sign = -1.0 if code & 0x80 else 1.0
    exp = (code >> 3) & 0xF
    man = code & 0x7
    if exp == 0xF and man == 0x7:
        return float("nan")
    if exp == 0:
        return sign * (man / 8.0) * 2.0 ** (1 - 7)  # subnormal: 0.mmm * 2^-6
    return sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)


_E4M3_TABLE = None


def e4m3_decode(codes, scale: float = 1.0):
    """float64 array of ``scale * value(code)`` for an array of E4M3 codes (uint8)."""
    import numpy as np

    global _E4M3_TABLE
    if _E4M3_TABLE is None:
        _E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
    return _E4M3_TABLE[np.asarray(codes, dtype=np.uint8)] * float(scale)
