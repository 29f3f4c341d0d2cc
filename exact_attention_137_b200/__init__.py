"""Exact grouped-query attention for NVIDIA B200 (sm_100a).

The compute lives in the C-ABI library ``libattn137.so`` (``include/attn.h``);
this package is a thin binding plus seeded synthetic inputs (``workloads``).

* ``attn_fwd(q, k, v, causal, scale)`` -- prefill forward returning ``(O, LSE)``.
* ``attn_decode(q, k_cache, v_cache, seqlens, max_seqlen, block_table=None)`` --
  single-token decode over a contiguous or paged KV cache.
* ``kv_cache_bytes``, ``paged_pool_blocks``, ``decode_plan`` -- host-side sizing.
"""

from ._lib import (  # noqa: F401
    AttnError,
    attn_bwd,
    attn_decode,
    attn_decode_fp8,
    attn_fwd,
    decode_check,
    decode_plan,
    decode_workspace,
    decode_workspace_bytes,
    device_status,
    kv_cache_bytes,
    load,
    paged_pool_blocks,
    paged_pool_bytes,
)

__all__ = [
    "AttnError",
    "attn_bwd",
    "attn_decode",
    "attn_decode_fp8",
    "attn_fwd",
    "decode_check",
    "decode_plan",
    "decode_workspace",
    "decode_workspace_bytes",
    "device_status",
    "kv_cache_bytes",
    "load",
    "paged_pool_blocks",
    "paged_pool_bytes",
]
