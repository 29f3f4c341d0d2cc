"""Restatement of the library's split-KV decode plan, for bit-exact bookkeeping checks.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The plan is a scheduling choice of this library (the pages give none); it is
restated here from the formula documented beside ``attn_decode_plan`` in the C
header so that tests can compare the two integer for integer.  Any plan gives the
same attention result; the decode parity tests check that.

* heads per CTA ``G``: the largest of 8, 4, 2, 1 that divides ``g = Hq / Hkv``;
* independent streams ``U = B * Hkv * (g / G)``;
* splits wanted ``ceil(TARGET_CTAS / U)`` with ``TARGET_CTAS = 1184``, clamped to
  ``[1, min(128, max(1, ceil(max_seqlen / 512)))]``;
* ``chunk = 64 * ceil(ceil(max_seqlen / splits) / 64)`` tokens per split (at least 64);
* ``max_splits = max(1, ceil(max_seqlen / chunk))``;
* sequence ``b`` uses ``ceil(seqlen_b / chunk)`` splits.
"""

from __future__ import annotations

__all__ = ["decode_plan_ref", "decode_heads_per_cta_ref", "TARGET_CTAS"]

TARGET_CTAS = 1184
MAX_SPLITS = 128


def _cdiv(a: int, b: int) -> int:
    return -(-a // b)


def decode_heads_per_cta_ref(hq: int, hkv: int) -> int:
    g = hq // hkv
    for cand in (8, 4, 2, 1):
        if g % cand == 0:
            return cand
    return 1


def decode_plan_ref(batch: int, hq: int, hkv: int, max_seqlen: int):
    """Return ``(chunk_tokens, max_splits, heads_per_cta)``."""
    if batch <= 0 or hkv <= 0 or hq <= 0 or hq % hkv or max_seqlen < 0:
        raise ValueError("bad decode plan arguments")
    g = hq // hkv
    G = decode_heads_per_cta_ref(hq, hkv)
    streams = batch * hkv * (g // G)
    splits = _cdiv(TARGET_CTAS, streams)
    splits = max(1, min(splits, max(1, _cdiv(max_seqlen, 512)), MAX_SPLITS))
    chunk = max(64, 64 * _cdiv(_cdiv(max(max_seqlen, 1), splits), 64))
    max_splits = max(1, _cdiv(max_seqlen, chunk))
    return chunk, max_splits, G
