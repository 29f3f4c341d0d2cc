"""Plain fp64 attention: the definition written out, no tiling, no fusion.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources (page titles abbreviated; the pages are explainers, none prints a kernel):

* CSDN interview article «注意力变体深挖», §五: the NumPy ``grouped_query_attention``
  fixes the layout ``[batch, heads, seq, d_head]``, the default scale
  ``1/sqrt(d_head)``, the precondition ``Hq % Hkv == 0``, the max-subtracted softmax
  and the head mapping: K/V are repeated ``group_size = Hq // Hkv`` times along the
  head axis, so query head ``h`` reads K/V head ``h // group_size``.
* gocoding blog «different attention mechanisms», §1: per head
  ``softmax(Q_i K_i^T / sqrt(d_k)) V_i``; §3 GQA: N query heads in G groups;
  §5 PagedAttention: a per-sequence page table maps logical to physical blocks.
* CSDN §6.2: the tiled online-softmax forward (``flash_blockwise_ref``).
* CSDN §七: with a KV cache each step computes only the new token's Q against the
  cached K/V.

Readings where the pages are silent or garbled:

1. CSDN §6.2 uses ``Sij_softmax`` without defining it.  It is read as the block-local
   *unnormalised* ``exp(Sij - block_max)``: that is the only reading under which the
   final ``O / row_sum`` is right (a normalised block softmax would divide twice).
2. Causal masking is never defined.  Key ``j`` is allowed for query ``i`` iff
   ``j <= i + Sk - Sq`` (lower triangle when ``Sq == Sk``; bottom-right aligned
   otherwise, so a decode step equals the last row of a causal prefill).
3. A query row with no allowed key (``Sq > Sk`` causal rows, or ``seqlen == 0`` in
   decode) returns ``O = 0`` and ``LSE = -inf``.
4. The log-sum-exp is not on the pages.  ``LSE_i = ln sum_j exp(scale * q_i . k_j)``
   over allowed ``j`` (natural log of the *scaled* scores).
5. ``scale`` is explicit; ``None`` means ``1/sqrt(D)`` (CSDN §五 default).
6. Sliding-window attention is named on the CSDN page (追问4, among the long-context
   KV-cache optimisations) but not defined.  With a window ``W >= 1`` a query at
   absolute position ``p = i + Sk - Sq`` attends to keys ``p - W < j <= p``: causal,
   bottom-right aligned as in reading 2, and ``W`` keys including its own.  A decode
   step (``p = seqlen - 1``) therefore attends to the last ``W`` cached tokens.
   ``W <= 0`` means no window.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "allowed_mask",
    "attention_ref",
    "attention_rows_ref",
    "brute_force_attention",
    "decode_ref",
    "flash_blockwise_ref",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _default_scale(d: int, scale):
    # CSDN §五: ``scale = 1.0 / np.sqrt(d_head)`` when not given.
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def allowed_mask(sq: int, sk: int, causal: bool, rows=None, window: int = 0) -> np.ndarray:
    """Boolean ``[len(rows), sk]``: may query row ``i`` attend to key ``j``? (readings 2, 6)."""
    rows = np.arange(sq) if rows is None else np.asarray(rows, dtype=np.int64)
    cols = np.arange(sk)
    if not causal:
        if window > 0:
            raise ValueError("a sliding window is defined for causal attention only")
        return np.ones((rows.size, sk), dtype=bool)
    pos = rows[:, None] + (sk - sq)  # absolute position of the query
    allowed = cols[None, :] <= pos
    if window > 0:
        allowed &= cols[None, :] > pos - window
    return allowed


def _softmax_times_v(s: np.ndarray, allowed: np.ndarray, v: np.ndarray):
    """Rows of ``softmax(s) @ v`` with masked entries removed, plus the row LSE.

    Max-subtracted softmax as in CSDN §五 ``softmax``; fully masked rows follow
    reading 3.
    """
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1)
    has = np.isfinite(m)
    m0 = np.where(has, m, 0.0)
    p = np.exp(s - m0[:, None])  # masked entries: exp(-inf) = 0
    l = p.sum(axis=1)
    o = np.zeros((s.shape[0], v.shape[1]), dtype=np.float64)
    if has.any():
        o[has] = (p[has] @ v) / l[has, None]
    lse = np.full(s.shape[0], -np.inf)
    lse[has] = m0[has] + np.log(l[has])
    return o, lse


def _check_heads(hq: int, hkv: int) -> int:
    # CSDN §五: ``assert num_query_heads % num_kv_heads == 0``.
    if hkv <= 0 or hq % hkv != 0:
        raise ValueError(f"query heads {hq} must be a multiple of kv heads {hkv}")
    return hq // hkv


def attention_rows_ref(q, k, v, causal: bool = False, scale=None, rows=None, window: int = 0):
    """Exact attention for a subset of query rows (all rows when ``rows is None``).

    ``q``: ``[B, Hq, Sq, D]``; ``k``, ``v``: ``[B, Hkv, Sk, D]``.  Returns
    ``O [B, Hq, R, D]`` and ``LSE [B, Hq, R]`` for the ``R`` selected rows, each
    computed over its full allowed key range (so a sampled row is exactly the row
    of the full result).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    b_, hq, sq, d = q.shape
    _, hkv, sk, dv = v.shape
    g = _check_heads(hq, hkv)
    sc = _default_scale(d, scale)
    rows = np.arange(sq) if rows is None else np.asarray(rows, dtype=np.int64)
    # CSDN §五: ``k = np.repeat(k, group_size, axis=1)`` -- query head h reads K/V head h // g.
    k_rep = np.repeat(k, g, axis=1)
    v_rep = np.repeat(v, g, axis=1)
    allowed = allowed_mask(sq, sk, causal, rows, window)
    o = np.zeros((b_, hq, rows.size, dv))
    lse = np.zeros((b_, hq, rows.size))
    for b in range(b_):
        for h in range(hq):
            s = (q[b, h, rows] @ k_rep[b, h].T) * sc  # scores = Q @ K^T * scale
            o[b, h], lse[b, h] = _softmax_times_v(s, allowed, v_rep[b, h])
    return o, lse


def attention_ref(q, k, v, causal: bool = False, scale=None, window: int = 0):
    """Exact GQA attention, all rows: ``O [B, Hq, Sq, D]``, ``LSE [B, Hq, Sq]``."""
    return attention_rows_ref(q, k, v, causal=causal, scale=scale, rows=None, window=window)


def flash_blockwise_ref(q, k, v, block_q: int, block_kv: int, scale=None):
    """Tiled online-softmax forward of one head, CSDN «注意力变体深挖» §6.2.

    ``q``: ``[Nq, d]``, ``k``/``v``: ``[Nk, d]``; non-causal, as on the page.  Outer
    loop over query blocks, inner loop over key/value blocks; per block the block row
    max and the sum of ``exp(S - block_max)`` are merged into the running max and
    denominator, the old partial output is rescaled by ``exp(old_max - new_max)``, and
    the final output is divided by the running sum (reading 1 for ``Sij_softmax``).
    Also returns the row LSE ``row_max + ln(row_sum)`` (reading 4).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    nq, d = q.shape
    nk = k.shape[0]
    sc = _default_scale(d, scale)
    out = np.zeros((nq, v.shape[1]))
    lse = np.zeros(nq)
    for i in range(0, nq, block_q):
        qi = q[i : i + block_q]
        oi = np.zeros((qi.shape[0], v.shape[1]))
        row_sum = np.zeros(qi.shape[0])
        row_max = np.full(qi.shape[0], -np.inf)
        for j in range(0, nk, block_kv):
            kj = k[j : j + block_kv]
            vj = v[j : j + block_kv]
            sij = (qi @ kj.T) * sc
            block_max = sij.max(axis=1)
            pij = np.exp(sij - block_max[:, None])  # reading 1: unnormalised block exponentials
            block_sum = pij.sum(axis=1)
            new_max = np.maximum(row_max, block_max)
            old_w = np.exp(row_max - new_max)
            blk_w = np.exp(block_max - new_max)
            oi = oi * old_w[:, None] + blk_w[:, None] * (pij @ vj)
            row_sum = row_sum * old_w + block_sum * blk_w
            row_max = new_max
        out[i : i + block_q] = oi / row_sum[:, None]
        lse[i : i + block_q] = row_max + np.log(row_sum)
    return out, lse


def brute_force_attention(q, k, v, causal: bool = False, scale=None, window: int = 0):
    """Scalar-loop attention for tiny inputs (nested lists in, nested lists out).

    Independent of the NumPy path: every score, exponential and sum is a Python
    float operation (``math.fsum`` for sums).  Same head mapping, mask and
    conventions as the module readings.
    """
    bsz = len(q)
    hq = len(q[0])
    sq = len(q[0][0])
    d = len(q[0][0][0])
    hkv = len(k[0])
    sk = len(k[0][0])
    if hq % hkv:
        raise ValueError("query heads must be a multiple of kv heads")
    g = hq // hkv
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out, lse = [], []
    for b in range(bsz):
        ob, lb = [], []
        for h in range(hq):
            kvh = h // g
            oh, lh = [], []
            for i in range(sq):
                p = i + sk - sq
                keys = [j for j in range(sk) if (not causal) or (j <= p and (window <= 0 or j > p - window))]
                if not keys:
                    oh.append([0.0] * len(v[b][kvh][0]))
                    lh.append(-math.inf)
                    continue
                s = {j: sc * math.fsum(float(q[b][h][i][e]) * float(k[b][kvh][j][e]) for e in range(d)) for j in keys}
                m = max(s.values())
                w = {j: math.exp(s[j] - m) for j in keys}
                den = math.fsum(w.values())
                dv = len(v[b][kvh][0])
                oh.append([math.fsum(w[j] * float(v[b][kvh][j][e]) for j in keys) / den for e in range(dv)])
                lh.append(m + math.log(den))
            ob.append(oh)
            lb.append(lh)
        out.append(ob)
        lse.append(lb)
    return out, lse


def decode_ref(q, k_cache, v_cache, seqlens, block_table=None, block_size=None, scale=None, window: int = 0):
    """One query token per sequence against its cached keys/values.

    ``q``: ``[B, Hq, D]``.  Contiguous cache (``block_table is None``):
    ``k_cache``/``v_cache`` ``[B, Hkv, cap, D]`` and sequence ``b`` owns tokens
    ``0 .. seqlens[b]-1``.  Paged cache: a pool ``[num_blocks, Hkv, block_size, D]``;
    logical token ``t`` of sequence ``b`` lives in physical block
    ``block_table[b][t // block_size]`` at slot ``t % block_size`` (gocoding §5 page
    table).  The gather is a host loop over the page table; the new token attends
    to every cached token (CSDN §七), so no causal mask applies.  ``seqlens[b]``
    counts the cached tokens including the current one.  With ``window >= 1`` only the
    last ``window`` of them are attended to (reading 6).  Returns ``O [B, Hq, D]`` and
    ``LSE [B, Hq]``.
    """
    q = _f64(q)
    bsz, hq, d = q.shape
    hkv = k_cache.shape[1]
    g = _check_heads(hq, hkv)
    sc = _default_scale(d, scale)
    dv = v_cache.shape[-1]
    out = np.zeros((bsz, hq, dv))
    lse = np.full((bsz, hq), -np.inf)
    for b in range(bsz):
        n = int(seqlens[b])
        if n <= 0:
            continue
        kb = np.empty((hkv, n, d))
        vb = np.empty((hkv, n, dv))
        if block_table is None:
            kb[:] = k_cache[b, :, :n]
            vb[:] = v_cache[b, :, :n]
        else:
            bs = int(block_size)
            for i in range((n + bs - 1) // bs):
                blk = int(block_table[b][i])
                cnt = min(bs, n - i * bs)
                kb[:, i * bs : i * bs + cnt] = k_cache[blk, :, :cnt]
                vb[:, i * bs : i * bs + cnt] = v_cache[blk, :, :cnt]
        visible = np.ones((1, n), dtype=bool)
        if window > 0:
            visible[0, : max(0, n - window)] = False
        for h in range(hq):
            s = (kb[h // g] @ q[b, h]) * sc
            o, l = _softmax_times_v(s[None, :], visible, vb[h // g])
            out[b, h] = o[0]
            lse[b, h] = l[0]
    return out, lse
