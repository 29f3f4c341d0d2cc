"""Gradients of exact attention in fp64: the definition differentiated, written out.

TEST INFRASTRUCTURE ONLY (see the package docstring).

CSDN interview article «注意力变体深挖» §6.2 (technique 2, recomputation) and 追问2/追问3:
the backward pass does not keep the attention matrix; it recomputes it from the saved
Q, K, V, which keeps memory O(n).  The pages print no gradient formulas; those below are
the plain derivative of ``O = softmax(scale * Q K^T + mask) V`` (readings 2, 3 and 6 of
``oracle/attention.py`` for the mask), with P recomputed here from Q, K and the forward's
LSE exactly as a recomputing backward does:

* ``P_ij = exp(scale * q_i . k_j - LSE_i)`` on allowed pairs, 0 elsewhere;
* ``dV = P^T dO``;  ``dP = dO V^T``;
* ``Delta_i = sum_j P_ij dP_ij = dO_i . O_i``;  ``dS = P * (dP - Delta)``;
* ``dQ = scale * dS K``;  ``dK = scale * dS^T Q``;
* GQA: K/V head ``h // g`` serves query head ``h``, so dK and dV of a KV head are the sums
  over its ``g`` query heads.
"""

from __future__ import annotations

import numpy as np

from .attention import _check_heads, _default_scale, allowed_mask, attention_ref

__all__ = ["attention_bwd_ref"]


def attention_bwd_ref(q, k, v, dout, causal: bool = False, scale=None, window: int = 0):
    """``(dQ, dK, dV)`` for ``q [B,Hq,Sq,D]``, ``k``/``v`` ``[B,Hkv,Sk,D]``, ``dout [B,Hq,Sq,D]``."""
    q, k, v, dout = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dout))
    b_, hq, sq, d = q.shape
    _, hkv, sk, _ = k.shape
    g = _check_heads(hq, hkv)
    sc = _default_scale(d, scale)
    o, lse = attention_ref(q, k, v, causal=causal, scale=scale, window=window)
    allowed = allowed_mask(sq, sk, causal, None, window)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(b_):
        for h in range(hq):
            kh = h // g
            s = (q[b, h] @ k[b, kh].T) * sc
            has = np.isfinite(lse[b, h])
            p = np.zeros_like(s)
            ex = np.exp(s - np.where(has, lse[b, h], 0.0)[:, None])
            p[has] = np.where(allowed[has], ex[has], 0.0)
            dv[b, kh] += p.T @ dout[b, h]
            dp = dout[b, h] @ v[b, kh].T
            delta = np.sum(dout[b, h] * o[b, h], axis=1)
            ds = p * (dp - delta[:, None])
            dq[b, h] = sc * (ds @ k[b, kh])
            dk[b, kh] += sc * (ds.T @ q[b, h])
    return dq, dk, dv
