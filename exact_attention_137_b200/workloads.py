"""Seeded synthetic inputs shared by the tests, the bench and the smoke run.

This module holds no attention arithmetic: it draws random numbers, rounds them to
the storage dtype, builds page tables, and converts tensors for the fp64 checker.

Recipe (every draw is seeded):

* ``torch.Generator('cpu').manual_seed(seed)`` draws q, then k, then v as fp32
  N(0, 1); bf16 storage rounds them to nearest-even (``Tensor.to``).
* ``numpy.random.Generator(PCG64(seed))`` draws sequence lengths, the physical block
  permutation of a paged pool and the rows of spiked keys.
* Spiked keys (long-context stress input): per (batch, kv head) ``round(frac * Sk)``
  distinct key rows are multiplied by a power of two after rounding, which bf16
  represents exactly.
* KV-cache slots at or beyond a sequence's length hold NaN, so any read past the
  valid tokens poisons the output.
* fp8 caches (``kv_dtype="fp8"``): the same fp32 draws divided by a per-tensor scale of
  ``2^-6``, clamped to +-448 and rounded to OCP FP8 E4M3 codes (``torch.float8_e4m3fn``),
  stored as uint8; unused slots hold the NaN code 0x7F.
"""

from __future__ import annotations

import math

import numpy as np
import torch

__all__ = [
    "prefill_inputs",
    "decode_contiguous_inputs",
    "decode_paged_inputs",
    "to_f64",
    "torch_dtype",
]


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32, "fp32": torch.float32}[name]


def _randn(shape, gen: torch.Generator, dtype: torch.dtype, chunk_elems: int = 1 << 26) -> torch.Tensor:
    """N(0,1) fp32 draws rounded to ``dtype``, produced in chunks to bound memory, on the
    generator's device."""
    out = torch.empty(shape, dtype=dtype, device=gen.device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        flat[s:e] = torch.randn(e - s, generator=gen, dtype=torch.float32, device=gen.device).to(dtype)
    return out


def prefill_inputs(B: int, Hq: int, Hkv: int, Sq: int, Sk: int, D: int, dtype: str = "bf16",
                   seed: int = 0, spike_frac: float = 0.0, spike_factor: float = 8.0):
    """q ``[B,Hq,Sq,D]``, k/v ``[B,Hkv,Sk,D]`` on the CPU; returns a dict.

    ``spike_frac > 0`` multiplies ``round(spike_frac * Sk)`` distinct key rows per
    (b, kv head) by ``spike_factor`` (the rows are returned as ``spike_rows``).
    """
    dt = torch_dtype(dtype)
    gen = torch.Generator("cpu").manual_seed(seed)
    q = _randn((B, Hq, Sq, D), gen, dt)
    k = _randn((B, Hkv, Sk, D), gen, dt)
    v = _randn((B, Hkv, Sk, D), gen, dt)
    spike_rows = None
    if spike_frac > 0:
        if math.log2(spike_factor) != int(math.log2(spike_factor)):
            raise ValueError("spike_factor must be a power of two (exact in bf16)")
        n_spike = int(round(spike_frac * Sk))
        rng = np.random.Generator(np.random.PCG64(seed))
        spike_rows = np.zeros((B, Hkv, n_spike), dtype=np.int64)
        for b in range(B):
            for h in range(Hkv):
                rows = np.sort(rng.choice(Sk, size=n_spike, replace=False))
                spike_rows[b, h] = rows
                idx = torch.from_numpy(rows)
                k[b, h, idx] = k[b, h, idx] * spike_factor
    return {"q": q, "k": k, "v": v, "spike_rows": spike_rows}


def _lengths(rng: np.random.Generator, B: int, lo: int, hi: int) -> np.ndarray:
    return rng.integers(lo, hi + 1, size=B).astype(np.int32)


def decode_contiguous_inputs(B: int, Hq: int, Hkv: int, D: int, cap: int, len_lo: int, len_hi: int,
                             seed: int = 0, seqlens=None, kv_dtype: str = "bf16"):
    """One query token per sequence and a dense cache ``[B,Hkv,cap,D]`` (bf16).

    Lengths are uniform in ``[len_lo, len_hi]`` unless ``seqlens`` is given; slots at
    or beyond a length hold NaN.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = _lengths(rng, B, len_lo, len_hi) if seqlens is None else np.asarray(seqlens, dtype=np.int32)
    if lens.max(initial=0) > cap:
        raise ValueError("a length exceeds the cache capacity")
    gen = torch.Generator("cpu").manual_seed(seed)
    q = _randn((B, Hq, D), gen, torch.bfloat16)
    k = _randn((B, Hkv, cap, D), gen, torch.bfloat16)
    v = _randn((B, Hkv, cap, D), gen, torch.bfloat16)
    for b in range(B):
        k[b, :, int(lens[b]):] = float("nan")
        v[b, :, int(lens[b]):] = float("nan")
    out = {"q": q, "k_cache": k, "v_cache": v, "seqlens": torch.from_numpy(lens),
           "block_table": None, "block_size": cap, "max_seqlen": int(lens.max(initial=0))}
    return _fp8_cache(out) if kv_dtype == "fp8" else out


FP8_SCALE = 2.0 ** -6


def _to_fp8(x: torch.Tensor) -> torch.Tensor:
    """E4M3 codes (uint8) of ``x / FP8_SCALE`` (NaN stays NaN)."""
    y = (x.float() / FP8_SCALE).clamp(-448.0, 448.0)
    y = torch.where(torch.isnan(x.float()), x.float(), y)
    return y.to(torch.float8_e4m3fn).view(torch.uint8)


def _fp8_cache(x: dict) -> dict:
    x = dict(x)
    x["k_cache"] = _to_fp8(x["k_cache"])
    x["v_cache"] = _to_fp8(x["v_cache"])
    x["k_scale"] = x["v_scale"] = FP8_SCALE
    return x


def decode_paged_inputs(B: int, Hq: int, Hkv: int, D: int, block_size: int, len_lo: int, len_hi: int,
                        seed: int = 0, max_blocks: int | None = None, seqlens=None, extra_blocks: int = 0,
                        device=None, kv_dtype: str = "bf16"):
    """One query token per sequence and a paged pool ``[num_blocks,Hkv,block_size,D]`` (bf16).

    The pool has ``sum(ceil(len/block_size)) + extra_blocks`` blocks; a seeded
    permutation of the pool assigns physical blocks to the sequences' logical blocks
    in order.  ``block_table`` is int32 ``[B, max_blocks]`` padded with -1.  Slots
    past a sequence's last token, and every slot of unassigned blocks, hold NaN.

    ``device`` (timing-only inputs): draw q and the pool with a generator on that device,
    seeded the same way, instead of on the CPU; lengths and the table are unchanged.
    ``kv_dtype="fp8"`` returns the pool as E4M3 codes with ``k_scale``/``v_scale``.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = _lengths(rng, B, len_lo, len_hi) if seqlens is None else np.asarray(seqlens, dtype=np.int32)
    nblk = (lens.astype(np.int64) + block_size - 1) // block_size
    used = int(nblk.sum())
    total = used + int(extra_blocks)
    perm = rng.permutation(total)
    if max_blocks is None:
        max_blocks = max(1, -(-int(len_hi) // block_size), int(nblk.max(initial=0)))
    table = np.full((B, max_blocks), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        table[b, : nblk[b]] = perm[off : off + nblk[b]]
        off += int(nblk[b])
    gen = torch.Generator("cpu" if device is None else device).manual_seed(seed)
    q = _randn((B, Hq, D), gen, torch.bfloat16)
    k = _randn((total, Hkv, block_size, D), gen, torch.bfloat16)
    v = _randn((total, Hkv, block_size, D), gen, torch.bfloat16)
    for b in range(B):
        if nblk[b] == 0:
            continue
        tail = int(lens[b]) - (int(nblk[b]) - 1) * block_size
        last = int(table[b, nblk[b] - 1])
        k[last, :, tail:] = float("nan")
        v[last, :, tail:] = float("nan")
    if used < total:
        idx = torch.from_numpy(perm[used:].astype(np.int64)).to(k.device)
        k[idx] = float("nan")
        v[idx] = float("nan")
    out = {"q": q, "k_cache": k, "v_cache": v, "seqlens": torch.from_numpy(lens),
           "block_table": torch.from_numpy(table), "block_size": block_size,
           "max_seqlen": int(lens.max(initial=0)), "num_blocks": total}
    return _fp8_cache(out) if kv_dtype == "fp8" else out


def to_f64(t) -> np.ndarray:
    """Exact float64 copy of a (CPU or GPU) tensor for the fp64 checker."""
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu", torch.float64).numpy()
