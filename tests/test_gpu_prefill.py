"""Prefill parity: the CUDA path through the C ABI against the fp64 oracle.

Small shapes span several 128-row tiles, ragged tails, every head-grouping path of
the tensor-core kernel (head pairs, odd leftover head, MHA, MQA), Sq != Sk causal
alignment and fully masked rows; they are compared on every element.  The full-size
workloads (S=2048 head-sharing sweep, S=16384 long context with spiked keys) run in
the launch configuration the bench times and are compared on sampled rows, each
row exact over its whole visible key range.
"""

import numpy as np
import pytest
import torch

from oracle import attention_ref, attention_rows_ref
from exact_attention_137_b200 import _lib, attn_fwd, device_status
from exact_attention_137_b200.workloads import prefill_inputs, to_f64

from parity import BF16_TOL, F32_TOL, compare

pytestmark = pytest.mark.gpu


def _run(x, causal, scale=None):
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = attn_fwd(q, k, v, causal=causal, scale=scale)
    torch.cuda.synchronize()
    return o, lse


def _ref(x, causal, scale=None, rows=None):
    return attention_rows_ref(to_f64(x["q"]), to_f64(x["k"]), to_f64(x["v"]), causal=causal, scale=scale,
                              rows=rows)


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_fp32_config(cuda_lib, causal):
    # B=1, Hq=4, Hkv=2, Sq=Sk=128, D=64, fp32, seed 0, scale 1/sqrt(64).
    x = prefill_inputs(1, 4, 2, 128, 128, 64, dtype="f32", seed=0)
    o, lse = _run(x, causal)
    o_ref, l_ref = _ref(x, causal)
    compare(o, lse, o_ref, l_ref, F32_TOL, "fp32 tiny")


@pytest.mark.parametrize("shape", [(1, 4, 1, 70, 90, 128, True), (2, 2, 2, 33, 300, 64, False),
                                   (1, 3, 1, 200, 150, 128, True)])
def test_fp32_ragged(cuda_lib, shape):
    B, Hq, Hkv, Sq, Sk, D, causal = shape
    x = prefill_inputs(B, Hq, Hkv, Sq, Sk, D, dtype="f32", seed=3)
    o, lse = _run(x, causal)
    compare(o, lse, *_ref(x, causal), F32_TOL, f"fp32 {shape}")


BF16_SHAPES = [
    # B, Hq, Hkv, Sq, Sk, D, causal
    (1, 4, 2, 128, 128, 64, False),
    (1, 4, 2, 128, 128, 64, True),
    (1, 4, 2, 300, 300, 128, False),
    (1, 4, 2, 300, 300, 128, True),
    (2, 8, 1, 257, 257, 64, True),     # MQA, ragged tail
    (1, 3, 3, 520, 520, 128, True),    # MHA: odd groups, pairs of query tiles
    (1, 6, 2, 384, 384, 128, True),    # g = 3: a head pair plus a leftover head
    (1, 4, 2, 100, 300, 128, True),    # Sq < Sk: bottom-right aligned mask
    (1, 4, 2, 300, 100, 128, True),    # Sq > Sk: fully masked leading rows
    (1, 2, 1, 130, 129, 128, False),
    (1, 2, 1, 1, 1, 128, True),
    (1, 2, 2, 5, 7, 64, False),
    (3, 4, 4, 256, 640, 64, False),
]


@pytest.mark.parametrize("shape", BF16_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_bf16_small_all_elements(cuda_lib, shape):
    B, Hq, Hkv, Sq, Sk, D, causal = shape
    x = prefill_inputs(B, Hq, Hkv, Sq, Sk, D, dtype="bf16", seed=sum(shape))
    o, lse = _run(x, causal)
    compare(o, lse, *_ref(x, causal), BF16_TOL, f"bf16 {shape}")


def test_bf16_output_only_16_byte_aligned(cuda_lib):
    # O at a 16-byte (not 32-byte) aligned address takes the 16-byte store path.
    x = prefill_inputs(1, 4, 2, 200, 200, 128, dtype="bf16", seed=4)
    buf = torch.zeros(x["q"].numel() + 8, dtype=torch.bfloat16, device="cuda")
    o = buf[8:].view(x["q"].shape)
    assert o.data_ptr() % 32 == 16
    _, lse = attn_fwd(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), causal=True, o=o)
    torch.cuda.synchronize()
    compare(o, lse, *_ref(x, True), BF16_TOL, "O at 16 mod 32")
    assert torch.all(buf[:8] == 0)


def test_bf16_empty_keys(cuda_lib):
    x = prefill_inputs(1, 2, 1, 9, 0, 64, dtype="bf16", seed=1)
    o, lse = _run(x, False)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_bf16_large_scores_and_scale(cuda_lib):
    # Scores of several hundred (scale 1): the online max must keep exp in range.
    x = prefill_inputs(1, 4, 2, 256, 256, 128, dtype="bf16", seed=9)
    x["q"] = (x["q"].float() * 4).to(torch.bfloat16)
    o, lse = _run(x, True, scale=1.0)
    compare(o, lse, *_ref(x, True, scale=1.0), BF16_TOL, "large scores")


def test_bf16_decode_row_equals_last_causal_row(cuda_lib):
    from exact_attention_137_b200 import attn_decode

    x = prefill_inputs(2, 8, 2, 200, 200, 128, dtype="bf16", seed=5)
    o, lse = _run(x, True)
    q = x["q"][:, :, -1].contiguous().cuda()
    seqlens = torch.full((2,), 200, dtype=torch.int32, device="cuda")
    od, ld = attn_decode(q, x["k"].cuda(), x["v"].cuda(), seqlens, max_seqlen=200)
    torch.cuda.synchronize()
    assert (od.float() - o[:, :, -1].float()).abs().max().item() <= 2e-2
    assert (ld - lse[:, :, -1]).abs().max().item() <= 1e-3


def _sample_rows(S, n, seed, must=()):
    rows = set(range(min(8, S))) | set(range(max(0, S - 8), S)) | {int(r) for r in must if r < S}
    rng = np.random.Generator(np.random.PCG64(seed))
    while len(rows) < min(n, S):
        rows.add(int(rng.integers(0, S)))
    return np.array(sorted(rows))


@pytest.mark.parametrize("hkv", [32, 8, 1])
def test_full_size_head_sharing_sweep_sampled(cuda_lib, hkv):
    # B=2, Hq=32, Hkv in {32, 8, 1}, Sq=Sk=2048, D=128, bf16, causal (the bench's workload).
    x = prefill_inputs(2, 32, hkv, 2048, 2048, 128, dtype="bf16", seed=0)
    o, lse = _run(x, True)
    rows = _sample_rows(2048, 192, seed=hkv)
    o_ref, l_ref = _ref(x, True, rows=rows)
    compare(o[:, :, rows], lse[:, :, rows], o_ref, l_ref, BF16_TOL, f"S=2048 Hkv={hkv}")


def test_full_size_long_context_spiked_sampled(cuda_lib):
    # B=1, Hq=64, Hkv=8, S=16384, D=128, bf16, causal, 0.1% of key rows x8.
    x = prefill_inputs(1, 64, 8, 16384, 16384, 128, dtype="bf16", seed=0, spike_frac=0.001)
    o, lse = _run(x, True)
    spikes = x["spike_rows"].reshape(-1)
    rows = _sample_rows(16384, 192, seed=4, must=spikes[:: max(1, spikes.size // 64)])
    o_ref, l_ref = _ref(x, True, rows=rows)
    compare(o[:, :, rows], lse[:, :, rows], o_ref, l_ref, BF16_TOL, "S=16384 spiked")


def test_no_device_error_raised(cuda_lib):
    assert device_status(clear=True) == 0


def test_polynomial_exp2_against_exp2(cuda_lib):
    from exact_attention_137_b200 import _lib

    x = torch.cat([torch.linspace(-125.0, 8.0, 1 << 20), torch.tensor([0.0, -0.5, 0.5, 1.0, -1.0, 7.99])])
    y = _lib.selftest_exp2_poly(x.cuda()).cpu().double().numpy()
    ref = np.exp2(x.double().numpy())
    rel = np.abs(y - ref) / ref
    assert rel.max() <= 8e-5, rel.max()
    # below the clamp: tiny, positive, finite
    z = _lib.selftest_exp2_poly(torch.tensor([-200.0, -1e30, -127.5], device="cuda")).cpu()
    assert torch.all(z >= 0) and torch.all(z < 1e-37)


# ---------------------------------------------------------------- sliding window


WINDOW_SHAPES = [
    # B, Hq, Hkv, Sq, Sk, D, window
    (1, 4, 2, 520, 520, 128, 200),    # head pairs, window not a multiple of the tile
    (1, 3, 3, 700, 700, 128, 128),    # MHA: the two query tiles of an item start at different KV tiles
    (1, 6, 2, 640, 640, 128, 300),    # g = 3: head pair plus leftover head
    (2, 8, 1, 300, 450, 64, 50),      # Sq < Sk, D = 64
    (1, 4, 2, 384, 256, 128, 64),     # Sq > Sk: fully masked leading rows
    (1, 2, 1, 260, 260, 128, 1),      # each row sees only its own key
]


@pytest.mark.parametrize("shape", WINDOW_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_bf16_window_all_elements(cuda_lib, shape):
    B, Hq, Hkv, Sq, Sk, D, W = shape
    x = prefill_inputs(B, Hq, Hkv, Sq, Sk, D, dtype="bf16", seed=sum(shape))
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = attn_fwd(q, k, v, causal=True, window=W)
    torch.cuda.synchronize()
    ref = attention_rows_ref(to_f64(x["q"]), to_f64(x["k"]), to_f64(x["v"]), causal=True, window=W)
    compare(o, lse, *ref, BF16_TOL, f"window {shape}")


def test_window_covering_all_keys_is_causal_bit_for_bit(cuda_lib):
    x = prefill_inputs(1, 4, 2, 600, 600, 128, dtype="bf16", seed=11)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = attn_fwd(q, k, v, causal=True)
    o2, l2 = attn_fwd(q, k, v, causal=True, window=600)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fp32_window(cuda_lib):
    x = prefill_inputs(1, 4, 2, 200, 200, 64, dtype="f32", seed=12)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = attn_fwd(q, k, v, causal=True, window=33)
    torch.cuda.synchronize()
    compare(o, lse, *attention_rows_ref(to_f64(x["q"]), to_f64(x["k"]), to_f64(x["v"]), causal=True, window=33),
            F32_TOL, "fp32 window")


@pytest.mark.parametrize("hkv", [8, 32])
def test_window_4k_sampled(cuda_lib, hkv):
    x = prefill_inputs(1, 32, hkv, 4096, 4096, 128, dtype="bf16", seed=13)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = attn_fwd(q, k, v, causal=True, window=1000)
    torch.cuda.synchronize()
    rows = _sample_rows(4096, 160, seed=hkv, must=(999, 1000, 1001, 2047, 2048))
    ref = attention_rows_ref(to_f64(x["q"]), to_f64(x["k"]), to_f64(x["v"]), causal=True, rows=rows, window=1000)
    compare(o[:, :, rows], lse[:, :, rows], *ref, BF16_TOL, f"window 4k Hkv={hkv}")


def test_window_rejects_negative_and_non_causal(cuda_lib):
    x = prefill_inputs(1, 2, 1, 16, 16, 64, dtype="bf16", seed=14)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    with pytest.raises(_lib.AttnError):
        attn_fwd(q, k, v, causal=True, window=-1)
    with pytest.raises(ValueError):
        attn_fwd(q, k, v, causal=False, window=4)
