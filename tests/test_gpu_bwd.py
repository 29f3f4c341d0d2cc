"""Backward parity: attn_bwd through the C ABI against the fp64 oracle's gradients.

The GPU backward takes the GPU forward's O and LSE (as a training step would); the
oracle recomputes everything in fp64 from the same bf16 inputs.  Covers causal and
non-causal, GQA / MHA / MQA, ragged tails, Sq < Sk, Sq > Sk (rows with no key), a
sliding window, D = 64 and 128, and a 1024-token case.
"""

import pytest
import torch

from oracle import attention_bwd_ref
from exact_attention_137_b200 import _lib, attn_bwd, attn_fwd, device_status
from exact_attention_137_b200.workloads import prefill_inputs, to_f64

from parity import compare_grad

pytestmark = pytest.mark.gpu

SHAPES = [
    # B, Hq, Hkv, Sq, Sk, D, causal, window
    (1, 4, 2, 130, 130, 64, True, 0),
    (1, 2, 2, 200, 170, 128, False, 0),
    (2, 8, 1, 257, 257, 128, True, 0),     # MQA, ragged
    (1, 3, 3, 100, 300, 64, True, 0),      # MHA, Sq < Sk
    (1, 4, 2, 300, 100, 128, True, 0),     # Sq > Sk: rows with no visible key
    (1, 4, 2, 400, 400, 128, True, 150),   # sliding window
    (1, 8, 2, 1024, 1024, 128, True, 0),
]


def _grad_case(shape, seed):
    B, Hq, Hkv, Sq, Sk, D, causal, window = shape
    x = prefill_inputs(B, Hq, Hkv, Sq, Sk, D, dtype="bf16", seed=seed)
    gen = torch.Generator().manual_seed(seed + 1)
    dout = torch.randn(B, Hq, Sq, D, generator=gen).to(torch.bfloat16)
    q, k, v, do = (t.cuda() for t in (x["q"], x["k"], x["v"], dout))
    o, lse = attn_fwd(q, k, v, causal=causal, window=window if window > 0 else None)
    dq, dk, dv = attn_bwd(q, k, v, o, lse, do, causal=causal, window=window)
    torch.cuda.synchronize()
    ref = attention_bwd_ref(to_f64(x["q"]), to_f64(x["k"]), to_f64(x["v"]), to_f64(dout), causal=causal,
                            window=window)
    return (dq, dk, dv), ref


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_bwd_matches_oracle(cuda_lib, shape):
    got, ref = _grad_case(shape, seed=sum(shape))
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        compare_grad(g, r, what=f"{name} {shape}")
    assert device_status(clear=True) == 0


def test_bwd_rejects_bad_arguments(cuda_lib):
    x = prefill_inputs(1, 2, 1, 16, 16, 64, dtype="bf16", seed=3)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = attn_fwd(q, k, v, causal=True)
    with pytest.raises(_lib.AttnError):
        attn_bwd(q, k, v, o, lse, o, causal=False, window=4)  # a window needs causal
    with pytest.raises(_lib.AttnError):
        attn_bwd(q, k, v, o, lse, o, causal=True, scale=0.0)
