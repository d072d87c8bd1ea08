"""GPU parity of attn_prefill_backward (dQ, dK, dV) against the fp64 oracle,
through the C ABI. The forward inputs, O and LSE come from attn_prefill (the
kernel's own forward, itself checked against the oracle elsewhere); dO is a
seeded bf16 normal draw."""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_softmax_attention_causal_b200 import prefill, prefill_backward, workloads
from parity import assert_grad_parity

pytestmark = pytest.mark.gpu

MASK_IDS = {"full": oracle.MASK_FULL, "causal": oracle.MASK_CAUSAL, "window": oracle.MASK_SLIDING_WINDOW}


def _grad_output(shape, seed):
    g = torch.Generator("cpu").manual_seed(10_000 + seed)
    return torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def _run(B, Hq, Hkv, N, d, mask, window=0, seed=0):
    x = workloads.prefill_inputs(B, Hq, Hkv, N, d, seed)
    d_o = _grad_output((B, Hq, N, d), seed)
    q, k, v, g = (t.cuda() for t in (x.q, x.k, x.v, d_o))
    o, lse = prefill(q, k, v, mask=mask, window=window)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dk, dv = prefill_backward(q, k, v, o, lse, g, mask=mask, window=window, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return x, d_o, dq.cpu(), dk.cpu(), dv.cpu()


def _check(B, Hq, Hkv, N, d, mask, window=0, seed=0):
    x, d_o, dq, dk, dv = _run(B, Hq, Hkv, N, d, mask, window, seed)
    r_q, r_k, r_v = oracle.prefill_backward_ref(x.q, x.k, x.v, d_o, MASK_IDS[mask], window, 1 / math.sqrt(d))
    what = f"{B}x{Hq}/{Hkv}x{N}x{d} {mask} w={window}"
    assert_grad_parity(dq, r_q, what=f"dQ {what}")
    assert_grad_parity(dk, r_k, what=f"dK {what}")
    assert_grad_parity(dv, r_v, what=f"dV {what}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mask,window", [("causal", 0), ("full", 0), ("window", 1), ("window", 100),
                                         ("window", 257)])
def test_ragged_multi_tile(d, mask, window):
    # N = 300: three 128-row tiles, the last ragged
    _check(1, 4, 2, 300, d, mask, window, seed=1)


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 1), (6, 3)])
def test_head_maps(hq, hkv):
    _check(2, hq, hkv, 256, 128, "causal", seed=2)


@pytest.mark.parametrize("N", [1, 7, 129, 640])
def test_sizes(N):
    _check(1, 2, 1, N, 128, "causal", seed=3)
    _check(1, 2, 1, N, 64, "full", seed=3)


def test_deterministic():
    a = _run(1, 4, 1, 512, 128, "causal", seed=4)
    b = _run(1, 4, 1, 512, 128, "causal", seed=4)
    for u, w in zip(a[2:], b[2:]):
        assert torch.equal(u, w)


def test_full_size_one_kv_head_sampled():
    """llama3_8b_causal_gqa shapes (B=4, Hq=32, Hkv=8, N=4096, d=128): the
    gradients of the first sequence's first K/V head and its four query heads
    against the oracle."""
    cfg = workloads.PREFILL_WORKLOADS["llama3_8b_causal_gqa"]
    B, Hq, Hkv, N, d = cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["N"], cfg["d"]
    x, d_o, dq, dk, dv = _run(B, Hq, Hkv, N, d, "causal", seed=0)
    g = Hq // Hkv
    r_q, r_k, r_v = oracle.prefill_backward_ref(x.q[:1, :g], x.k[:1, :1], x.v[:1, :1], d_o[:1, :g],
                                                oracle.MASK_CAUSAL, 0, 1 / math.sqrt(d))
    assert_grad_parity(dq[:1, :g], r_q, what="dQ")
    assert_grad_parity(dk[:1, :1], r_k, what="dK")
    assert_grad_parity(dv[:1, :1], r_v, what="dV")
    assert all(torch.isfinite(t.float()).all() for t in (dq, dk, dv))
