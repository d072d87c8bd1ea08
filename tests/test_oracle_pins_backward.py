"""Pins of the oracle's attention backward pass.

The gradients are checked against central finite differences of the forward
oracle (itself pinned by brute force), which shares nothing with the
backward formulas; the identity D = rowsum(dO * O) and the GQA summation are
checked as well, and planted mistakes must fail.
"""

import numpy as np
import pytest

import oracle
from oracle import backward as ob

MASKS = [(oracle.MASK_FULL, 0), (oracle.MASK_CAUSAL, 0), (oracle.MASK_SLIDING_WINDOW, 2)]


def _loss(q, k, v, d_o, mask_kind, window, scale):
    o, _ = oracle.prefill_ref(q, k, v, mask_kind, window, scale)
    return float((o * d_o).sum())  # L = <dO, O>, so dL/dO = dO


def _numeric_grad(f, x, eps=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + eps
        fp = f()
        x[i] = old - eps
        fm = f()
        x[i] = old
        g[i] = (fp - fm) / (2 * eps)
    return g


@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2), (2, 1)])
@pytest.mark.parametrize("mask_kind,window", MASKS)
def test_gradients_match_finite_differences(hq, hkv, mask_kind, window):
    rng = np.random.default_rng(hq * 10 + hkv + 3 * mask_kind)
    B, N, d, scale = 1, 5, 3, 0.7
    q, k, v = rng.standard_normal((B, hq, N, d)), rng.standard_normal((B, hkv, N, d)), rng.standard_normal((B, hkv, N, d))
    d_o = rng.standard_normal((B, hq, N, d))
    d_q, d_k, d_v = oracle.prefill_backward_ref(q, k, v, d_o, mask_kind, window, scale)
    f = lambda: _loss(q, k, v, d_o, mask_kind, window, scale)  # noqa: E731
    np.testing.assert_allclose(d_q, _numeric_grad(f, q), rtol=0, atol=1e-7)
    np.testing.assert_allclose(d_k, _numeric_grad(f, k), rtol=0, atol=1e-7)
    np.testing.assert_allclose(d_v, _numeric_grad(f, v), rtol=0, atol=1e-7)


def test_d_is_rowsum_of_do_times_o():
    rng = np.random.default_rng(1)
    R, T, d = 6, 9, 4
    q, k, v, d_o = (rng.standard_normal(s) for s in ((R, d), (T, d), (T, d), (R, d)))
    allowed = oracle.allowed_mask(R, T, oracle.MASK_CAUSAL)
    o, _ = oracle.sdpa_rows(q, k, v, allowed, 0.5)
    _, _, _, dd = ob.sdpa_backward_rows(q, k, v, allowed, 0.5, d_o)
    np.testing.assert_allclose(dd, (d_o * o).sum(axis=1), rtol=0, atol=1e-13)


def test_gqa_gradients_sum_over_the_group():
    """dK, dV of a K/V head equal the sums over its query heads computed as
    independent MHA heads on repeated K/V."""
    rng = np.random.default_rng(2)
    B, hq, hkv, N, d = 1, 4, 2, 6, 3
    q, d_o = rng.standard_normal((B, hq, N, d)), rng.standard_normal((B, hq, N, d))
    k, v = rng.standard_normal((B, hkv, N, d)), rng.standard_normal((B, hkv, N, d))
    d_q, d_k, d_v = oracle.prefill_backward_ref(q, k, v, d_o, oracle.MASK_CAUSAL, 0, 0.4)
    k_rep, v_rep = np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1)
    d_q2, d_k2, d_v2 = oracle.prefill_backward_ref(q, k_rep, v_rep, d_o, oracle.MASK_CAUSAL, 0, 0.4)
    np.testing.assert_allclose(d_q, d_q2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(d_k, d_k2.reshape(B, hkv, 2, N, d).sum(axis=2), rtol=0, atol=1e-13)
    np.testing.assert_allclose(d_v, d_v2.reshape(B, hkv, 2, N, d).sum(axis=2), rtol=0, atol=1e-13)


def _mutant(kind):
    def sdpa_backward_rows(q_rows, k, v, allowed, scale, d_o):
        s = np.where(allowed, (q_rows @ k.T) * scale, -np.inf)
        e = np.exp(s - s.max(axis=1, keepdims=True))
        p = e / e.sum(axis=1, keepdims=True)
        d_v = p.T @ d_o
        d_p = d_o @ v.T
        dd = (p * d_p).sum(axis=1)
        d_s = p * (d_p - (0.0 if kind == "no_jacobian_term" else dd[:, None]))
        d_q = (1.0 if kind == "no_scale" else scale) * (d_s @ k)
        d_k = scale * ((d_s if kind != "no_transpose" else d_s[::-1]).T @ q_rows)
        return d_q, d_k, d_v, dd
    return sdpa_backward_rows


@pytest.mark.parametrize("kind", ["no_jacobian_term", "no_scale", "no_transpose"])
def test_planted_mistakes_are_caught(kind, monkeypatch):
    rng = np.random.default_rng(4)
    q, k, v, d_o = (rng.standard_normal((1, 2, 5, 3)) for _ in range(4))
    f = lambda: _loss(q, k, v, d_o, oracle.MASK_CAUSAL, 0, 0.7)  # noqa: E731
    g = (_numeric_grad(f, q), _numeric_grad(f, k))
    monkeypatch.setattr(ob, "sdpa_backward_rows", _mutant(kind))
    d_q, d_k, _ = ob.prefill_backward_ref(q, k, v, d_o, oracle.MASK_CAUSAL, 0, 0.7)
    assert max(np.abs(d_q - g[0]).max(), np.abs(d_k - g[1]).max()) > 1e-4
