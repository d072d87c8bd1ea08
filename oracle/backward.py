"""Plain fp64 definition of the attention backward pass (the gradients of
prefill attention).

TEST INFRASTRUCTURE ONLY (see the package docstring): slow, obviously correct,
CPU-only, never on the product path.

Sources (page title, section):

* "Inference attention" post (brunomaga.github.io), section "FlashAttention":
  during training the backward pass recomputes S and P (tile by tile in the
  kernel) instead of storing them. The pages state no formulas for the
  gradients; they are the derivative of the forward definition
  ("Module 5. Modern Attention Mechanisms", section 4: O = softmax(scale QK^T
  + M) V, masked entries -inf), written out by the chain rule:

      P = softmax(scale Q K^T + M)     (rows; masked entries are 0)
      dV = P^T dO
      dP = dO V^T
      dS = P * (dP - D),   D_i = sum_j P_ij dP_ij   (the softmax Jacobian)
      dQ = scale dS K,     dK = scale dS^T Q

  for an upstream gradient dO of the output. Grouped-query heads (section 6):
  query head h reads K/V head h // (Hq / Hkv), so dK and dV of a K/V head sum
  the contributions of its query heads.

The oracle computes P directly (full score rows, as the forward oracle does),
then the formulas above. `D` is also available as rowsum(dO * O), the form a
kernel uses; the pins check both.
"""

from __future__ import annotations

import numpy as np

from .attention import _as_f64, _check_heads, allowed_mask


def sdpa_backward_rows(q_rows, k, v, allowed, scale: float, d_o):
    """Gradients for one head: q_rows [R, d], k [T, d], v [T, d_v], allowed
    [R, T] bool, d_o [R, d_v]. Returns (dQ [R, d], dK [T, d], dV [T, d_v],
    D [R]) in float64. Every row must see at least one key."""
    q_rows, k, v, d_o = (_as_f64(x) for x in (q_rows, k, v, d_o))
    allowed = np.asarray(allowed, dtype=bool)
    if not allowed.any(axis=1).all():
        raise ValueError("fully masked rows")
    s = np.where(allowed, (q_rows @ k.T) * float(scale), -np.inf)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    p = e / e.sum(axis=1, keepdims=True)
    d_v = p.T @ d_o
    d_p = d_o @ v.T
    dd = (p * d_p).sum(axis=1)
    d_s = p * (d_p - dd[:, None])
    d_q = float(scale) * (d_s @ k)
    d_k = float(scale) * (d_s.T @ q_rows)
    return d_q, d_k, d_v, dd


def prefill_backward_ref(q, k, v, d_o, mask_kind: int, window: int, scale: float):
    """Gradients of prefill attention for q [B, Hq, N, d], k, v [B, Hkv, N, d]
    and the output gradient d_o [B, Hq, N, d]. Returns (dQ [B, Hq, N, d],
    dK [B, Hkv, N, d], dV [B, Hkv, N, d]) in float64."""
    q, k, v, d_o = (_as_f64(x) for x in (q, k, v, d_o))
    b_, hq, n, d = q.shape
    hkv = k.shape[1]
    g = _check_heads(hq, hkv)
    allowed = allowed_mask(n, k.shape[2], mask_kind, window)
    d_q = np.zeros_like(q)
    d_k = np.zeros_like(k)
    d_v = np.zeros_like(v)
    for bi in range(b_):
        for h in range(hq):
            kvh = h // g
            dq_h, dk_h, dv_h, _ = sdpa_backward_rows(q[bi, h], k[bi, kvh], v[bi, kvh], allowed, scale, d_o[bi, h])
            d_q[bi, h] = dq_h
            d_k[bi, kvh] += dk_h
            d_v[bi, kvh] += dv_h
    return d_q, d_k, d_v
