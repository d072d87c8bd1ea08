"""Pins of the oracle's row-subset path, prefill_rows_ref and allowed_mask(rows=).

prefill_rows_ref is the checker for every full-size prefill parity test (it
computes chosen rows of one (batch, head) directly), so it is pinned here on
its own: against a pure-Python brute force that takes positions from the pages'
rule, and against the rows of the full prefill_ref. The cases cover every mask
kind, the prefix alignment (n_q < n_k), every head map (MHA, GQA, MQA) and row
subsets that are random, unsorted, repeated or on the boundaries. The planted
mistakes at the end (a row offset off by one, the tile-order head map, the row
subset ignored) must make the pin fail.

Passages: "Module 5. Modern Attention Mechanisms", section 4 (query row i of an
n_q-row block after a prefix of n_k - n_q positions sits at position
n_k - n_q + i; causal p_k <= p_q; a window of W positions including the
current one, 0 <= p_q - p_k < W) and section 6 (query head h reads K/V head
floor(h / g), g = Hq / Hkv).
"""

import math

import numpy as np
import pytest

import oracle
from oracle import attention as oa

MASKS = [(oracle.MASK_FULL, 0), (oracle.MASK_CAUSAL, 0), (oracle.MASK_SLIDING_WINDOW, 1),
         (oracle.MASK_SLIDING_WINDOW, 3), (oracle.MASK_SLIDING_WINDOW, 100)]
HEAD_MAPS = [(4, 2), (4, 4), (4, 1)]


def _visible_pos(p_q, p_k, mask_kind, window):
    if mask_kind == oracle.MASK_FULL:
        return True
    if mask_kind == oracle.MASK_CAUSAL:
        return p_k <= p_q
    return 0 <= p_q - p_k < window


def _brute_rows(q, k, v, b, h, rows, mask_kind, window, scale):
    """Scalar loops over positions: row i of q sits at n_k - n_q + i."""
    hq, n_q, d = q.shape[1], q.shape[2], q.shape[3]
    hkv, n_k = k.shape[1], k.shape[2]
    kv = h // (hq // hkv)
    out = np.zeros((len(rows), v.shape[-1]))
    lse = np.zeros(len(rows))
    for r, i in enumerate(rows):
        p_q = n_k - n_q + int(i)
        sc = []
        for j in range(n_k):
            if _visible_pos(p_q, j, mask_kind, window):
                s = 0.0
                for t in range(d):
                    s += float(q[b, h, i, t]) * float(k[b, kv, j, t])
                sc.append((j, s * scale))
        mx = max(s for _, s in sc)
        w = [(j, math.exp(s - mx)) for j, s in sc]
        den = sum(x for _, x in w)
        for t in range(v.shape[-1]):
            out[r, t] = sum(x * float(v[b, kv, j, t]) for j, x in w) / den
        lse[r] = mx + math.log(den)
    return out, lse


def _row_sets(n_q, rng):
    """Random, unsorted, repeated and boundary subsets of range(n_q)."""
    return [
        [0],
        [n_q - 1],
        [n_q - 1, 0, n_q // 2],                      # unsorted, both ends
        rng.permutation(n_q)[: max(1, n_q // 2)].tolist(),  # random, unsorted
        [2, 2, 1, 2] if n_q > 2 else [0, 0],         # repeated rows
        list(range(n_q)),                            # every row
    ]


def _inputs(rng, B, hq, hkv, n_q, n_k, d):
    return (rng.standard_normal((B, hq, n_q, d)), rng.standard_normal((B, hkv, n_k, d)),
            rng.standard_normal((B, hkv, n_k, d)))


def _worst_rows_error(q, k, v, mask_kind, window, scale, rng):
    """Largest |prefill_rows_ref - brute force| over every (b, h) and row set."""
    B, hq = q.shape[0], q.shape[1]
    worst = 0.0
    for b in range(B):
        for h in range(hq):
            for rows in _row_sets(q.shape[2], rng):
                o, l = oa.prefill_rows_ref(q, k, v, b, h, rows, mask_kind, window, scale)
                o_bf, l_bf = _brute_rows(q, k, v, b, h, rows, mask_kind, window, scale)
                worst = max(worst, float(np.abs(o - o_bf).max()), float(np.abs(l - l_bf).max()))
    return worst


@pytest.mark.parametrize("hq,hkv", HEAD_MAPS)
@pytest.mark.parametrize("mask_kind,window", MASKS)
def test_rows_equal_brute_force_and_full_prefill(hq, hkv, mask_kind, window):
    rng = np.random.default_rng(200 + 10 * hq + hkv + window)
    B, N, d = 2, 9, 5
    q, k, v = _inputs(rng, B, hq, hkv, N, N, d)
    scale = 1 / math.sqrt(d)
    assert _worst_rows_error(q, k, v, mask_kind, window, scale, rng) <= 1e-12
    o_full, l_full = oracle.prefill_ref(q, k, v, mask_kind, window, scale)
    for b in range(B):
        for h in range(hq):
            for rows in _row_sets(N, rng):
                o, l = oracle.prefill_rows_ref(q, k, v, b, h, rows, mask_kind, window, scale)
                np.testing.assert_allclose(o, o_full[b, h, rows], rtol=0, atol=1e-13)
                np.testing.assert_allclose(l, l_full[b, h, rows], rtol=0, atol=1e-13)


@pytest.mark.parametrize("hq,hkv", HEAD_MAPS)
@pytest.mark.parametrize("mask_kind,window", MASKS)
def test_rows_prefix_alignment(hq, hkv, mask_kind, window):
    """n_q < n_k: the query rows are the newest n_q positions (bottom-right)."""
    rng = np.random.default_rng(300 + 10 * hq + hkv + window)
    B, n_q, n_k, d = 1, 5, 12, 4
    q, k, v = _inputs(rng, B, hq, hkv, n_q, n_k, d)
    assert _worst_rows_error(q, k, v, mask_kind, window, 0.45, rng) <= 1e-12


def test_rows_mask_matches_full_mask_rows():
    """allowed_mask(rows=R) is the full mask's rows R, in R's order, repeats kept."""
    rng = np.random.default_rng(4)
    for n_q, n_k in ((7, 7), (4, 11)):
        for kind, w in MASKS:
            full = oracle.allowed_mask(n_q, n_k, kind, w)
            for rows in _row_sets(n_q, rng):
                assert np.array_equal(oracle.allowed_mask(n_q, n_k, kind, w, rows=rows), full[rows])


def test_rows_mask_counts_closed_form():
    """Row i of an n-row causal block sees i + 1 keys, a W window min(i + 1, W);
    after a prefix P the counts shift to P + i + 1 and min(P + i + 1, W)."""
    n_q, n_k, w = 6, 10, 4
    rows = [5, 0, 3]
    p = n_k - n_q
    causal = oracle.allowed_mask(n_q, n_k, oracle.MASK_CAUSAL, rows=rows).sum(axis=1)
    window = oracle.allowed_mask(n_q, n_k, oracle.MASK_SLIDING_WINDOW, w, rows=rows).sum(axis=1)
    assert causal.tolist() == [p + i + 1 for i in rows]
    assert window.tolist() == [min(p + i + 1, w) for i in rows]


def test_rows_accepts_torch_cpu_tensors():
    """The GPU tests pass bf16 CPU tensors; the rows must equal the numpy path
    on the same (exactly widened) values."""
    import torch

    g = torch.Generator("cpu").manual_seed(3)
    q = torch.randn(1, 4, 20, 8, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 2, 20, 8, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 2, 20, 8, generator=g).to(torch.bfloat16)
    rows = [19, 3, 7]
    o_t, l_t = oracle.prefill_rows_ref(q, k, v, 0, 3, rows, oracle.MASK_CAUSAL, 0, 0.3)
    qn, kn, vn = (t.to(torch.float64).numpy() for t in (q, k, v))
    o_n, l_n = _brute_rows(qn, kn, vn, 0, 3, rows, oracle.MASK_CAUSAL, 0, 0.3)
    assert np.abs(o_t - o_n).max() <= 1e-12 and np.abs(l_t - l_n).max() <= 1e-12


# --------------------------------------------------------------------------
# planted mistakes in the row path: each must fail the brute-force pin
# --------------------------------------------------------------------------
def _plant(monkeypatch, kind):
    real_mask = oa.allowed_mask

    if kind == "row_offset":  # position n_k - n_q + i + 1 instead of n_k - n_q + i
        def mask(n_q, n_k, mask_kind, window=0, rows=None, n_sink=0):
            rows = np.arange(n_q) if rows is None else np.asarray(rows)
            return real_mask(n_q + 1, n_k + 1, mask_kind, window, rows=rows + 1, n_sink=n_sink)[:, :n_k]
        monkeypatch.setattr(oa, "allowed_mask", mask)
    elif kind == "rows_ignored":  # the first len(rows) rows' mask, whatever rows holds
        def mask(n_q, n_k, mask_kind, window=0, rows=None, n_sink=0):
            rows = np.arange(n_q) if rows is None else np.asarray(rows)
            return real_mask(n_q, n_k, mask_kind, window, rows=np.arange(len(rows)) % n_q, n_sink=n_sink)
        monkeypatch.setattr(oa, "allowed_mask", mask)
    elif kind == "tile_heads":  # h % Hkv instead of h // g
        monkeypatch.setattr(oa, "kv_head_of", lambda h, hq, hkv: h % hkv)
    else:
        raise ValueError(kind)


@pytest.mark.parametrize("kind", ["row_offset", "rows_ignored", "tile_heads"])
def test_planted_row_mistakes_are_caught(kind, monkeypatch):
    rng = np.random.default_rng(11)
    q, k, v = _inputs(rng, 1, 4, 2, 6, 6, 4)
    cases = [(oracle.MASK_CAUSAL, 0, q), (oracle.MASK_SLIDING_WINDOW, 3, q), (oracle.MASK_CAUSAL, 0, q[:, :, :3])]
    # the brute force is computed before the mistake is planted
    refs = []
    for kind_m, w, qq in cases:
        rows = [qq.shape[2] - 1, 0, 1]
        refs.append(_brute_rows(qq, k, v, 0, 1, rows, kind_m, w, 0.5))
    _plant(monkeypatch, kind)
    worst = 0.0
    for (kind_m, w, qq), (o_bf, l_bf) in zip(cases, refs):
        rows = [qq.shape[2] - 1, 0, 1]
        o, l = oa.prefill_rows_ref(qq, k, v, 0, 1, rows, kind_m, w, 0.5)
        worst = max(worst, float(np.abs(o - o_bf).max()), float(np.abs(l - l_bf).max()))
    assert worst > 1e-3, f"planted mistake {kind} not caught (worst {worst:.2e})"
