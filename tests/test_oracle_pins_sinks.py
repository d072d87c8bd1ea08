"""Pins of the oracle's sliding-window decode with sinks.

"Module 5. Modern Attention Mechanisms", section 10 (two kinds of attention
sink) and section 12 (the mask builder and SDPA with a sink column):

* StreamingLLM sinks: with a finite window the first n_sink real positions
  stay visible.
* gpt-oss learned sinks: one logit s_h per query head, appended as a score
  column, normalised with the row and dropped before the product with V.

Each test checks the oracle against something other than itself: the
percentages the page prints, a hand-enumerated mask, the page's own
equivalences (an extra key with a constant coordinate and a zero value; the
shift check; eviction of the middle of the cache), closed forms and limits.
The last group plants mistakes and checks that these pins catch them.
"""

import math
import os

import numpy as np
import pytest

import oracle
from oracle import attention as oa
from exact_softmax_attention_causal_b200 import accounting

from test_oracle_pins import _paged_from_contiguous


def _golden_rows(golden_dir, name):
    return [line.split() for line in open(os.path.join(golden_dir, name))
            if line.strip() and not line.startswith("#")]


# --------------------------------------------------------------------------
# learned sink logit
# --------------------------------------------------------------------------
def _sink_mass_case(s, sdpa=None):
    """128 token scores all zero (q = 0) and one sink logit s. Returns the sink
    mass recovered from the LSE, the output and the mean of V."""
    sdpa = sdpa or oa.sdpa_rows
    rng = np.random.default_rng(21)
    k, v = rng.standard_normal((128, 16)), rng.standard_normal((128, 16))
    o, lse = sdpa(np.zeros((1, 16)), k, v, np.ones((1, 128), dtype=bool), 0.25, sink=s)
    return math.exp(s - lse[0]), o[0], v.mean(axis=0)


def test_sink_mass_matches_printed_percentages(golden_dir):
    rows = _golden_rows(golden_dir, "sink_mass_128_zero_scores.txt")
    assert len(rows) == 3
    for s, pct in rows:
        p, o, vbar = _sink_mass_case(float(s))
        assert round(100 * p, 2) == float(pct)
        # the tokens share the remaining mass equally: O = (1 - p) * mean(V)
        np.testing.assert_allclose(o, (1 - p) * vbar, rtol=0, atol=1e-13)


def _extend_with_sink_key(q, k, v, allowed, scale, s):
    """The page's equivalent form: one more coordinate, 1 in every query; one
    more key whose extra coordinate is s / scale (its score is exactly s) and
    whose value is zero, visible to every row."""
    r, d = q.shape
    q2 = np.concatenate([q, np.ones((r, 1))], axis=1)
    k2 = np.concatenate([np.concatenate([k, np.zeros((k.shape[0], 1))], axis=1),
                         np.concatenate([np.zeros((1, d)), [[s / scale]]], axis=1)])
    v2 = np.concatenate([v, np.zeros((1, v.shape[1]))])
    a2 = np.concatenate([allowed, np.ones((r, 1), dtype=bool)], axis=1)
    return q2, k2, v2, a2


@pytest.mark.parametrize("s", [-3.0, 0.0, 1.7, 9.0])
def test_sink_equals_extra_zero_value_key(s):
    rng = np.random.default_rng(23)
    R, T, d, scale = 7, 19, 8, 0.35
    q, k, v = rng.standard_normal((R, d)) * 2, rng.standard_normal((T, d)), rng.standard_normal((T, d))
    allowed = rng.random((R, T)) < 0.6
    allowed[3] = False  # one row with no visible token: all mass on the sink
    o, lse = oa.sdpa_rows(q, k, v, allowed, scale, sink=s)
    q2, k2, v2, a2 = _extend_with_sink_key(q, k, v, allowed, scale, s)
    o2, lse2 = oa.sdpa_rows(q2, k2, v2, a2, scale)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-13)
    assert np.array_equal(o[3], np.zeros(d)) and lse[3] == s


def test_shifting_tokens_alone_changes_output_shifting_all_does_not():
    """Section 10's check: adding c to the token logits but not to the sink
    changes the output; adding c to every logit, the sink too, does not."""
    rng = np.random.default_rng(29)
    R, T, d, scale, s, c = 4, 11, 6, 0.5, 1.3, 2.5
    q, k, v = rng.standard_normal((R, d)), rng.standard_normal((T, d)), rng.standard_normal((T, d))
    allowed = np.ones((R, T), dtype=bool)
    # shift every token score by c through a constant coordinate
    q2 = np.concatenate([q, np.ones((R, 1))], axis=1)
    k2 = np.concatenate([k, np.full((T, 1), c / scale)], axis=1)
    o, lse = oa.sdpa_rows(q, k, v, allowed, scale, sink=s)
    o_tok, _ = oa.sdpa_rows(q2, k2, v, allowed, scale, sink=s)
    o_all, lse_all = oa.sdpa_rows(q2, k2, v, allowed, scale, sink=s + c)
    assert np.max(np.abs(o_tok - o)) > 1e-2
    np.testing.assert_allclose(o_all, o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse_all, lse + c, rtol=0, atol=1e-13)


def test_sink_limits():
    rng = np.random.default_rng(31)
    q, k, v = rng.standard_normal((3, 8)), rng.standard_normal((9, 8)), rng.standard_normal((9, 8))
    a = np.ones((3, 9), dtype=bool)
    o0, l0 = oa.sdpa_rows(q, k, v, a, 0.4)
    o_lo, l_lo = oa.sdpa_rows(q, k, v, a, 0.4, sink=-800.0)  # exp(-800) underflows to 0
    assert np.array_equal(o_lo, o0) and np.array_equal(l_lo, l0)
    o_hi, l_hi = oa.sdpa_rows(q, k, v, a, 0.4, sink=800.0)    # every row's mass on the sink
    assert np.abs(o_hi).max() == 0.0 and np.array_equal(l_hi, np.full(3, 800.0))
    with pytest.raises(ValueError):
        oa.sdpa_rows(q, k, v, a, 0.4, sink=np.inf)


# --------------------------------------------------------------------------
# StreamingLLM sink positions in the mask
# --------------------------------------------------------------------------
def test_window_sink_mask_matches_hand_enumeration(golden_dir):
    rows = [[int(x) for x in r] for r in _golden_rows(golden_dir, "window_sink_mask_n8_w3_s2.txt")]
    m = oracle.allowed_mask(8, 8, oracle.MASK_SLIDING_WINDOW, 3, n_sink=2)
    assert np.array_equal(m.astype(int), np.array(rows))


def _visible_pair(p_q, p_k, w, n_sink):
    if p_k > p_q:
        return False
    return p_q - p_k < w or p_k < n_sink


@pytest.mark.parametrize("n_k,n_q,w,n_sink", [(9, 9, 1, 1), (9, 9, 2, 9), (20, 20, 5, 3), (20, 6, 4, 2),
                                             (33, 1, 7, 4), (33, 1, 40, 4), (16, 3, 16, 0)])
def test_window_sink_mask_pairwise(n_k, n_q, w, n_sink):
    m = oracle.allowed_mask(n_q, n_k, oracle.MASK_SLIDING_WINDOW, w, n_sink=n_sink)
    for i in range(n_q):
        for j in range(n_k):
            assert m[i, j] == _visible_pair(n_k - n_q + i, j, w, n_sink)


@pytest.mark.parametrize("n,w,n_sink", [(1, 1, 0), (50, 1, 1), (50, 7, 3), (50, 7, 9), (50, 60, 5), (50, 50, 50)])
def test_window_sink_row_counts_closed_form(n, w, n_sink):
    """Row i sees min(i + 1, W) window keys plus the sink keys below the
    window's first position: max(0, min(n_sink, i - W + 1))."""
    m = oracle.allowed_mask(n, n, oracle.MASK_SLIDING_WINDOW, w, n_sink=n_sink)
    for i in range(n):
        assert int(m[i].sum()) == min(i + 1, w) + max(0, min(n_sink, i - w + 1))
    assert [accounting.decode_visible_tokens(i + 1, w, n_sink) for i in range(n)] == m.sum(axis=1).tolist()


def test_n_sink_only_with_a_window():
    with pytest.raises(ValueError):
        oracle.allowed_mask(4, 4, oracle.MASK_CAUSAL, 0, n_sink=1)
    with pytest.raises(ValueError):
        oracle.allowed_mask(4, 4, oracle.MASK_SLIDING_WINDOW, 2, n_sink=5)
    assert np.array_equal(oracle.allowed_mask(6, 6, oracle.MASK_SLIDING_WINDOW, 3, n_sink=0),
                          oracle.allowed_mask(6, 6, oracle.MASK_SLIDING_WINDOW, 3))


# --------------------------------------------------------------------------
# windowed decode == full decode over the evicted (rolling) cache
# --------------------------------------------------------------------------
@pytest.mark.parametrize("n,w,n_sink,with_sinks", [(40, 8, 0, False), (40, 8, 4, False), (40, 8, 4, True),
                                                    (40, 38, 4, True), (40, 64, 2, True), (1, 3, 1, True),
                                                    (25, 1, 3, False)])
def test_windowed_decode_equals_decode_over_kept_tokens(n, w, n_sink, with_sinks):
    """Section 10: StreamingLLM keeps the first tokens alongside the recent
    window. Decoding with the window mask over the whole cache must equal an
    unmasked decode over a cache that holds only the kept tokens (the first
    n_sink, then the last W, each once, in position order)."""
    rng = np.random.default_rng(n * 100 + w)
    Hq, Hkv, d, bs, scale = 4, 2, 8, 4, 0.3
    k_seq, v_seq = rng.standard_normal((n, Hkv, d)), rng.standard_normal((n, Hkv, d))
    q = rng.standard_normal((1, Hq, d))
    sinks = rng.uniform(-1, 4, Hq) if with_sinks else None
    kept = sorted(set(range(min(n_sink, n))) | set(range(max(0, n - w), n)))
    kc, vc, table, lens = _paged_from_contiguous([k_seq], [v_seq], bs, 1)
    o_w, l_w = oracle.decode_paged_ref(q, kc, vc, table, lens, scale, window=w, n_sink=n_sink, sinks=sinks)
    kc2, vc2, table2, lens2 = _paged_from_contiguous([k_seq[kept]], [v_seq[kept]], bs, 2)
    o_k, l_k = oracle.decode_paged_ref(q, kc2, vc2, table2, lens2, scale, sinks=sinks)
    np.testing.assert_allclose(o_w, o_k, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l_w, l_k, rtol=0, atol=1e-13)


def test_windowed_decode_is_last_row_of_windowed_prefill():
    rng = np.random.default_rng(37)
    Hq, Hkv, N, d, w = 4, 2, 13, 8, 5
    q, k, v = (rng.standard_normal((1, h, N, d)) for h in (Hq, Hkv, Hkv))
    o_p, l_p = oracle.prefill_ref(q, k, v, oracle.MASK_SLIDING_WINDOW, w, 0.3)
    kc, vc, table, lens = _paged_from_contiguous([k[0].transpose(1, 0, 2)], [v[0].transpose(1, 0, 2)], 4, 3)
    o_d, l_d = oracle.decode_paged_ref(q[:, :, N - 1], kc, vc, table, lens, 0.3, window=w)
    np.testing.assert_allclose(o_d[0], o_p[0, :, N - 1], rtol=0, atol=1e-13)
    np.testing.assert_allclose(l_d[0], l_p[0, :, N - 1], rtol=0, atol=1e-13)


# --------------------------------------------------------------------------
# planted mistakes
# --------------------------------------------------------------------------
def _sdpa_sink_mutant(kind):
    def sdpa_rows(q_rows, k, v, allowed, scale, sink=None):
        q_rows, k, v = (np.asarray(x, dtype=np.float64) for x in (q_rows, k, v))
        sc = np.where(allowed, q_rows @ k.T * scale, -np.inf)
        mx = sc.max(axis=1)
        e = np.exp(sc - mx[:, None])
        den = e.sum(axis=1)
        if kind == "sink_ignored":
            pass
        elif kind == "sink_scaled":  # sink treated like a raw dot product and scaled
            den = den + np.exp(sink * scale - mx)
        elif kind == "sink_has_value":  # the sink column kept in the product with V (value = mean of V)
            den = den + np.exp(sink - mx)
            out = (e @ v + np.exp(sink - mx)[:, None] * v.mean(axis=0)) / den[:, None]
            return out, mx + np.log(den)
        return (e / den[:, None]) @ v, mx + np.log(den)
    return sdpa_rows


@pytest.mark.parametrize("kind", ["sink_ignored", "sink_scaled", "sink_has_value"])
def test_planted_sink_mistakes_are_caught(kind, golden_dir):
    caught = False
    for s, pct in _golden_rows(golden_dir, "sink_mass_128_zero_scores.txt"):
        p, o, vbar = _sink_mass_case(float(s), sdpa=_sdpa_sink_mutant(kind))
        caught |= round(100 * p, 2) != float(pct) or np.max(np.abs(o - (1 - p) * vbar)) > 1e-9
    assert caught


def test_planted_sink_off_by_one_is_caught(golden_dir, monkeypatch):
    real = oa.allowed_mask

    def off_by_one(n_q, n_k, mask_kind, window=0, rows=None, n_sink=0):
        return real(n_q, n_k, mask_kind, window, rows, min(n_sink + 1, n_k) if n_sink else 0)

    monkeypatch.setattr(oa, "allowed_mask", off_by_one)
    rows = [[int(x) for x in r] for r in _golden_rows(golden_dir, "window_sink_mask_n8_w3_s2.txt")]
    assert not np.array_equal(oa.allowed_mask(8, 8, oracle.MASK_SLIDING_WINDOW, 3, n_sink=2).astype(int),
                              np.array(rows))
