"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: printed
values (tests/golden/, each file citing its passage), closed forms,
invariants, an independent brute force, or an independent online-softmax
restatement. The last group plants mistakes in a copy of the oracle's
arithmetic and checks that the pins catch them.
"""

import math
import os

import numpy as np
import pytest

import oracle
from oracle import attention as oa
from exact_softmax_attention_causal_b200 import accounting, workloads

MASKS = [(oracle.MASK_FULL, 0), (oracle.MASK_CAUSAL, 0), (oracle.MASK_SLIDING_WINDOW, 1),
         (oracle.MASK_SLIDING_WINDOW, 3), (oracle.MASK_SLIDING_WINDOW, 100)]


def _rand(rng, *shape):
    return rng.standard_normal(shape)


# --------------------------------------------------------------------------
# pin 1: brute force on tiny inputs (pure Python, no numpy matmul)
# --------------------------------------------------------------------------
def _visible_py(i, j, mask_kind, window):
    if mask_kind == oracle.MASK_FULL:
        return True
    if mask_kind == oracle.MASK_CAUSAL:
        return j <= i
    return 0 <= i - j < window


def _brute_force(q, k, v, mask_kind, window, scale):
    """softmax(QK^T * scale + M) V written with scalar loops and math.exp."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    out = np.zeros((B, Hq, N, v.shape[-1]))
    lse = np.zeros((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            kv = h // g
            for i in range(N):
                sc = []
                for j in range(N):
                    if _visible_py(i, j, mask_kind, window):
                        s = 0.0
                        for t in range(d):
                            s += float(q[b, h, i, t]) * float(k[b, kv, j, t])
                        sc.append((j, s * scale))
                mx = max(s for _, s in sc)
                w = [(j, math.exp(s - mx)) for j, s in sc]
                den = sum(x for _, x in w)
                for t in range(v.shape[-1]):
                    out[b, h, i, t] = sum(x * float(v[b, kv, j, t]) for j, x in w) / den
                lse[b, h, i] = mx + math.log(den)
    return out, lse


@pytest.mark.parametrize("hq,hkv", [(4, 2), (4, 4), (4, 1)])
@pytest.mark.parametrize("mask_kind,window", MASKS)
def test_pin1_brute_force(hq, hkv, mask_kind, window):
    rng = np.random.default_rng(100 + hq * 10 + hkv)
    B, N, d = 2, 7, 5
    q, k, v = _rand(rng, B, hq, N, d), _rand(rng, B, hkv, N, d), _rand(rng, B, hkv, N, d)
    scale = 1 / math.sqrt(d)
    o_ref, l_ref = _brute_force(q, k, v, mask_kind, window, scale)
    o, l = oracle.prefill_ref(q, k, v, mask_kind, window, scale)
    assert np.max(np.abs(o - o_ref)) <= 1e-12
    assert np.max(np.abs(l - l_ref)) <= 1e-12


# --------------------------------------------------------------------------
# pin 2: online softmax (the pages' recurrence) == direct softmax
# --------------------------------------------------------------------------
def _online(q, k, v, mask_kind, window, scale, block):
    """FlashAttention's recurrence, restated independently of the oracle.

    Modern Attention Mechanisms, section 8: per row carry (m, l, n); for each
    key tile m' = max(m, max x), alpha = e^(m - m'), p = e^(x - m'),
    l' = alpha l + sum p, n' = alpha n + sum p v; init m = -inf, l = 0, n = 0,
    alpha = 0 on the first non-empty tile, fully masked tiles skipped;
    O = n / l. LSE = m + log l.
    """
    B, Hq, N, d = q.shape
    g = Hq // k.shape[1]
    out = np.zeros((B, Hq, N, v.shape[-1]))
    lse = np.zeros((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            kv = h // g
            for i in range(N):
                m, l, n = -math.inf, 0.0, np.zeros(v.shape[-1])
                for j0 in range(0, N, block):
                    js = [j for j in range(j0, min(N, j0 + block)) if _visible_py(i, j, mask_kind, window)]
                    if not js:
                        continue  # fully masked tile: skipped
                    x = np.array([np.dot(q[b, h, i], k[b, kv, j]) * scale for j in js])
                    m_new = max(m, x.max())
                    alpha = 0.0 if m == -math.inf else math.exp(m - m_new)
                    p = np.exp(x - m_new)
                    l = alpha * l + p.sum()
                    n = alpha * n + (p[:, None] * v[b, kv, js]).sum(axis=0)
                    m = m_new
                out[b, h, i] = n / l
                lse[b, h, i] = m + math.log(l)
    return out, lse


@pytest.mark.parametrize("block", [1, 7, 16, 64])
@pytest.mark.parametrize("mask_kind,window", MASKS)
def test_pin2_online_equals_direct(block, mask_kind, window):
    rng = np.random.default_rng(7)
    B, Hq, Hkv, N, d = 1, 4, 2, 19, 8
    q, k, v = _rand(rng, B, Hq, N, d) * 2, _rand(rng, B, Hkv, N, d), _rand(rng, B, Hkv, N, d)
    scale = 1 / math.sqrt(d)
    o_on, l_on = _online(q, k, v, mask_kind, window, scale, block)
    o, l = oracle.prefill_ref(q, k, v, mask_kind, window, scale)
    assert np.max(np.abs(o - o_on)) <= 1e-12
    assert np.max(np.abs(l - l_on)) <= 1e-12


# --------------------------------------------------------------------------
# pin 3: Hkv == Hq equals independent single-head attention; head order
# --------------------------------------------------------------------------
def _single_head(qh, kh, vh, allowed, scale):
    s = qh @ kh.T * scale
    s = np.where(allowed, s, -np.inf)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    return (p / p.sum(axis=1, keepdims=True)) @ vh


def test_pin3_mha_equals_independent_heads():
    rng = np.random.default_rng(3)
    B, H, N, d = 2, 4, 11, 6
    q, k, v = _rand(rng, B, H, N, d), _rand(rng, B, H, N, d), _rand(rng, B, H, N, d)
    allowed = np.tril(np.ones((N, N), dtype=bool))
    o, _ = oracle.prefill_ref(q, k, v, oracle.MASK_CAUSAL, 0, 0.4)
    for b in range(B):
        for h in range(H):
            np.testing.assert_allclose(o[b, h], _single_head(q[b, h], k[b, h], v[b, h], allowed, 0.4),
                                       rtol=0, atol=1e-12)


def test_pin3_gqa_is_consecutive_repeat_not_tile():
    """Modern Attention Mechanisms, section 6: kv heads repeat consecutively
    (kv0, kv0, ..., kv1, ...); tiling the K/V block gives the wrong heads."""
    rng = np.random.default_rng(5)
    B, Hq, Hkv, N, d = 1, 4, 2, 9, 8
    q, k, v = _rand(rng, B, Hq, N, d), _rand(rng, B, Hkv, N, d), _rand(rng, B, Hkv, N, d)
    o, _ = oracle.prefill_ref(q, k, v, oracle.MASK_CAUSAL, 0, 0.3)
    rep_k, rep_v = np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1)
    o_rep, _ = oracle.prefill_ref(q, rep_k, rep_v, oracle.MASK_CAUSAL, 0, 0.3)
    np.testing.assert_allclose(o, o_rep, rtol=0, atol=1e-13)
    tile_k, tile_v = np.tile(k, (1, 2, 1, 1)), np.tile(v, (1, 2, 1, 1))
    o_tile, _ = oracle.prefill_ref(q, tile_k, tile_v, oracle.MASK_CAUSAL, 0, 0.3)
    assert np.max(np.abs(o - o_tile)) > 1e-2


def test_pin3_rejects_indivisible_heads():
    rng = np.random.default_rng(0)
    with pytest.raises(ValueError):
        oracle.prefill_ref(_rand(rng, 1, 3, 4, 2), _rand(rng, 1, 2, 4, 2), _rand(rng, 1, 2, 4, 2),
                           oracle.MASK_CAUSAL, 0, 1.0)


# --------------------------------------------------------------------------
# pin 4: causal row 0 sees only key 0 -> O = v_0, LSE = scale q_0.k_0
# --------------------------------------------------------------------------
def test_pin4_causal_row0_is_v0():
    rng = np.random.default_rng(11)
    B, Hq, Hkv, N, d = 2, 4, 2, 13, 16
    q, k, v = _rand(rng, B, Hq, N, d), _rand(rng, B, Hkv, N, d), _rand(rng, B, Hkv, N, d)
    o, l = oracle.prefill_ref(q, k, v, oracle.MASK_CAUSAL, 0, 0.25)
    for b in range(B):
        for h in range(Hq):
            assert np.array_equal(o[b, h, 0], v[b, h // 2, 0])
            assert abs(l[b, h, 0] - 0.25 * float(np.dot(q[b, h, 0], k[b, h // 2, 0]))) <= 1e-14


def test_pin4_causal_rows_match_printed_table(golden_dir):
    rows = {}
    for line in open(os.path.join(golden_dir, "causal_rows_n6.txt")):
        if line.startswith("#") or not line.strip():
            continue
        r, cols = line.split(":")
        rows[int(r)] = [int(c) for c in cols.split()]
    allowed = oracle.allowed_mask(6, 6, oracle.MASK_CAUSAL)
    for r, cols in rows.items():
        assert np.nonzero(allowed[r])[0].tolist() == cols


# --------------------------------------------------------------------------
# pin 5: equal scores give the mean of the visible values; LSE = ln(count)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("mask_kind,window", MASKS)
def test_pin5_equal_scores_mean(mask_kind, window):
    rng = np.random.default_rng(2)
    B, Hq, Hkv, N, d = 1, 2, 1, 10, 4
    q = np.zeros((B, Hq, N, d))
    k, v = _rand(rng, B, Hkv, N, d), _rand(rng, B, Hkv, N, d)
    o, l = oracle.prefill_ref(q, k, v, mask_kind, window, 1.0)
    for i in range(N):
        if mask_kind == oracle.MASK_FULL:
            vis = list(range(N))
        elif mask_kind == oracle.MASK_CAUSAL:
            vis = list(range(i + 1))
        else:
            vis = list(range(max(0, i - window + 1), i + 1))
        for h in range(Hq):
            np.testing.assert_allclose(o[0, h, i], v[0, 0, vis].mean(axis=0), rtol=0, atol=1e-14)
            assert abs(l[0, h, i] - math.log(len(vis))) <= 1e-14


# --------------------------------------------------------------------------
# pin 6: a window of at least N equals causal, exactly
# --------------------------------------------------------------------------
def test_pin6_wide_window_is_causal():
    rng = np.random.default_rng(4)
    B, Hq, Hkv, N, d = 1, 2, 2, 12, 8
    q, k, v = _rand(rng, B, Hq, N, d), _rand(rng, B, Hkv, N, d), _rand(rng, B, Hkv, N, d)
    o_c, l_c = oracle.prefill_ref(q, k, v, oracle.MASK_CAUSAL, 0, 0.5)
    for w in (N, N + 5, 2 * N):
        o_w, l_w = oracle.prefill_ref(q, k, v, oracle.MASK_SLIDING_WINDOW, w, 0.5)
        assert np.array_equal(o_w, o_c) and np.array_equal(l_w, l_c)


def test_pin11_window_mask_matches_printed_matrix(golden_dir):
    rows = [[int(x) for x in line.split()]
            for line in open(os.path.join(golden_dir, "sliding_window_mask_n6_w3.txt"))
            if line.strip() and not line.startswith("#")]
    assert np.array_equal(oracle.allowed_mask(6, 6, oracle.MASK_SLIDING_WINDOW, 3).astype(int), np.array(rows))


def test_window_one_is_self_only():
    rng = np.random.default_rng(9)
    q, k, v = _rand(rng, 1, 1, 6, 3), _rand(rng, 1, 1, 6, 3), _rand(rng, 1, 1, 6, 3)
    o, _ = oracle.prefill_ref(q, k, v, oracle.MASK_SLIDING_WINDOW, 1, 1.0)
    assert np.array_equal(o[0, 0], v[0, 0])


def test_prefix_alignment_is_bottom_right():
    """Modern Attention Mechanisms, section 4: after a prefix of P keys, query
    row i has position P + i, so the last query row sees every key."""
    m = oracle.allowed_mask(2, 6, oracle.MASK_CAUSAL)
    assert m.tolist() == [[1, 1, 1, 1, 1, 0], [1, 1, 1, 1, 1, 1]]


def test_fully_masked_row_rejected():
    with pytest.raises(ValueError):
        oa.sdpa_rows(np.ones((2, 3)), np.ones((4, 3)), np.ones((4, 3)),
                     np.array([[True, False, False, False], [False] * 4]), 1.0)


# --------------------------------------------------------------------------
# pin 7: paged == contiguous under any permutation
# --------------------------------------------------------------------------
def _paged_from_contiguous(k_seq, v_seq, block_size, perm_seed, extra=3):
    """Scatter contiguous per-sequence caches into a permuted pool."""
    import torch

    B = len(k_seq)
    lens = [x.shape[0] for x in k_seq]
    gen = torch.Generator("cpu").manual_seed(perm_seed)
    maxb = max(workloads.blocks_needed(n, block_size) for n in lens)
    table, pool = workloads.paged_layout(lens, block_size, maxb, gen, extra_blocks=extra)
    hkv, d = k_seq[0].shape[1:]
    kc = np.full((pool, block_size, hkv, d), np.nan)
    vc = np.full((pool, block_size, hkv, d), np.nan)
    for b in range(B):
        for t in range(lens[b]):
            phys = int(table[b, t // block_size])
            kc[phys, t % block_size] = k_seq[b][t]
            vc[phys, t % block_size] = v_seq[b][t]
    return kc, vc, table.numpy(), np.array(lens)


def test_pin7_paged_equals_contiguous_any_permutation():
    rng = np.random.default_rng(21)
    Hq, Hkv, d, bs = 4, 2, 8, 4
    lens = [5, 13, 1, 16]
    k_seq = [rng.standard_normal((n, Hkv, d)) for n in lens]
    v_seq = [rng.standard_normal((n, Hkv, d)) for n in lens]
    q = rng.standard_normal((len(lens), Hq, d))
    results = []
    for seed in (1, 2, 3):
        kc, vc, table, sl = _paged_from_contiguous(k_seq, v_seq, bs, seed)
        gk = oracle.gather_paged_ref(kc, table, sl, max(lens))
        for b, n in enumerate(lens):
            assert np.array_equal(gk[b, :, :n].transpose(1, 0, 2), k_seq[b])
            assert np.all(gk[b, :, n:] == 0)
        results.append(oracle.decode_paged_ref(q, kc, vc, table, sl, 0.35))
    for o, l in results[1:]:
        assert np.array_equal(o, results[0][0]) and np.array_equal(l, results[0][1])
    # and it equals contiguous attention over the unpaged cache
    for b, n in enumerate(lens):
        for h in range(Hq):
            o_c = _single_head(q[b, h][None], k_seq[b][:, h // 2], v_seq[b][:, h // 2],
                               np.ones((1, n), dtype=bool), 0.35)
            np.testing.assert_allclose(results[0][0][b, h], o_c[0], rtol=0, atol=1e-13)


def test_pin7_gather_rejects_bad_entries():
    kc = np.zeros((2, 4, 1, 2))
    with pytest.raises(ValueError):
        oracle.gather_paged_ref(kc, np.array([[0, 2]]), np.array([6]), 8)
    with pytest.raises(ValueError):
        oracle.gather_paged_ref(kc, np.array([[0, -1]]), np.array([5]), 8)


def test_paging_demo_counts(golden_dir):
    kv = {}
    for line in open(os.path.join(golden_dir, "paging_demo.txt")):
        if line.startswith("#") or not line.strip():
            continue
        key, *vals = line.split()
        kv[key] = [int(x) for x in vals]
    lens, bs = kv["lengths"], kv["block_size"][0]
    blocks = sum(workloads.blocks_needed(n, bs) for n in lens)
    assert blocks == kv["paged_blocks"][0]
    assert blocks * bs == kv["paged_slots"][0]
    assert blocks * bs - sum(lens) == kv["paged_waste_tokens"][0]
    assert 512 * len(lens) == kv["contiguous_slots"][0]
    assert workloads.blocks_needed(kv["tiny_tokens"][0], kv["tiny_block_size"][0]) == kv["tiny_blocks"][0]


# --------------------------------------------------------------------------
# pin 8: KV size formula against printed values
# --------------------------------------------------------------------------
def test_pin8_kv_cache_bytes(golden_dir):
    n = 0
    for line in open(os.path.join(golden_dir, "kv_cache_bytes.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        L, hkv, dh, b, pos, expect = (int(x) for x in line.split())
        assert oracle.kv_cache_bytes(L, hkv, dh, b, pos) == expect
        n += 1
    assert n == 13
    # gpt-oss window-capped total: 4.50439453125 GiB (Modern Attention Mechanisms, section 5)
    total = oracle.kv_cache_bytes(18, 8, 64, 2, 131072) + oracle.kv_cache_bytes(18, 8, 64, 2, 128)
    assert total / 2**30 == 4.50439453125


# --------------------------------------------------------------------------
# pin 9: cached decode == the matching row of a full causal forward
# --------------------------------------------------------------------------
def test_pin9_cached_decode_equals_full_forward():
    rng = np.random.default_rng(13)
    Hq, Hkv, N, d, bs = 4, 2, 11, 8, 4
    q = rng.standard_normal((1, Hq, N, d))
    k = rng.standard_normal((1, Hkv, N, d))
    v = rng.standard_normal((1, Hkv, N, d))
    o_full, l_full = oracle.prefill_ref(q, k, v, oracle.MASK_CAUSAL, 0, 0.3)
    for t in range(1, N + 1):
        k_seq = [k[0, :, :t].transpose(1, 0, 2)]
        v_seq = [v[0, :, :t].transpose(1, 0, 2)]
        kc, vc, table, sl = _paged_from_contiguous(k_seq, v_seq, bs, t)
        o_d, l_d = oracle.decode_paged_ref(q[:, :, t - 1], kc, vc, table, sl, 0.3)
        np.testing.assert_allclose(o_d[0], o_full[0, :, t - 1], rtol=0, atol=1e-13)
        np.testing.assert_allclose(l_d[0], l_full[0, :, t - 1], rtol=0, atol=1e-13)


# --------------------------------------------------------------------------
# pin 10: LSE merge of any split == the single pass
# --------------------------------------------------------------------------
@pytest.mark.parametrize("cuts", [(5,), (1, 2, 3), (0, 7, 7, 20), (10, 19)])
def test_pin10_split_merge(cuts):
    rng = np.random.default_rng(17)
    T, d = 23, 6
    q = rng.standard_normal(d) * 3
    k, v = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    o_all, l_all = oa.sdpa_rows(q[None], k, v, np.ones((1, T), dtype=bool), 0.5)
    bounds = [0, *cuts, T]
    o_parts, l_parts = [], []
    for a, b in zip(bounds[:-1], bounds[1:]):
        if a == b:  # empty chunk: no keys, lse = -inf, output unused
            o_parts.append(np.zeros(d))
            l_parts.append(-np.inf)
            continue
        o_s, l_s = oa.sdpa_rows(q[None], k[a:b], v[a:b], np.ones((1, b - a), dtype=bool), 0.5)
        o_parts.append(o_s[0])
        l_parts.append(l_s[0])
    o_m, l_m = oracle.lse_merge_ref(np.array(o_parts), np.array(l_parts))
    np.testing.assert_allclose(o_m, o_all[0], rtol=0, atol=1e-13)
    assert abs(l_m - l_all[0]) <= 1e-13


# --------------------------------------------------------------------------
# accounting helpers against brute-force mask counts
# --------------------------------------------------------------------------
@pytest.mark.parametrize("n,mask,w", [(1, "causal", 0), (37, "causal", 0), (37, "full", 0), (37, "window", 1),
                                      (37, "window", 8), (37, "window", 37), (37, "window", 90)])
def test_visible_pairs_closed_form(n, mask, w):
    kind = accounting.MASK_IDS[mask]
    assert accounting.visible_pairs(n, mask, w) == int(oracle.allowed_mask(n, n, kind, w).sum())


def test_config_flop_counts():
    # 4 * B * Hq * d * pairs, with the pair counts written out by hand.
    assert accounting.prefill_flops(4, 32, 4096, 128, "causal") == 4 * 4 * 32 * 128 * (4096 * 4097 // 2)
    assert accounting.prefill_flops(1, 32, 32768, 128, "causal") == 4 * 32 * 128 * (32768 * 32769 // 2)
    assert accounting.prefill_flops(1, 32, 32768, 128, "window", 4096) == \
        4 * 32 * 128 * (4096 * 4097 // 2 + (32768 - 4096) * 4096)
    assert accounting.prefill_flops(2, 32, 8192, 128, "causal") == 4 * 2 * 32 * 128 * (8192 * 8193 // 2)
    # the rounded figures quoted for these workloads: 0.5499, 8.796, 2.062, 1.0996 TFLOP
    assert round(accounting.prefill_flops(4, 32, 4096, 128, "causal") / 1e12, 4) == 0.5499
    assert round(accounting.prefill_flops(1, 32, 32768, 128, "causal") / 1e12, 3) == 8.796
    assert round(accounting.prefill_flops(1, 32, 32768, 128, "window", 4096) / 1e12, 3) == 2.062


# --------------------------------------------------------------------------
# planted mistakes: a wrong oracle must fail the pins
# --------------------------------------------------------------------------
def _mutant(kind):
    def sdpa_rows(q_rows, k, v, allowed, scale):
        q_rows, k, v = (np.asarray(x, dtype=np.float64) for x in (q_rows, k, v))
        s = q_rows @ k.T * (1.0 if kind == "no_scale" else scale)
        if kind == "no_mask":
            allowed = np.ones_like(allowed)
        s = np.where(allowed, s, -np.inf)
        mx = s.max(axis=1)
        e = np.exp(s - mx[:, None])
        den = e.sum(axis=1)
        vv = v[::-1] if kind == "reversed_v" else v
        out = (e / den[:, None]) @ vv
        lse = mx + np.log(den) + (1e-6 if kind == "lse_offset" else 0.0)
        return out, lse
    return sdpa_rows


@pytest.mark.parametrize("kind", ["no_scale", "no_mask", "reversed_v", "lse_offset"])
def test_planted_mistakes_are_caught(kind, monkeypatch):
    monkeypatch.setattr(oa, "sdpa_rows", _mutant(kind))
    rng = np.random.default_rng(1)
    B, N, d = 1, 6, 4
    q, k, v = _rand(rng, B, 4, N, d), _rand(rng, B, 2, N, d), _rand(rng, B, 2, N, d)
    o_ref, l_ref = _brute_force(q, k, v, oracle.MASK_CAUSAL, 0, 0.5)
    o, l = oa.prefill_ref(q, k, v, oracle.MASK_CAUSAL, 0, 0.5)
    assert np.max(np.abs(o - o_ref)) > 1e-12 or np.max(np.abs(l - l_ref)) > 1e-12


def test_planted_wrong_head_map_is_caught(monkeypatch):
    # tile order (h % Hkv) instead of consecutive groups (h // g)
    monkeypatch.setattr(oa, "kv_head_of", lambda h, hq, hkv: h % hkv)
    rng = np.random.default_rng(5)
    q, k, v = _rand(rng, 1, 4, 5, 3), _rand(rng, 1, 2, 5, 3), _rand(rng, 1, 2, 5, 3)
    o, _ = oa.prefill_ref(q, k, v, oracle.MASK_CAUSAL, 0, 0.5)
    o_ref, _ = _brute_force(q, k, v, oracle.MASK_CAUSAL, 0, 0.5)
    assert np.max(np.abs(o - o_ref)) > 1e-3


def test_planted_wrong_window_is_caught(monkeypatch):
    # a window that admits w + 1 keys (i - w <= j <= i) instead of w
    real = oa.allowed_mask

    def wide(n_q, n_k, mask_kind, window=0):
        if mask_kind == oracle.MASK_SLIDING_WINDOW:
            return real(n_q, n_k, mask_kind, window + 1)
        return real(n_q, n_k, mask_kind, window)

    monkeypatch.setattr(oa, "allowed_mask", wide)
    rng = np.random.default_rng(6)
    q, k, v = _rand(rng, 1, 2, 8, 3), _rand(rng, 1, 1, 8, 3), _rand(rng, 1, 1, 8, 3)
    o, _ = oa.prefill_ref(q, k, v, oracle.MASK_SLIDING_WINDOW, 3, 0.5)
    o_ref, _ = _brute_force(q, k, v, oracle.MASK_SLIDING_WINDOW, 3, 0.5)
    assert np.max(np.abs(o - o_ref)) > 1e-3


# --------------------------------------------------------------------------
# prefix (chunked) prefill over a paged context
# --------------------------------------------------------------------------
def test_paged_prefill_square_case_is_prefill():
    """seq_len == Nq: the chunk is the whole sequence, so the paged prefix
    prefill is the plain prefill of the gathered cache."""
    rng = np.random.default_rng(31)
    Hq, Hkv, N, d, bs = 4, 2, 9, 6, 4
    q = rng.standard_normal((1, Hq, N, d))
    k = rng.standard_normal((1, Hkv, N, d))
    v = rng.standard_normal((1, Hkv, N, d))
    kc, vc, table, sl = _paged_from_contiguous([k[0].transpose(1, 0, 2)], [v[0].transpose(1, 0, 2)], bs, 5)
    for kind, w in [(oracle.MASK_CAUSAL, 0), (oracle.MASK_FULL, 0), (oracle.MASK_SLIDING_WINDOW, 3)]:
        o_p, l_p = oracle.prefill_paged_ref(q, kc, vc, table, sl, kind, w, 0.4)
        o_c, l_c = oracle.prefill_ref(q, k, v, kind, w, 0.4)
        assert np.array_equal(o_p, o_c) and np.array_equal(l_p, l_c)


@pytest.mark.parametrize("kind,w", [(oracle.MASK_CAUSAL, 0), (oracle.MASK_SLIDING_WINDOW, 4)])
def test_chunked_prefill_equals_full_forward(kind, w):
    """Module 09, "Chunked Prefill": slicing a prompt into chunks changes the
    schedule, never the result. Chunk c's rows, attending to every position up
    to the chunk's end, equal the same rows of the one-shot prefill."""
    rng = np.random.default_rng(37)
    Hq, Hkv, N, d, bs = 2, 1, 13, 5, 4
    q = rng.standard_normal((1, Hq, N, d))
    k = rng.standard_normal((1, Hkv, N, d))
    v = rng.standard_normal((1, Hkv, N, d))
    o_full, l_full = oracle.prefill_ref(q, k, v, kind, w, 0.5)
    for a, b in [(0, 5), (5, 6), (6, 13)]:
        kc, vc, table, sl = _paged_from_contiguous([k[0, :, :b].transpose(1, 0, 2)],
                                                   [v[0, :, :b].transpose(1, 0, 2)], bs, b)
        o_c, l_c = oracle.prefill_paged_ref(q[:, :, a:b], kc, vc, table, sl, kind, w, 0.5)
        np.testing.assert_allclose(o_c[0], o_full[0, :, a:b], rtol=0, atol=1e-13)
        np.testing.assert_allclose(l_c[0], l_full[0, :, a:b], rtol=0, atol=1e-13)


@pytest.mark.parametrize("n_k,n_q,mask,w", [(10, 10, "causal", 0), (10, 3, "causal", 0), (300, 77, "full", 0),
                                            (300, 77, "window", 100), (300, 77, "window", 250), (300, 77, "window", 5),
                                            (77, 77, "window", 1000), (5, 1, "window", 2)])
def test_prefix_visible_pairs_closed_form(n_k, n_q, mask, w):
    kind = accounting.MASK_IDS[mask]
    assert accounting.prefix_visible_pairs(n_k, n_q, mask, w) == int(oracle.allowed_mask(n_q, n_k, kind, w).sum())


@pytest.mark.parametrize("n,mask,w", [(9, "full", 0), (9, "causal", 0), (9, "window", 4), (9, "window", 20)])
def test_row_visible_keys_sum_to_visible_pairs(n, mask, w):
    kind = accounting.MASK_IDS[mask]
    counts = oracle.allowed_mask(n, n, kind, w).sum(axis=1).tolist()
    assert counts == [accounting.row_visible_keys(n, i, mask, w) for i in range(n)]
    assert sum(counts) == accounting.visible_pairs(n, mask, w)
