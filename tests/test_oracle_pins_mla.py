"""Pins of the oracle's absorbed MLA decode.

"Module 5. Modern Attention Mechanisms", section 7, and "Module 09: Efficient
Attention", the MLA section: the absorbed computation (one transformed query
against the cached latents, values aggregated in latent space, a separate
positional key, scale 1 / sqrt(d_head + d_h^R)) must equal attention with the
per-head keys and values reconstructed explicitly. The cache size is pinned
to the page's DeepSeek-V2 numbers.
"""

import math
import os

import numpy as np
import pytest

import oracle
from oracle import mla as om
from exact_softmax_attention_causal_b200 import accounting, workloads

from test_oracle_pins import _paged_from_contiguous


def _explicit_and_absorbed(rng, H=4, n=23, d_c=12, d_r=4, d_k=6, d_v=5, bs=4):
    """Random up-projections A_h (keys), B_h (values), latents c_t, positional
    keys k^R_t and per-head queries [q^C ; q^R]. Returns the explicit per-head
    attention (keys [A_h c_t ; k^R_t], values B_h c_t, scale 1/sqrt(d_k + d_r))
    and the oracle's absorbed result expanded by B_h."""
    A = rng.standard_normal((H, d_k, d_c))
    Bm = rng.standard_normal((H, d_v, d_c))
    c = rng.standard_normal((n, d_c))
    kr = rng.standard_normal((n, d_r))
    qc = rng.standard_normal((H, d_k))
    qr = rng.standard_normal((H, d_r))
    scale = 1 / math.sqrt(d_k + d_r)
    o_exp, l_exp = [], []
    for h in range(H):
        k = np.concatenate([c @ A[h].T, kr], axis=1)
        v = c @ Bm[h].T
        o, l = oracle.sdpa_rows(np.concatenate([qc[h], qr[h]])[None], k, v, np.ones((1, n), dtype=bool), scale)
        o_exp.append(o[0])
        l_exp.append(l[0])
    # absorbed: q_h = [A_h^T q^C_h ; q^R_h], cache rows [c_t ; k^R_t], paged
    q = np.concatenate([np.einsum("hkc,hk->hc", A, qc), qr], axis=1)[None]
    cache, _, table, lens = _paged_from_contiguous([np.concatenate([c, kr], axis=1)[:, None, :]],
                                                   [np.zeros((n, 1, 1))], bs, 5)
    cache = cache[:, :, 0, :]
    return (np.array(o_exp), np.array(l_exp)), (q, cache, table, lens, Bm, scale, d_c)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_absorbed_equals_explicit_reconstruction(seed):
    (o_exp, l_exp), (q, cache, table, lens, Bm, scale, d_c) = _explicit_and_absorbed(np.random.default_rng(seed))
    o_lat, lse = om.mla_decode_rows_ref(q, cache, table, lens, 0, range(q.shape[1]), d_c, scale)
    o_abs = np.einsum("hvc,hc->hv", Bm, o_lat)  # expand after aggregation: B_h (sum_t p_t c_t)
    np.testing.assert_allclose(o_abs, o_exp, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, l_exp, rtol=0, atol=1e-12)


def test_planted_head_dim_scale_is_caught():
    """Module 09's listed pitfall: dividing by sqrt(d_head) instead of
    sqrt(d_head + d_h^R) must not pass the reconstruction pin."""
    (o_exp, _), (q, cache, table, lens, Bm, scale, d_c) = _explicit_and_absorbed(np.random.default_rng(3))
    d_k, d_r = 6, 4
    o_lat, _ = om.mla_decode_rows_ref(q, cache, table, lens, 0, range(q.shape[1]), d_c, 1 / math.sqrt(d_k))
    assert np.max(np.abs(np.einsum("hvc,hc->hv", Bm, o_lat) - o_exp)) > 1e-3
    assert scale == 1 / math.sqrt(d_k + d_r)


def test_planted_dropped_positional_term_is_caught():
    (o_exp, _), (q, cache, table, lens, Bm, scale, d_c) = _explicit_and_absorbed(np.random.default_rng(4))
    q2 = q.copy()
    q2[..., d_c:] = 0.0  # the positional branch left out of the logit
    o_lat, _ = om.mla_decode_rows_ref(q2, cache, table, lens, 0, range(q.shape[1]), d_c, scale)
    assert np.max(np.abs(np.einsum("hvc,hc->hv", Bm, o_lat) - o_exp)) > 1e-3


def test_mla_cache_numbers_match_the_page(golden_dir):
    rows = [line.split() for line in open(os.path.join(golden_dir, "mla_cache_numbers.txt"))
            if line.strip() and not line.startswith("#")]
    (d_c, d_r, per_token, d_head, groups), = rows
    assert om.mla_cache_bytes(1, 1, int(d_c), int(d_r), 1) == int(per_token)
    assert om.mla_cache_bytes(1, 1, int(d_c), int(d_r), 1) / (2 * int(d_head)) == float(groups)
    assert om.mla_cache_bytes(61, 1000, 512, 64, 2) == 61 * 1000 * 576 * 2
    assert accounting.mla_decode_bytes([1000, 24], 512, 64) == om.mla_cache_bytes(1, 1024, 512, 64, 2)


def test_paged_latent_cache_any_permutation():
    rng = np.random.default_rng(7)
    n, width, d_c = 37, 20, 16
    rows = rng.standard_normal((n, 1, width))
    q = rng.standard_normal((1, 3, width))
    ref = None
    for perm_seed in (1, 2, 3):
        cache, _, table, lens = _paged_from_contiguous([rows], [np.zeros((n, 1, 1))], 8, perm_seed)
        o, l = om.mla_decode_rows_ref(q, cache[:, :, 0, :], table, lens, 0, range(3), d_c, 0.2)
        if ref is None:
            ref = (o, l)
        assert np.array_equal(o, ref[0]) and np.array_equal(l, ref[1])


def test_mla_flop_count():
    # per head per token: 2 * 576 for the logit, 2 * 512 for the latent output
    assert accounting.mla_decode_flops([1], 1, 512, 64) == 2176
    assert accounting.mla_decode_flops([10, 6], 128, 512, 64) == 16 * 128 * 2176


def test_workload_inputs_shapes():
    x = workloads.mla_decode_inputs(2, 4, 32, 8, seq_lens=[5, 40], block_size=16, seed=0)
    assert x.q.shape == (2, 4, 40) and x.cache.shape[1:] == (16, 40)
    o, l = oracle.mla_decode_ref(x.q, x.cache, x.block_table, x.seq_lens, 32, 0.1)
    assert o.shape == (2, 4, 32) and np.isfinite(o).all() and np.isfinite(l).all()
