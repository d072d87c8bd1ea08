"""Plain fp64 definition of Multi-head Latent Attention (MLA) decode in its
absorbed form.

TEST INFRASTRUCTURE ONLY (see the package docstring): slow, obviously correct,
CPU-only, never on the product path.

Sources (page title, section):

* "Module 5. Modern Attention Mechanisms" (vladkulikov.com), section 7 "MLA:
  cache a shared latent and move the projections": with k_t = A c_t and
  v_t = B c_t, q.k_t = (A^T q).c_t, so one transformed query is compared with
  every cached latent c_t, and sum_t p_t v_t = B (sum_t p_t c_t), so values are
  aggregated in latent space and expanded afterwards. A separate small RoPE
  key is cached beside the latent and its term is added to the logit.
* "Module 09: Efficient Attention" (learnllm.pages.dev), section "Multi-head
  Latent Attention: A Different Lever": each head's key and query are the
  concatenations [k^C ; k^R] and [q^C ; q^R], the score is their dot product
  divided by sqrt(d_head + d_h^R), and the cache holds d_c + d_h^R numbers per
  token per layer (DeepSeek-V2: d_c = 512, d_h^R = 64, 128 heads of 128).

Absorbed decode, as computed here: the query of head h is the row
[A_h^T q^C_h ; q^R_h] (d_c + d_R numbers); token t's cache row is
[c_t ; k^R_t] (the same width, shared by every head). The logit is the dot
product of the two rows times `scale` (1 / sqrt(d_head + d_R) per the pages),
the softmax runs over the cached tokens, and the output is the latent
sum_t p_t c_t (d_c numbers; the value up-projection B_h is applied by the
caller). LSE is the natural-log log-sum-exp of the scaled logits.
"""

from __future__ import annotations

import numpy as np

from .attention import _as_f64, _as_int, _gather_one, sdpa_rows


def mla_cache_bytes(layers: int, positions: int, d_latent: int, d_rope: int, bytes_per_elem: int) -> int:
    """L * n * (d_c + d_h^R) * b ("Module 09", MLA section: no factor of two
    for K and V, nothing that scales with the head count)."""
    return layers * positions * (d_latent + d_rope) * bytes_per_elem


def mla_decode_rows_ref(q, cache, block_table, seq_lens, b: int, heads, d_latent: int, scale: float):
    """One absorbed MLA decode query per head of sequence b against its paged
    latent cache.

    q [B, H, d_c + d_R] (absorbed content query, then rotated positional
    query); cache [num_blocks, block_size, d_c + d_R] (latent, then positional
    key), token t of sequence b in slot t % block_size of block
    block_table[b][t // block_size] ("Module 09", paged cache section). Every
    cached token is visible to the new query. Returns
    (O_latent [len(heads), d_c], LSE [len(heads)]) in float64.
    """
    n = int(_as_int(seq_lens)[b])
    if n <= 0:
        raise ValueError("a decode row needs at least one cached token")
    width = cache.shape[-1]
    if q.shape[-1] != width or not 0 < d_latent < width:
        raise ValueError("q and cache rows must both be d_c + d_R wide")
    rows = _gather_one(cache, _as_int(block_table)[b], n)  # [n, d_c + d_R]
    qb = _as_f64(q[b])
    allowed = np.ones((1, n), dtype=bool)
    outs, lses = [], []
    for h in heads:
        # keys: the whole row (content and positional parts); values: the latent part
        o, l = sdpa_rows(qb[h][None, :], rows, rows[:, :d_latent], allowed, scale)
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.asarray(lses)


def mla_decode_ref(q, cache, block_table, seq_lens, d_latent: int, scale: float, seqs=None):
    """Absorbed MLA decode for every head of the sequences in `seqs` (all when
    None): (O_latent [B, H, d_c], LSE [B, H]); other sequences stay zero."""
    b_, h_ = q.shape[0], q.shape[1]
    out = np.zeros((b_, h_, d_latent), dtype=np.float64)
    lse = np.zeros((b_, h_), dtype=np.float64)
    for bi in (range(b_) if seqs is None else seqs):
        o, l = mla_decode_rows_ref(q, cache, block_table, seq_lens, bi, range(h_), d_latent, scale)
        out[bi] = o
        lse[bi] = l
    return out, lse
