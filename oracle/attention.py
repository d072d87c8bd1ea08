"""Plain fp64 definition of exact softmax attention, prefill and paged decode.

TEST INFRASTRUCTURE ONLY (see the package docstring): slow, obviously correct,
CPU-only, never on the product path.

Sources (page title, section):

* "Module 5. Modern Attention Mechanisms" (vladkulikov.com, modern LLMs,
  module 04), section 4 "SDPA, masks, and the square-root scale": the
  operator softmax(QK^T/sqrt(d_h) + M)V, the additive mask (0 allowed, -inf
  forbidden), position-aware causality p_k <= p_q, the window rule
  0 <= p_q - p_k < W including the current position, and the fully masked row
  policy (we take "reject").
* same page, section 6 "GQA is a grouping invariant": query head h uses KV
  head floor(h / g), g = H_q / H_kv, consecutive groups kv0, kv0, ..., kv1.
* same page, section 1 "What grows with the context?" and section 5: the KV
  bytes per token 2 * L * H_kv * d_h * b.
* "Module 09: Efficient Attention" (learnllm.pages.dev), section "Code: A
  Paged KV Cache from Scratch": the pool (num_blocks, block_size,
  num_kv_heads, head_dim) and token t of a sequence at
  (block_table[t // block_size], t % block_size).
* "USAAIO Lesson 90: KV Cache & Attention Efficiency" (naruhodotutoring.com),
  part 2: a decode step attends the new query over the whole cache, its own
  K/V already appended.
* "Inference attention" post (brunomaga.github.io), section "FlashDecoding":
  partial outputs of key chunks with their softmax statistics, combined with
  the online softmax's rescaling.
* "Module 5. Modern Attention Mechanisms", section 10 "Attention sink refers
  to two different objects" and section 12 (its mask builder and SDPA): the
  StreamingLLM rule that keeps the first n_sink real positions visible next
  to a finite window, and the learned per-head sink logit s_h, an extra score
  column that takes softmax mass but adds no value vector.

The oracle computes a DIRECT softmax: it materialises full score rows (in
row blocks only to bound memory), applies the mask, subtracts the row max,
exponentiates, normalises and multiplies by V. No online softmax, no tiling.

Precision: the caller passes the bf16-rounded inputs the GPU sees; they are
widened exactly to float64 and everything after that is float64.

LSE is the natural-log log-sum-exp over the visible keys of the scaled scores,
log(sum_j exp(scale * q.k_j)): the "running log-sum-exp" the slides name,
written as m + log(l) in the online softmax's notation. With a learned sink
the row that is normalised has one more column, so LSE includes it:
log(sum_j exp(scale * q.k_j) + exp(s_h)) (the log of the softmax denominator).
"""

from __future__ import annotations

import math

import numpy as np

MASK_FULL = 0
MASK_CAUSAL = 1
MASK_SLIDING_WINDOW = 2


def _as_f64(x) -> np.ndarray:
    """Widen an array-like (numpy array or CPU/GPU torch tensor) to float64.

    bf16 -> fp64 is exact, so the oracle sees exactly the values the GPU sees.
    """
    if hasattr(x, "detach"):  # a torch tensor; imported lazily, CPU ops only
        import torch

        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _as_int(x) -> np.ndarray:
    if hasattr(x, "detach"):
        return x.detach().cpu().numpy().astype(np.int64)
    return np.asarray(x, dtype=np.int64)


def allowed_mask(n_q: int, n_k: int, mask_kind: int, window: int = 0, rows=None, n_sink: int = 0) -> np.ndarray:
    """Boolean [n_q, n_k] visibility, True = query row i may attend key j.

    Modern Attention Mechanisms, section 4: causality compares positions,
    p_k <= p_q; a window of W positions including the current one requires
    0 <= p_q - p_k < W. After a prefix of length P = n_k - n_q, query row i has
    position P + i (keys sit at positions 0..n_k-1). For the square case
    (n_q == n_k) this is j <= i and i - W < j <= i. ``rows`` restricts the
    result to those query rows (all rows when None).

    Section 10 / section 12 (StreamingLLM sinks): with a finite window, the
    first ``n_sink`` positions stay visible to every query at or after them,
    p_k < n_sink and p_k <= p_q. n_sink is accepted only with the window mask
    and must lie in [0, n_k].
    """
    if n_q <= 0 or n_k <= 0 or n_q > n_k:
        raise ValueError("need 0 < n_q <= n_k")
    if n_sink < 0 or n_sink > n_k:
        raise ValueError("n_sink must satisfy 0 <= n_sink <= n_k")
    if n_sink and mask_kind != MASK_SLIDING_WINDOW:
        raise ValueError("n_sink is meaningful only together with a finite window")
    rows = np.arange(n_q) if rows is None else np.asarray(rows, dtype=np.int64)
    p_q = (n_k - n_q) + rows[:, None]
    p_k = np.arange(n_k)[None, :]
    if mask_kind == MASK_FULL:
        return np.ones((rows.shape[0], n_k), dtype=bool)
    if mask_kind == MASK_CAUSAL:
        return p_k <= p_q
    if mask_kind == MASK_SLIDING_WINDOW:
        if window <= 0:
            raise ValueError("window must be positive")
        diff = p_q - p_k
        allowed = (diff >= 0) & (diff < window)
        return allowed | ((p_k < n_sink) & (p_k <= p_q))
    raise ValueError(f"unknown mask kind {mask_kind}")


def sdpa_rows(q_rows, k, v, allowed, scale: float, sink=None):
    """Direct softmax attention of some query rows against one K/V head.

    Modern Attention Mechanisms, section 4 (the SDPA definition and the
    additive -inf mask) and section 12 (subtract the row maximum, exponentiate,
    normalise; a row with no visible key is rejected, the "error" policy).

    ``sink`` (a finite scalar or one value per row) is section 10's learned
    sink logit: one more score column, in the units of the scaled scores,
    that enters the row maximum and the denominator and is dropped before the
    product with V. With a sink a row without visible keys is well defined
    (all mass on the sink: O = 0, LSE = sink).

    q_rows [R, d], k [T, d], v [T, d_v], allowed [R, T] bool.
    Returns (O [R, d_v], LSE [R]) in float64.
    """
    q_rows = _as_f64(q_rows)
    k = _as_f64(k)
    v = _as_f64(v)
    allowed = np.asarray(allowed, dtype=bool)
    has_key = allowed.any(axis=1)
    if sink is None and not has_key.all():
        bad = np.nonzero(~has_key)[0][:8].tolist()
        raise ValueError(f"fully masked rows: {bad}")
    scores = (q_rows @ k.T) * float(scale)
    scores = np.where(allowed, scores, -np.inf)
    token_max = scores.max(axis=1)  # -inf on a row without keys
    if sink is None:
        row_max = token_max
    else:
        sink = np.broadcast_to(_as_f64(sink), token_max.shape)
        if not np.isfinite(sink).all():
            raise ValueError("sink logits must be finite")
        row_max = np.maximum(token_max, sink)
    e = np.exp(scores - row_max[:, None])  # exp(-inf) == 0 for masked keys
    denom = e.sum(axis=1)
    if sink is not None:
        denom = denom + np.exp(sink - row_max)
    out = (e / denom[:, None]) @ v
    lse = row_max + np.log(denom)
    return out, lse


def _check_heads(hq: int, hkv: int) -> int:
    # Modern Attention Mechanisms, section 2/6: g = H_q / H_kv must be an integer.
    if hq <= 0 or hkv <= 0 or hq % hkv != 0:
        raise ValueError("Hq must be a positive multiple of Hkv")
    return hq // hkv


def kv_head_of(h: int, hq: int, hkv: int) -> int:
    """Query head h reads KV head floor(h / g), g = Hq / Hkv (Modern Attention
    Mechanisms, section 6: consecutive groups kv0, kv0, ..., kv1, kv1, ...)."""
    return h // _check_heads(hq, hkv)


def prefill_ref(q, k, v, mask_kind: int, window: int, scale: float, row_block: int = 512):
    """Prefill attention over grouped-query heads, full output.

    q [B, Hq, N, d]; k, v [B, Hkv, N, d] (heads on axis 1, as in Modern
    Attention Mechanisms, section 6, block B05). Query head h reads KV head
    h // (Hq // Hkv). Returns (O [B, Hq, N, d], LSE [B, Hq, N]) float64.
    Row blocks only bound memory; every row sees its full score row.
    """
    q = _as_f64(q)
    k = _as_f64(k)
    v = _as_f64(v)
    b_, hq, n, d = q.shape
    _, hkv, n_k, _ = k.shape
    _check_heads(hq, hkv)
    allowed = allowed_mask(n, n_k, mask_kind, window)
    out = np.empty((b_, hq, n, v.shape[-1]), dtype=np.float64)
    lse = np.empty((b_, hq, n), dtype=np.float64)
    for bi in range(b_):
        for h in range(hq):
            kvh = kv_head_of(h, hq, hkv)
            for r0 in range(0, n, row_block):
                r1 = min(n, r0 + row_block)
                o_blk, l_blk = sdpa_rows(q[bi, h, r0:r1], k[bi, kvh], v[bi, kvh], allowed[r0:r1], scale)
                out[bi, h, r0:r1] = o_blk
                lse[bi, h, r0:r1] = l_blk
    return out, lse


def prefill_rows_ref(q, k, v, b: int, h: int, rows, mask_kind: int, window: int, scale: float):
    """The same definition as prefill_ref, for chosen rows of one (batch, head).

    Used for sampled parity at sizes where the full oracle would take too long.
    Returns (O [len(rows), d], LSE [len(rows)]) float64.
    """
    hq, n = q.shape[1], q.shape[2]
    hkv, n_k = k.shape[1], k.shape[2]
    kvh = kv_head_of(h, hq, hkv)
    rows = np.asarray(rows, dtype=np.int64)
    allowed = allowed_mask(n, n_k, mask_kind, window, rows=rows)
    q_rows = _as_f64(q[b, h])[rows]
    return sdpa_rows(q_rows, _as_f64(k[b, kvh]), _as_f64(v[b, kvh]), allowed, scale)


def gather_paged_ref(cache, block_table, seq_lens, max_seq_len: int):
    """Walk each sequence's block table token by token into a contiguous cache.

    Module 09: Efficient Attention, "Code: A Paged KV Cache from Scratch":
    token t sits in slot t % block_size of physical block
    block_table[t // block_size]. cache [num_blocks, block_size, Hkv, d].
    Returns [B, Hkv, max_seq_len, d] float64, zero beyond each seq_len.
    Raises on a referenced table entry outside [0, num_blocks).
    """
    cache = _as_f64(cache)
    table = _as_int(block_table)
    lens = _as_int(seq_lens)
    num_blocks, bs, hkv, d = cache.shape
    b_ = table.shape[0]
    out = np.zeros((b_, hkv, max_seq_len, d), dtype=np.float64)
    for bi in range(b_):
        n = int(lens[bi])
        if n < 0 or n > max_seq_len:
            raise ValueError(f"seq_len {n} outside [0, {max_seq_len}]")
        for t in range(n):
            phys = int(table[bi, t // bs])
            if phys < 0 or phys >= num_blocks:
                raise ValueError(f"block table entry {phys} outside the pool")
            out[bi, :, t, :] = cache[phys, t % bs]
    return out


def _gather_one(cache, table_row, n: int) -> np.ndarray:
    """Token-by-token gather of one sequence: [n, Hkv, d] float64. Each row is
    widened as it is copied, so the pool itself is never converted whole."""
    num_blocks, bs = cache.shape[0], cache.shape[1]
    rows = np.empty((n,) + tuple(cache.shape[2:]), dtype=np.float64)
    for t in range(n):
        phys = int(table_row[t // bs])
        if phys < 0 or phys >= num_blocks:
            raise ValueError(f"block table entry {phys} outside the pool")
        rows[t] = _as_f64(cache[phys, t % bs])
    return rows


def decode_rows_ref(q, k_cache, v_cache, block_table, seq_lens, b: int, heads, scale: float, window: int = 0,
                    n_sink: int = 0, sinks=None):
    """One decode query per head of sequence b against its paged cache.

    USAAIO Lesson 90, part 2: the new query attends over the cached keys and
    values (its own already appended), so it sits at position n - 1. K/V are
    gathered through the block table (Module 09, paged cache section) and the
    direct softmax of sdpa_rows does the rest. Without a window every cached
    token is visible; with ``window`` = W > 0 the query sees the positions
    n - W .. n - 1 plus the first ``n_sink`` (allowed_mask with n_q = 1).
    ``sinks`` [Hq] holds each query head's learned sink logit (or None).
    q [B, Hq, d]; caches [num_blocks, block_size, Hkv, d].
    Returns (O [len(heads), d], LSE [len(heads)]).
    """
    hq = q.shape[1]
    hkv = k_cache.shape[2]
    _check_heads(hq, hkv)
    n = int(_as_int(seq_lens)[b])
    if n <= 0:
        raise ValueError("a decode row needs at least one cached token")
    kind = MASK_SLIDING_WINDOW if window > 0 else MASK_CAUSAL
    allowed = allowed_mask(1, n, kind, window, n_sink=min(int(n_sink), n))
    row = _as_int(block_table)[b]
    k_seq = _gather_one(k_cache, row, n)
    v_seq = _gather_one(v_cache, row, n)
    qb = _as_f64(q[b])
    sk = None if sinks is None else _as_f64(sinks)
    outs, lses = [], []
    for h in heads:
        kvh = kv_head_of(h, hq, hkv)
        o, l = sdpa_rows(qb[h][None, :], k_seq[:, kvh], v_seq[:, kvh], allowed, scale,
                         sink=None if sk is None else sk[h])
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.asarray(lses)


def decode_paged_ref(q, k_cache, v_cache, block_table, seq_lens, scale: float, window: int = 0, n_sink: int = 0,
                     sinks=None):
    """Paged decode for every sequence and head: (O [B, Hq, d], LSE [B, Hq])."""
    b_, hq = q.shape[0], q.shape[1]
    out = np.empty((b_, hq, q.shape[2]), dtype=np.float64)
    lse = np.empty((b_, hq), dtype=np.float64)
    for bi in range(b_):
        o, l = decode_rows_ref(q, k_cache, v_cache, block_table, seq_lens, bi, range(hq), scale, window, n_sink,
                               sinks)
        out[bi] = o
        lse[bi] = l
    return out, lse


def prefill_paged_ref(q, k_cache, v_cache, block_table, seq_lens, mask_kind: int, window: int, scale: float,
                      seqs=None):
    """Prefix prefill over a paged context: the definition composed of two
    pinned pieces.

    Module 09: Efficient Attention, "Chunked Prefill": a prompt is processed in
    chunks, each chunk's queries attending to everything cached before it and to
    itself. Sequence b's keys are its seq_lens[b] cached tokens, gathered token
    by token through its block table (gather_paged_ref); its Nq query rows are
    the newest Nq positions (Modern Attention Mechanisms, section 4: after a
    prefix of length P, query row i has position P + i), which allowed_mask
    applies when n_q < n_k. q [B, Hq, Nq, d]. Returns (O [B, Hq, Nq, d],
    LSE [B, Hq, Nq]) for the sequences in `seqs` (all when None; others zero).
    """
    q = _as_f64(q)
    lens = _as_int(seq_lens)
    b_, hq, n_q, d = q.shape
    seqs = range(b_) if seqs is None else seqs
    out = np.zeros((b_, hq, n_q, d), dtype=np.float64)
    lse = np.zeros((b_, hq, n_q), dtype=np.float64)
    table = _as_int(block_table)
    for bi in seqs:
        n_k = int(lens[bi])
        kb = gather_paged_ref(k_cache, table[bi:bi + 1], lens[bi:bi + 1], n_k)
        vb = gather_paged_ref(v_cache, table[bi:bi + 1], lens[bi:bi + 1], n_k)
        o_b, l_b = prefill_ref(q[bi:bi + 1], kb, vb, mask_kind, window, scale)
        out[bi] = o_b[0]
        lse[bi] = l_b[0]
    return out, lse


def lse_merge_ref(o_parts, lse_parts):
    """Combine per-chunk partial results into the full softmax result.

    Inference attention post, "FlashDecoding": each key chunk yields its
    normalised partial output O_s and log-sum-exp lse_s; the combination uses
    the online softmax's rescaling: lse = log(sum_s exp(lse_s)) and
    O = sum_s exp(lse_s - lse) * O_s. An empty chunk has lse_s = -inf and
    weight 0. o_parts [S, d], lse_parts [S]. Returns (O [d], lse).
    """
    o_parts = _as_f64(o_parts)
    lse_parts = _as_f64(lse_parts)
    live = np.isfinite(lse_parts)
    if not live.any():
        raise ValueError("every chunk is empty")
    top = lse_parts[live].max()
    total = top + math.log(float(np.exp(lse_parts[live] - top).sum()))
    weights = np.where(live, np.exp(np.where(live, lse_parts, top) - total), 0.0)
    return (weights[:, None] * o_parts).sum(axis=0), total


def kv_cache_bytes(layers: int, hkv: int, d_head: int, bytes_per_elem: int, positions: int = 1) -> int:
    """K/V payload bytes: 2 * L * H_kv * n * d_h * b.

    Modern Attention Mechanisms, section 1 (b_KV = 2 L H_kv d_h b per token) and
    Module 09: Efficient Attention, "Intuition: The Memory Wall" (the same
    formula with the sequence length n).
    """
    return 2 * layers * hkv * positions * d_head * bytes_per_elem
