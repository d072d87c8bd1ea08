"""Closed-form work and byte counts for the roofline figures.

Prefill FLOPs count only visible (query, key) pairs: 2*d for q.k plus 2*d for
p*v per pair, so 4 * d per pair per query head. Visible pairs per head:
full N^2, causal N(N+1)/2, window sum_i min(i+1, w).

Decode bytes count the K and V bytes a step must read from HBM:
sum_b seq_len_b * Hkv * d * 2 (K and V) * 2 (bf16). A windowed decode reads
only the visible tokens: the last W positions plus the first n_sink ones.
"""

from __future__ import annotations

MASK_IDS = {"full": 0, "causal": 1, "window": 2}


def visible_pairs(n: int, mask: str, window: int = 0) -> int:
    if mask == "full":
        return n * n
    if mask == "causal":
        return n * (n + 1) // 2
    if mask == "window":
        w = min(int(window), n)
        # rows 0..w-1 see i+1 keys, the remaining n-w rows see w keys
        return w * (w + 1) // 2 + (n - w) * w
    raise ValueError(mask)


def row_visible_keys(n: int, i: int, mask: str, window: int = 0) -> int:
    """Keys visible to query row i of an n-row square prefill."""
    if mask == "full":
        return n
    if mask == "causal":
        return i + 1
    if mask == "window":
        return min(i + 1, int(window))
    raise ValueError(mask)


def prefill_flops(B: int, Hq: int, N: int, d: int, mask: str, window: int = 0) -> int:
    return 4 * B * Hq * d * visible_pairs(N, mask, window)


def prefill_io_bytes(B: int, Hq: int, Hkv: int, N: int, d: int) -> int:
    """Compulsory HBM bytes of one prefill: Q, K, V read, O (bf16) and LSE (fp32) written."""
    return 2 * B * N * d * (2 * Hq + 2 * Hkv) + 4 * B * Hq * N


def decode_kv_bytes(seq_lens, Hkv: int, d: int) -> int:
    return sum(int(n) for n in seq_lens) * Hkv * d * 2 * 2


def decode_io_bytes(seq_lens, B: int, Hq: int, Hkv: int, d: int, block_size: int) -> int:
    """KV bytes plus q, o, lse, block-table and seq_len bytes."""
    tables = sum(-(-int(n) // block_size) for n in seq_lens) * 4 + 4 * B
    return decode_kv_bytes(seq_lens, Hkv, d) + B * Hq * d * 2 * 2 + B * Hq * 4 + tables


def prefix_visible_pairs(n_k: int, n_q: int, mask: str, window: int = 0) -> int:
    """Visible (query, key) pairs when the n_q query rows are the newest of n_k
    positions (row i at position n_k - n_q + i)."""
    p0 = n_k - n_q
    if mask == "full":
        return n_q * n_k
    # row i sees min(p0 + i + 1, w) keys (causal: w = infinity)
    w = n_k if mask == "causal" else min(int(window), n_k)
    first, last = p0 + 1, p0 + n_q  # keys seen by the first and last rows before the window cap
    if last <= w:
        return (first + last) * n_q // 2
    if first >= w:
        return w * n_q
    below = w - first  # rows whose count is still below the cap
    return (first + w - 1) * below // 2 + w * (n_q - below)


def prefill_paged_flops(seq_lens, n_q: int, Hq: int, d: int, mask: str, window: int = 0) -> int:
    return 4 * Hq * d * sum(prefix_visible_pairs(int(n), n_q, mask, window) for n in seq_lens)


def decode_visible_tokens(n: int, window: int = 0, n_sink: int = 0) -> int:
    """Tokens a decode query at position n - 1 sees: all n without a window;
    with window W the positions max(0, n - W) .. n - 1 plus the sink positions
    below that start (at most n_sink of them)."""
    n = int(n)
    if window <= 0:
        return n
    lo = max(0, n - int(window))
    return min(int(n_sink), lo) + (n - lo)


def decode_window_kv_bytes(seq_lens, Hkv: int, d: int, window: int = 0, n_sink: int = 0) -> int:
    return sum(decode_visible_tokens(n, window, n_sink) for n in seq_lens) * Hkv * d * 2 * 2


def mla_decode_bytes(seq_lens, d_latent: int, d_rope: int) -> int:
    """Latent-cache bytes an absorbed MLA decode step must read: one
    (d_c + d_R)-wide bf16 row per cached token, shared by every head."""
    return sum(int(n) for n in seq_lens) * (d_latent + d_rope) * 2


def mla_decode_flops(seq_lens, H: int, d_latent: int, d_rope: int) -> int:
    """2 (d_c + d_R) for the logit plus 2 d_c for the latent output, per head per token."""
    return sum(int(n) for n in seq_lens) * H * (2 * (d_latent + d_rope) + 2 * d_latent)


def prefill_backward_flops(B: int, Hq: int, N: int, d: int, mask: str, window: int = 0) -> int:
    """Five d-long products per visible (query, key) pair per query head (S
    recomputed, dP, dV, dK, dQ): 10 d FLOPs per pair, 2.5 x the forward."""
    return 10 * B * Hq * d * visible_pairs(N, mask, window)
