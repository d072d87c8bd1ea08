"""Seeded synthetic inputs for prefill and paged decode.

This module holds no attention arithmetic: it draws random numbers, rounds
them to bf16 and lays out a paged pool. Both the tests' fp64 oracle and the
CUDA path are fed from here, so they see identical inputs.

Recipe (all on the CPU, ``torch.Generator('cpu').manual_seed(seed)``):

* prefill: draw Q, K, V in that order as float32 standard normals, then round
  to bf16 (round-to-nearest-even). Shapes [B, Hq, N, d] and [B, Hkv, N, d].
* paged decode: draw ``seq_lens`` (uniform integers in [lo, hi]) unless given,
  then a permutation of the pool of sum(ceil(len / block_size)) physical
  blocks, handed out sequence-major to (sequence, logical block); table
  entries past a sequence's last block are -1. Then Q [B, Hq, d], the K pool
  and the V pool [num_blocks, block_size, Hkv, d], each float32 normal rounded
  to bf16. Large tensors are drawn in chunks of 2**24 elements, in order.
  With learned sinks, one float32 logit per query head is drawn last,
  uniform in [-1, 6) (the pages' examples use s = 0, 2, 5).

Paged layout: Module 09: Efficient Attention, "The Block Table" and "Code: A
Paged KV Cache from Scratch" (pool (num_blocks, block_size, num_kv_heads,
head_dim); a sequence of n tokens claims ceil(n / block_size) blocks; the
physical numbers come off a free list and are scattered).
"""

from __future__ import annotations

import dataclasses
import math

import torch

_CHUNK = 1 << 24


def _normal_bf16(shape, gen: torch.Generator) -> torch.Tensor:
    """float32 N(0, 1) drawn in fixed-size chunks, rounded to bf16."""
    out = torch.empty(shape, dtype=torch.bfloat16)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        flat[s:e] = torch.randn(e - s, generator=gen, dtype=torch.float32).to(torch.bfloat16)
    return out


def blocks_needed(n_tokens: int, block_size: int) -> int:
    """ceil(n / block_size): the blocks a sequence of n tokens claims."""
    return -(-int(n_tokens) // int(block_size))


@dataclasses.dataclass
class PrefillInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    seed: int


def prefill_inputs(B: int, Hq: int, Hkv: int, N: int, d: int, seed: int = 0) -> PrefillInputs:
    gen = torch.Generator("cpu").manual_seed(seed)
    q = _normal_bf16((B, Hq, N, d), gen)
    k = _normal_bf16((B, Hkv, N, d), gen)
    v = _normal_bf16((B, Hkv, N, d), gen)
    return PrefillInputs(q, k, v, seed)


@dataclasses.dataclass
class PagedDecodeInputs:
    q: torch.Tensor            # [B, Hq, d] bf16
    k_cache: torch.Tensor      # [num_blocks, block_size, Hkv, d] bf16
    v_cache: torch.Tensor      # [num_blocks, block_size, Hkv, d] bf16
    block_table: torch.Tensor  # [B, max_blocks] int32, -1 past the last block
    seq_lens: torch.Tensor     # [B] int32
    block_size: int
    max_seq_len: int
    seed: int
    sinks: torch.Tensor | None = None  # [Hq] float32 learned sink logits

    @property
    def num_blocks(self) -> int:
        return int(self.k_cache.shape[0])


def paged_layout(seq_lens, block_size: int, max_blocks: int, gen: torch.Generator,
                 extra_blocks: int = 0):
    """Scatter each sequence's logical blocks over a shuffled pool.

    Returns (block_table int32 [B, max_blocks], num_blocks). ``extra_blocks``
    adds pool blocks that no sequence references (they stay unreferenced).
    """
    lens = [int(x) for x in seq_lens]
    need = [blocks_needed(n, block_size) for n in lens]
    if max(need) > max_blocks:
        raise ValueError("max_blocks too small for the longest sequence")
    pool = sum(need) + int(extra_blocks)
    perm = torch.randperm(pool, generator=gen).to(torch.int32)
    table = torch.full((len(lens), max_blocks), -1, dtype=torch.int32)
    at = 0
    for b, nb in enumerate(need):
        table[b, :nb] = perm[at:at + nb]
        at += nb
    return table, pool


def paged_decode_inputs(B: int, Hq: int, Hkv: int, d: int, *, seq_lens=None, len_range=None,
                        block_size: int = 16, max_seq_len: int | None = None, seed: int = 0,
                        extra_blocks: int = 0, learned_sinks: bool = False) -> PagedDecodeInputs:
    gen = torch.Generator("cpu").manual_seed(seed)
    if seq_lens is None:
        lo, hi = len_range
        seq_lens = torch.randint(lo, hi + 1, (B,), generator=gen, dtype=torch.int64)
    seq_lens = torch.as_tensor(seq_lens, dtype=torch.int32).reshape(B)
    if max_seq_len is None:
        max_seq_len = int(len_range[1]) if len_range is not None else int(seq_lens.max())
    max_blocks = blocks_needed(max_seq_len, block_size)
    table, pool = paged_layout(seq_lens.tolist(), block_size, max_blocks, gen, extra_blocks)
    q = _normal_bf16((B, Hq, d), gen)
    k_cache = _normal_bf16((pool, block_size, Hkv, d), gen)
    v_cache = _normal_bf16((pool, block_size, Hkv, d), gen)
    sinks = None
    if learned_sinks:
        sinks = torch.rand(Hq, generator=gen, dtype=torch.float32) * 7.0 - 1.0
    return PagedDecodeInputs(q, k_cache, v_cache, table, seq_lens, block_size, int(max_seq_len), seed, sinks)


@dataclasses.dataclass
class PagedPrefillInputs:
    q: torch.Tensor            # [B, Hq, Nq, d] bf16: the newest Nq positions of each sequence
    k_cache: torch.Tensor      # [num_blocks, block_size, Hkv, d] bf16
    v_cache: torch.Tensor
    block_table: torch.Tensor  # [B, max_blocks] int32
    seq_lens: torch.Tensor     # [B] int32, each >= Nq
    block_size: int
    max_seq_len: int
    seed: int


def paged_prefill_inputs(B: int, Hq: int, Hkv: int, Nq: int, d: int, *, seq_lens=None, len_range=None,
                         block_size: int = 16, max_seq_len: int | None = None, seed: int = 0,
                         extra_blocks: int = 0) -> PagedPrefillInputs:
    """Same recipe as paged_decode_inputs, with Nq query rows per sequence."""
    gen = torch.Generator("cpu").manual_seed(seed)
    if seq_lens is None:
        lo, hi = len_range
        seq_lens = torch.randint(max(lo, Nq), hi + 1, (B,), generator=gen, dtype=torch.int64)
    seq_lens = torch.as_tensor(seq_lens, dtype=torch.int32).reshape(B)
    if max_seq_len is None:
        max_seq_len = int(len_range[1]) if len_range is not None else int(seq_lens.max())
    max_blocks = blocks_needed(max_seq_len, block_size)
    table, pool = paged_layout(seq_lens.tolist(), block_size, max_blocks, gen, extra_blocks)
    q = _normal_bf16((B, Hq, Nq, d), gen)
    k_cache = _normal_bf16((pool, block_size, Hkv, d), gen)
    v_cache = _normal_bf16((pool, block_size, Hkv, d), gen)
    return PagedPrefillInputs(q, k_cache, v_cache, table, seq_lens, block_size, int(max_seq_len), seed)


@dataclasses.dataclass
class MlaDecodeInputs:
    q: torch.Tensor            # [B, H, d_c + d_R] bf16: absorbed content query, then positional query
    cache: torch.Tensor        # [num_blocks, block_size, d_c + d_R] bf16: latent, then positional key
    block_table: torch.Tensor  # [B, max_blocks] int32
    seq_lens: torch.Tensor     # [B] int32
    d_latent: int
    block_size: int
    max_seq_len: int
    seed: int


def mla_decode_inputs(B: int, H: int, d_latent: int, d_rope: int, *, seq_lens=None, len_range=None,
                      block_size: int = 16, max_seq_len: int | None = None, seed: int = 0,
                      extra_blocks: int = 0) -> MlaDecodeInputs:
    """Same recipe as paged_decode_inputs with one latent row per token: draw
    seq_lens, lay out the pool, then Q and the cache as bf16-rounded normals."""
    gen = torch.Generator("cpu").manual_seed(seed)
    if seq_lens is None:
        lo, hi = len_range
        seq_lens = torch.randint(lo, hi + 1, (B,), generator=gen, dtype=torch.int64)
    seq_lens = torch.as_tensor(seq_lens, dtype=torch.int32).reshape(B)
    if max_seq_len is None:
        max_seq_len = int(len_range[1]) if len_range is not None else int(seq_lens.max())
    table, pool = paged_layout(seq_lens.tolist(), block_size, blocks_needed(max_seq_len, block_size), gen,
                               extra_blocks)
    q = _normal_bf16((B, H, d_latent + d_rope), gen)
    cache = _normal_bf16((pool, block_size, d_latent + d_rope), gen)
    return MlaDecodeInputs(q, cache, table, seq_lens, d_latent, block_size, int(max_seq_len), seed)


# Named workloads. Sizes follow the pages' shapes: Llama-style GQA-8
# ("USAAIO Lesson 90", GQA part), 131,072-token contexts ("Modern Attention
# Mechanisms", section 1) and 16-token blocks ("Module 09", "The Block Table").
PREFILL_WORKLOADS = {
    "tiny_causal_gqa": dict(B=1, Hq=4, Hkv=2, N=128, d=64, mask="causal", window=0),
    "llama3_8b_causal_gqa": dict(B=4, Hq=32, Hkv=8, N=4096, d=128, mask="causal", window=0),
    "long_causal_n32768": dict(B=1, Hq=32, Hkv=8, N=32768, d=128, mask="causal", window=0),
    "long_window4096_n32768": dict(B=1, Hq=32, Hkv=8, N=32768, d=128, mask="window", window=4096),
    "gqa_dial_prefill_mha": dict(B=2, Hq=32, Hkv=32, N=8192, d=128, mask="causal", window=0),
    "gqa_dial_prefill_gqa8": dict(B=2, Hq=32, Hkv=8, N=8192, d=128, mask="causal", window=0),
    "gqa_dial_prefill_mqa": dict(B=2, Hq=32, Hkv=1, N=8192, d=128, mask="causal", window=0),
}

# Chunked prefill: 512 new tokens per sequence on top of a paged context.
PAGED_PREFILL_WORKLOADS = {
    "chunked_prefill_b4_q512": dict(B=4, Hq=32, Hkv=8, Nq=512, d=128, len_range=(4096, 16384), block_size=16,
                                    mask="causal", window=0),
}

DECODE_WORKLOADS = {
    "paged_decode_b64": dict(B=64, Hq=32, Hkv=8, d=128, len_range=(1024, 32768), block_size=16),
    "gqa_dial_decode_mha": dict(B=1, Hq=32, Hkv=32, d=128, seq_lens=[131072], block_size=16),
    "gqa_dial_decode_gqa8": dict(B=1, Hq=32, Hkv=8, d=128, seq_lens=[131072], block_size=16),
    "gqa_dial_decode_mqa": dict(B=1, Hq=32, Hkv=1, d=128, seq_lens=[131072], block_size=16),
}

# Windowed decode with sinks. gpt-oss-120b shapes ("Modern Attention
# Mechanisms", the gpt-oss walk-through: 64 query heads over 8 K/V heads,
# head_dim 64, window 128 on the local layers, full causal on the others, one
# learned sink logit per head) and a StreamingLLM-style cache (window 4096, as
# in Mistral-7B-v0.1, plus the first 4 positions kept as sinks).
WINDOW_DECODE_WORKLOADS = {
    "gptoss_window128_sinks_b64": dict(B=64, Hq=64, Hkv=8, d=64, len_range=(1024, 32768), block_size=16,
                                       window=128, n_sink=0, learned_sinks=True),
    "gptoss_full_sinks_b64": dict(B=64, Hq=64, Hkv=8, d=64, len_range=(1024, 32768), block_size=16,
                                  window=0, n_sink=0, learned_sinks=True),
    "streaming_window4096_nsink4_b64": dict(B=64, Hq=32, Hkv=8, d=128, len_range=(8192, 32768), block_size=16,
                                            window=4096, n_sink=4, learned_sinks=False),
}


# Absorbed MLA decode with DeepSeek-V2's shapes ("Module 09", MLA section: a
# 512-wide latent and a 64-wide positional key per token, 128 heads of head
# dim 128, so the logit scale is 1 / sqrt(128 + 64)); the second keeps 16 of
# the 128 heads, as one GPU holds when the heads are split eight ways.
MLA_DECODE_WORKLOADS = {
    "deepseek_v2_mla_b64": dict(B=64, H=128, d_latent=512, d_rope=64, d_head=128, len_range=(1024, 32768),
                                block_size=16),
    "deepseek_v2_mla_h16_b64": dict(B=64, H=16, d_latent=512, d_rope=64, d_head=128, len_range=(1024, 32768),
                                    block_size=16),
}


def default_scale(d: int) -> float:
    """1 / sqrt(d): the SDPA scale of "Modern Attention Mechanisms", section 4."""
    return 1.0 / math.sqrt(d)
