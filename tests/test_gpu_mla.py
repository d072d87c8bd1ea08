"""GPU parity of attn_mla_decode_paged (absorbed MLA decode over a paged
latent cache) against the fp64 oracle, through the C ABI."""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_softmax_attention_causal_b200 import mla_decode_paged, workloads
from parity import assert_parity

pytestmark = pytest.mark.gpu

SCALE = 1 / math.sqrt(128 + 64)  # DeepSeek-V2: head dim 128 plus the 64-wide positional key


def _poison_unreferenced(x):
    used = torch.zeros(x.cache.shape[:2], dtype=torch.bool)
    for b, n in enumerate(x.seq_lens.tolist()):
        t = torch.arange(n)
        used[x.block_table[b, t // x.block_size].long(), t % x.block_size] = True
    x.cache[~used] = torch.tensor(float("nan"), dtype=torch.bfloat16)
    return x


def _run(x, status=None, table=None):
    o, lse = mla_decode_paged(x.q.cuda(), x.cache.cuda(), (x.block_table if table is None else table).cuda(),
                              x.seq_lens.cuda(), x.max_seq_len, SCALE, status=status)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def _check(x, seqs=None, heads=None, poison=True, what=""):
    if poison:
        x = _poison_unreferenced(x)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = _run(x, status)
    assert int(status.item()) == 0
    H = x.q.shape[1]
    heads = list(range(H)) if heads is None else heads
    for b in (range(x.q.shape[0]) if seqs is None else seqs):
        o_ref, l_ref = oracle.mla_decode_rows_ref(x.q, x.cache, x.block_table, x.seq_lens, b, heads, 512, SCALE)
        assert_parity(o[b, heads], o_ref, lse[b, heads], l_ref, what=f"{what} seq {b}")
    return o, lse


@pytest.mark.parametrize("H", [128, 64, 16, 100, 32, 20, 96, 80, 8, 12, 72])
def test_mixed_lengths(H):
    # one token, a ragged tile, several tiles, and enough tokens for several splits
    x = workloads.mla_decode_inputs(4, H, 512, 64, seq_lens=[1, 130, 700, 9000], block_size=16, seed=H,
                                    extra_blocks=3)
    _check(x, what=f"H={H}")


@pytest.mark.parametrize("bs", [32, 64, 128])
def test_block_sizes(bs):
    x = workloads.mla_decode_inputs(3, 128, 512, 64, seq_lens=[17, 1000, 4097], block_size=bs, seed=bs)
    _check(x, what=f"bs={bs}")


@pytest.mark.parametrize("H", [64, 16])
def test_deterministic_and_permutation_invariant(H):
    x = workloads.mla_decode_inputs(2, H, 512, 64, seq_lens=[300, 2000], block_size=16, seed=5, extra_blocks=4)
    o1, l1 = _run(x)
    o2, l2 = _run(x)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    # the same cached rows behind another block permutation give the same bits
    perm = torch.randperm(x.cache.shape[0], generator=torch.Generator().manual_seed(9))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(perm.numel())
    cache2 = x.cache[perm]  # block p of cache2 holds block perm[p] of the original
    table2 = torch.where(x.block_table >= 0, inv[x.block_table.clamp(min=0).long()].int(), x.block_table)
    o3, l3 = mla_decode_paged(x.q.cuda(), cache2.cuda(), table2.cuda(), x.seq_lens.cuda(), x.max_seq_len, SCALE)
    assert torch.equal(o3.cpu(), o1) and torch.equal(l3.cpu(), l1)


@pytest.mark.parametrize("H", [128, 16])
def test_bad_entry_and_seq_len_are_flagged(H):
    x = workloads.mla_decode_inputs(3, H, 512, 64, seq_lens=[200, 200, 200], block_size=16, seed=6)
    x.block_table[1, 5] = 10 ** 6
    x.seq_lens[2] = 0
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = _run(x, status)
    assert int(status.item()) & 0x1
    assert torch.isnan(o[1].float()).all() and torch.isnan(o[2].float()).all()
    o_ref, l_ref = oracle.mla_decode_rows_ref(x.q, x.cache, x.block_table, x.seq_lens, 0, range(H), 512, SCALE)
    assert_parity(o[0], o_ref, lse[0], l_ref)


@pytest.mark.parametrize("name", sorted(workloads.MLA_DECODE_WORKLOADS))
def test_full_size_sampled(name):
    cfg = dict(workloads.MLA_DECODE_WORKLOADS[name])
    B, H, d_c, d_r = cfg.pop("B"), cfg.pop("H"), cfg.pop("d_latent"), cfg.pop("d_rope")
    d_head = cfg.pop("d_head")
    assert math.isclose(SCALE, 1 / math.sqrt(d_head + d_r))
    x = workloads.mla_decode_inputs(B, H, d_c, d_r, seed=0, **cfg)
    rng = np.random.default_rng(4)
    seqs = sorted(set([0, B - 1] + rng.integers(0, B, 2).tolist()))
    heads = sorted(set([0, H - 1] + rng.integers(0, H, 6).tolist()))
    _check(x, seqs=seqs, heads=heads, poison=False, what=name)
