"""GPU parity of attn_decode_paged and attn_paged_gather against the fp64
oracle (through the C ABI)."""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_softmax_attention_causal_b200 import decode_paged, paged_gather, prefill, workloads
from parity import assert_parity

pytestmark = pytest.mark.gpu


def _to_cuda(x):
    return (x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.block_table.cuda(), x.seq_lens.cuda())


def _poison_unreferenced(x):
    """NaN into every pool slot no sequence references (whole unreferenced
    blocks and the slots past seq_len in each last block)."""
    used = torch.zeros(x.k_cache.shape[:2], dtype=torch.bool)
    for b, n in enumerate(x.seq_lens.tolist()):
        for t in range(n):
            used[int(x.block_table[b, t // x.block_size]), t % x.block_size] = True
    nan = torch.tensor(float("nan"), dtype=torch.bfloat16)
    x.k_cache[~used] = nan
    x.v_cache[~used] = nan
    return x


def _check(x, heads=None, seqs=None, poison=True, what=""):
    if poison:
        x = _poison_unreferenced(x)
    q, kc, vc, bt, sl = _to_cuda(x)
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = decode_paged(q, kc, vc, bt, sl, x.max_seq_len, scale=scale, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    o, lse = o.cpu(), lse.cpu()
    Hq = q.shape[1]
    seqs = range(q.shape[0]) if seqs is None else seqs
    heads = range(Hq) if heads is None else heads
    for b in seqs:
        o_ref, l_ref = oracle.decode_rows_ref(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens, b, heads, scale)
        assert_parity(o[b, list(heads)], o_ref, lse[b, list(heads)], l_ref, what=f"{what} seq {b}")
    return o, lse


@pytest.mark.parametrize("d", [64, 128])
def test_small_mixed_lengths(d):
    x = workloads.paged_decode_inputs(4, 8, 2, d, seq_lens=[1, 17, 300, 4096], block_size=16, seed=1,
                                      extra_blocks=5)
    _check(x, what=f"d={d}")


@pytest.mark.parametrize("hq,hkv", [(32, 32), (32, 1), (20, 1), (4, 4), (48, 2)])
def test_head_groups(hq, hkv):
    x = workloads.paged_decode_inputs(2, hq, hkv, 128, seq_lens=[33, 2500], block_size=16, seed=2,
                                      extra_blocks=3)
    _check(x, what=f"{hq}/{hkv}")


# More than 16 query heads per K/V head: CTAs of 32 heads whose warp pairs
# share one ring (20 and 24 heads leave padding rows; 64 heads take two CTAs
# per split), on both head sizes, both split-plan branches (a batch of 160
# sequences fills the GPU with one CTA per sequence and split) and one long
# sequence whose splits go to the merge kernel.
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(32, 1), (64, 2), (24, 1), (64, 1)])
def test_paired_head_groups(d, hq, hkv):
    x = workloads.paged_decode_inputs(3, hq, hkv, d, seq_lens=[1, 75, 9000], block_size=16, seed=31,
                                      extra_blocks=3)
    _check(x, what=f"paired {hq}/{hkv} d={d}")


def test_paired_batch_fills_gpu():
    lens = [1 + (37 * i) % 2100 for i in range(160)]
    x = workloads.paged_decode_inputs(160, 32, 1, 128, seq_lens=lens, block_size=16, seed=32)
    _check(x, seqs=[0, 1, 57, 158, 159], poison=False, what="paired batch")


def test_paired_single_sequence_merge_kernel():
    x = workloads.paged_decode_inputs(1, 32, 1, 128, seq_lens=[65536 + 13], block_size=16, seed=33)
    _check(x, poison=False, what="paired merge kernel")


@pytest.mark.parametrize("bs", [32, 64])
def test_block_sizes(bs):
    x = workloads.paged_decode_inputs(3, 8, 1, 128, seq_lens=[5, 1000, 777], block_size=bs, seed=3,
                                      extra_blocks=2)
    _check(x, what=f"bs={bs}")


def test_long_single_sequence_many_splits():
    x = workloads.paged_decode_inputs(1, 8, 2, 128, seq_lens=[20000], block_size=16, seed=4)
    _check(x, poison=False)


def test_permutation_invariance():
    x = workloads.paged_decode_inputs(2, 8, 2, 128, seq_lens=[900, 64], block_size=16, seed=5)
    q, kc, vc, bt, sl = _to_cuda(x)
    o1, l1 = decode_paged(q, kc, vc, bt, sl, x.max_seq_len)
    # move every block to a new physical slot and rewrite the table
    perm = torch.randperm(kc.shape[0], generator=torch.Generator().manual_seed(9)).cuda()
    kc2 = torch.empty_like(kc)
    vc2 = torch.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    bt2 = torch.where(bt >= 0, perm[bt.clamp(min=0).long()].int(), bt)
    o2, l2 = decode_paged(q, kc2, vc2, bt2, sl, x.max_seq_len)
    # a one-wave plan hands out its work at run time: equal up to the rounding
    # of the summation order
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-3
    assert (l1 - l2).abs().max().item() <= 1e-4


def test_gather_bit_exact():
    x = workloads.paged_decode_inputs(3, 4, 2, 128, seq_lens=[1, 40, 333], block_size=16, seed=6, extra_blocks=4)
    out = paged_gather(x.k_cache.cuda(), x.block_table.cuda(), x.seq_lens.cuda(), x.max_seq_len).cpu()
    ref = oracle.gather_paged_ref(x.k_cache, x.block_table, x.seq_lens, x.max_seq_len)
    assert torch.equal(out.double(), torch.from_numpy(ref))


def test_gather_bit_exact_decode_workload_shape():
    cfg = workloads.DECODE_WORKLOADS["paged_decode_b64"]
    x = workloads.paged_decode_inputs(8, 4, 8, 128, len_range=(1, 4096), block_size=16, seed=7)
    out = paged_gather(x.v_cache.cuda(), x.block_table.cuda(), x.seq_lens.cuda(), x.max_seq_len).cpu()
    ref = oracle.gather_paged_ref(x.v_cache, x.block_table, x.seq_lens, x.max_seq_len)
    assert torch.equal(out.double(), torch.from_numpy(ref))
    assert cfg["block_size"] == 16


def test_invalid_block_table_entry_is_flagged_not_read():
    x = workloads.paged_decode_inputs(3, 8, 2, 128, seq_lens=[100, 200, 50], block_size=16, seed=8)
    x.block_table[1, 3] = x.k_cache.shape[0] + 1000  # referenced (200 tokens use 13 blocks)
    q, kc, vc, bt, sl = _to_cuda(x)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = decode_paged(q, kc, vc, bt, sl, x.max_seq_len, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & 0x1
    assert torch.isnan(o[1].float()).all() and torch.isnan(lse[1]).all()
    scale = 1 / math.sqrt(128)
    for b in (0, 2):
        o_ref, l_ref = oracle.decode_rows_ref(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens, b, range(8),
                                              scale)
        assert_parity(o[b].cpu(), o_ref, lse[b].cpu(), l_ref)
    # the gather flags the same entry and NaNs that token's rows
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    g = paged_gather(kc, bt, sl, x.max_seq_len, status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) & 0x1
    assert torch.isnan(g[1, :, 48:64].float()).all() and not torch.isnan(g[0].float()).any()


@pytest.mark.parametrize("bad_len", [0, -3, 10 ** 6])
def test_invalid_seq_len_is_flagged(bad_len):
    x = workloads.paged_decode_inputs(2, 4, 2, 128, seq_lens=[64, 64], block_size=16, seed=9)
    x.seq_lens[0] = bad_len
    q, kc, vc, bt, sl = _to_cuda(x)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = decode_paged(q, kc, vc, bt, sl, 64, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & 0x1
    assert torch.isnan(o[0].float()).all()
    assert torch.isfinite(o[1].float()).all()


def test_decode_equals_prefill_last_row():
    """Cached decoding equals the full forward pass ("Module 09", the GQA cache
    demonstration): decode at context t == row t-1 of causal prefill."""
    B, Hq, Hkv, N, d = 1, 8, 2, 777, 128
    xp = workloads.prefill_inputs(B, Hq, Hkv, N, d, 10)
    q, k, v = (t.cuda() for t in (xp.q, xp.k, xp.v))
    o_pf, lse_pf = prefill(q, k, v, mask="causal")
    bs = 16
    nblk = -(-N // bs)
    perm = torch.randperm(nblk, generator=torch.Generator().manual_seed(3))
    kc = torch.zeros((nblk, bs, Hkv, d), dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    kt = xp.k[0].transpose(0, 1)  # [N, Hkv, d]
    vt = xp.v[0].transpose(0, 1)
    for lb in range(nblk):
        n = min(bs, N - lb * bs)
        kc[perm[lb], :n] = kt[lb * bs: lb * bs + n]
        vc[perm[lb], :n] = vt[lb * bs: lb * bs + n]
    table = perm.int()[None, :].cuda()
    for t in (1, 16, 17, 500, N):
        o_d, l_d = decode_paged(q[:, :, t - 1].contiguous(), kc.cuda(), vc.cuda(), table,
                                torch.tensor([t], dtype=torch.int32, device="cuda"), N)
        assert_parity(o_d[0].cpu(), o_pf[0, :, t - 1].cpu(), l_d[0].cpu(), lse_pf[0, :, t - 1].cpu(),
                      what=f"t={t}")


# --------------------------------------------------------------------------
# full-size workloads, sampled sequences and heads
# --------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["paged_decode_b64", "gqa_dial_decode_mha", "gqa_dial_decode_gqa8",
                                  "gqa_dial_decode_mqa"])
def test_full_size_sampled(name):
    cfg = dict(workloads.DECODE_WORKLOADS[name])
    B, Hq, Hkv, d = cfg.pop("B"), cfg.pop("Hq"), cfg.pop("Hkv"), cfg.pop("d")
    x = workloads.paged_decode_inputs(B, Hq, Hkv, d, seed=0, **cfg)
    rng = np.random.default_rng(1)
    seqs = sorted(set([0, B - 1] + rng.integers(0, B, 3).tolist()))
    heads = sorted(set([0, Hq - 1] + rng.integers(0, Hq, 4).tolist()))
    _check(x, heads=heads, seqs=seqs, poison=False, what=name)


# --------------------------------------------------------------------------
# the in-launch split merge: ticket counters in a reused, never-cleared
# workspace; the merge kernel; a result that does not depend on which CTA
# finished last
# --------------------------------------------------------------------------
def test_fixed_split_plan_is_bit_reproducible():
    """A batch that fills the GPU takes 2048-token splits fixed by the plan:
    repeated calls are bit-identical."""
    lens = [1 + (911 * i) % 9000 for i in range(80)]
    x = workloads.paged_decode_inputs(80, 8, 4, 128, seq_lens=lens, block_size=16, seed=25)
    t = _to_cuda(x)
    o1, l1 = decode_paged(*t, x.max_seq_len)
    o2, l2 = decode_paged(*t, x.max_seq_len)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_run_time_grains_cover_every_token():
    """One-wave plans hand out grains of two sub-blocks at run time: short and
    long sequences of one batch (most CTAs of the short ones receive no
    grain), the last grain partial, lengths around grain edges."""
    x = workloads.paged_decode_inputs(4, 16, 4, 128, seq_lens=[1, 31, 33, 50001], block_size=16, seed=26,
                                      extra_blocks=2)
    _check(x, what="run-time grains")


def test_merge_kernel_single_sequence():
    """16 query heads on one K/V head: more splits than one CTA stages at once
    (192 / 16 rows), so the split grid leaves its partials to the merge kernel
    (launched as a programmatic dependent of the one-wave split grid, with
    run-time grains in the split kernel)."""
    x = workloads.paged_decode_inputs(1, 16, 1, 128, seq_lens=[40000], block_size=16, seed=21)
    _check(x, poison=False, what="merge kernel")


def test_workspace_reused_with_garbage_and_other_plans():
    """The workspace is never cleared by the caller: random bytes, then the
    leftovers of a call with another plan, must not change any result.
    Repeated calls of a plan with fixed splits (here the 32-head CTAs) are
    bit-identical; a one-wave plan of 16-head CTAs hands out its work at run
    time, so its repeats agree to the rounding of a different summation
    order (both match the oracle)."""
    xa = workloads.paged_decode_inputs(2, 16, 4, 128, seq_lens=[30000, 7000], block_size=16, seed=22)
    xb = workloads.paged_decode_inputs(3, 32, 1, 64, seq_lens=[9000, 100, 25000], block_size=16, seed=23)
    from exact_softmax_attention_causal_b200 import decode_workspace_bytes

    nbytes = max(decode_workspace_bytes(2, 16, 4, 128, xa.max_seq_len, 16),
                 decode_workspace_bytes(3, 32, 1, 64, xb.max_seq_len, 16))
    gen = torch.Generator("cpu").manual_seed(24)
    ws = torch.randint(0, 256, (nbytes,), generator=gen, dtype=torch.uint8).cuda()
    a, b = _to_cuda(xa), _to_cuda(xb)
    outs = []
    for x, t in ((xa, a), (xb, b), (xa, a), (xb, b)):
        o, lse = decode_paged(*t, x.max_seq_len, workspace=ws[: decode_workspace_bytes(
            t[0].shape[0], t[0].shape[1], t[1].shape[2], t[0].shape[2], x.max_seq_len, 16)])
        outs.append((o.clone(), lse.clone()))
    torch.cuda.synchronize()
    assert (outs[0][0].float() - outs[2][0].float()).abs().max().item() <= 2e-3
    assert (outs[0][1] - outs[2][1]).abs().max().item() <= 1e-4
    assert torch.equal(outs[1][0], outs[3][0]) and torch.equal(outs[1][1], outs[3][1])
    for x, (o, lse) in ((xa, outs[0]), (xb, outs[1]), (xa, outs[2]), (xb, outs[3])):
        d = x.q.shape[-1]
        for bi in range(x.q.shape[0]):
            heads = [0, x.q.shape[1] - 1]
            o_ref, l_ref = oracle.decode_rows_ref(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens, bi, heads,
                                                  1.0 / math.sqrt(d))
            assert_parity(o[bi, heads].cpu(), o_ref, lse[bi, heads].cpu(), l_ref, what=f"reused workspace b={bi}")
