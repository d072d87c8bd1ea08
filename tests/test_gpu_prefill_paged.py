"""GPU parity of attn_prefill_paged (prefix / chunked prefill over a paged
context) against the fp64 oracle, through the C ABI."""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_softmax_attention_causal_b200 import prefill, prefill_paged, workloads
from parity import assert_parity

pytestmark = pytest.mark.gpu

MASK_IDS = {"full": oracle.MASK_FULL, "causal": oracle.MASK_CAUSAL, "window": oracle.MASK_SLIDING_WINDOW}


def _poison_unreferenced(x):
    """NaN into every pool slot no sequence references, including the slots
    past seq_len inside each sequence's last block."""
    used = torch.zeros(x.k_cache.shape[:2], dtype=torch.bool)
    for b, n in enumerate(x.seq_lens.tolist()):
        t = torch.arange(n)
        used[x.block_table[b, t // x.block_size].long(), t % x.block_size] = True
    nan = torch.tensor(float("nan"), dtype=torch.bfloat16)
    x.k_cache[~used] = nan
    x.v_cache[~used] = nan
    return x


def _run(x, mask, window=0, status=None):
    d = x.q.shape[-1]
    o, lse = prefill_paged(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.block_table.cuda(),
                           x.seq_lens.cuda(), x.max_seq_len, mask=mask, window=window, scale=1 / math.sqrt(d),
                           status=status)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def _check(x, mask, window=0, seqs=None, what=""):
    x = _poison_unreferenced(x)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = _run(x, mask, window, status)
    assert int(status.item()) == 0
    d = x.q.shape[-1]
    seqs = range(x.q.shape[0]) if seqs is None else seqs
    o_ref, l_ref = oracle.prefill_paged_ref(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens, MASK_IDS[mask],
                                            window, 1 / math.sqrt(d), seqs=seqs)
    for b in seqs:
        assert_parity(o[b], o_ref[b], lse[b], l_ref[b], what=f"{what} seq {b}")


@pytest.mark.parametrize("bs", [16, 32, 64, 128])
@pytest.mark.parametrize("mask,window", [("causal", 0), ("full", 0), ("window", 100)])
def test_mixed_contexts(bs, mask, window):
    # Nq = 77: one ragged query tile; contexts from Nq (no prefix) to several key tiles,
    # ending mid-block so the partly filled last block is exercised
    x = workloads.paged_prefill_inputs(3, 8, 2, 77, 128, seq_lens=[77, 300, 611], block_size=bs, seed=bs,
                                       extra_blocks=3)
    _check(x, mask, window, what=f"bs={bs} {mask}")


@pytest.mark.parametrize("Nq", [1, 128, 300])
def test_query_chunk_sizes_d64(Nq):
    x = workloads.paged_prefill_inputs(2, 4, 1, Nq, 64, seq_lens=[Nq + 5, Nq + 700], block_size=16, seed=Nq)
    _check(x, "causal", what=f"Nq={Nq}")


def test_square_case_equals_contiguous_prefill_bitwise():
    """seq_len == Nq: the same attention as attn_prefill on the gathered cache;
    the paged loads assemble the same shared-memory tiles, so bit-identical."""
    B, Hq, Hkv, N, d = 2, 8, 2, 333, 128
    x = workloads.paged_prefill_inputs(B, Hq, Hkv, N, d, seq_lens=[N, N], block_size=16, seed=3)
    o_p, l_p = _run(x, "causal")
    k = torch.from_numpy(oracle.gather_paged_ref(x.k_cache, x.block_table, x.seq_lens, N)).to(torch.bfloat16)
    v = torch.from_numpy(oracle.gather_paged_ref(x.v_cache, x.block_table, x.seq_lens, N)).to(torch.bfloat16)
    o_c, l_c = prefill(x.q.cuda(), k.cuda(), v.cuda(), mask="causal")
    assert torch.equal(o_p, o_c.cpu()) and torch.equal(l_p, l_c.cpu())


def test_chunks_reproduce_the_one_shot_prefill():
    """Module 09, "Chunked Prefill": chunking is scheduling, not arithmetic. A
    700-token prompt prefilled in three chunks against its growing paged cache
    matches the one-shot causal prefill row for row."""
    Hq, Hkv, N, d, bs = 8, 2, 700, 128, 16
    xp = workloads.prefill_inputs(1, Hq, Hkv, N, d, 11)
    o_full, l_full = prefill(xp.q.cuda(), xp.k.cuda(), xp.v.cuda(), mask="causal")
    nblk = -(-N // bs)
    perm = torch.randperm(nblk, generator=torch.Generator().manual_seed(2))
    kc = torch.zeros((nblk, bs, Hkv, d), dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    for lb in range(nblk):
        n = min(bs, N - lb * bs)
        kc[perm[lb], :n] = xp.k[0, :, lb * bs: lb * bs + n].transpose(0, 1)
        vc[perm[lb], :n] = xp.v[0, :, lb * bs: lb * bs + n].transpose(0, 1)
    table = perm.int()[None].cuda()
    for a, b in [(0, 256), (256, 500), (500, 700)]:
        o_c, l_c = prefill_paged(xp.q[:, :, a:b].contiguous().cuda(), kc.cuda(), vc.cuda(), table,
                                 torch.tensor([b], dtype=torch.int32, device="cuda"), N, mask="causal")
        assert_parity(o_c[0].cpu(), o_full[0, :, a:b].cpu(), l_c[0].cpu(), l_full[0, :, a:b].cpu(),
                      what=f"chunk {a}:{b}")


def test_bad_seq_len_and_bad_entry_are_flagged():
    x = workloads.paged_prefill_inputs(3, 4, 2, 64, 128, seq_lens=[64, 200, 300], block_size=16, seed=5)
    x.seq_lens[0] = 10           # shorter than the query chunk
    x.block_table[2, 3] = 10 ** 6  # a block the third sequence needs
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = _run(x, "causal", status=status)
    assert int(status.item()) & 0x1
    assert torch.isnan(o[0].float()).all() and torch.isnan(lse[0]).all()
    assert torch.isnan(o[2].float()).all()
    o_ref, l_ref = oracle.prefill_paged_ref(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens,
                                            oracle.MASK_CAUSAL, 0, 1 / math.sqrt(128), seqs=[1])
    assert_parity(o[1], o_ref[1], lse[1], l_ref[1])


def test_full_size_sampled():
    cfg = dict(workloads.PAGED_PREFILL_WORKLOADS["chunked_prefill_b4_q512"])
    mask, window = cfg.pop("mask"), cfg.pop("window")
    B, Hq, Hkv, Nq, d = (cfg.pop(k) for k in ("B", "Hq", "Hkv", "Nq", "d"))
    x = workloads.paged_prefill_inputs(B, Hq, Hkv, Nq, d, seed=0, **cfg)
    o, lse = _run(x, mask, window)
    assert torch.isfinite(o.float()).all()
    rng = np.random.default_rng(3)
    for b in (0, B - 1):
        for h in (0, Hq - 1, int(rng.integers(0, Hq))):
            n_k = int(x.seq_lens[b])
            rows = sorted(set([0, 1, 127, 128, 255, 256, Nq - 1] + rng.integers(0, Nq, 6).tolist()))
            kb = oracle.gather_paged_ref(x.k_cache, x.block_table[b:b + 1], x.seq_lens[b:b + 1], n_k)
            vb = oracle.gather_paged_ref(x.v_cache, x.block_table[b:b + 1], x.seq_lens[b:b + 1], n_k)
            q_b = x.q[b:b + 1].double().numpy()
            kvh = h // (Hq // Hkv)
            allowed = oracle.allowed_mask(Nq, n_k, MASK_IDS[mask], window, rows=rows)
            from oracle.attention import sdpa_rows
            o_ref, l_ref = sdpa_rows(q_b[0, h][rows], kb[0, kvh], vb[0, kvh], allowed, 1 / math.sqrt(d))
            assert_parity(o[b, h, rows], o_ref, lse[b, h, rows], l_ref, what=f"b={b} h={h}")
