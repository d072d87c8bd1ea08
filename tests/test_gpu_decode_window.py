"""GPU parity of attn_decode_paged_window (sliding window, StreamingLLM sink
positions, learned per-head sink logits) against the fp64 oracle, through
the C ABI."""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_softmax_attention_causal_b200 import accounting, decode_paged, decode_paged_window, workloads
from parity import assert_parity

pytestmark = pytest.mark.gpu


def _visible_tokens(n, window, n_sink):
    if window <= 0:
        return set(range(n))
    return set(range(max(0, n - window), n)) | set(range(min(n_sink, n)))


def _poison_invisible(x, window, n_sink):
    """NaN into every pool slot that holds no visible token of any sequence,
    so a kernel that reads or multiplies a hidden slot shows it."""
    keep = torch.zeros(x.k_cache.shape[:2], dtype=torch.bool)
    for b, n in enumerate(x.seq_lens.tolist()):
        for t in _visible_tokens(n, window, n_sink):
            keep[int(x.block_table[b, t // x.block_size]), t % x.block_size] = True
    nan = torch.tensor(float("nan"), dtype=torch.bfloat16)
    k, v = x.k_cache.clone(), x.v_cache.clone()
    k[~keep] = nan
    v[~keep] = nan
    return k, v


def _run(x, window, n_sink, sinks, k_cache=None, v_cache=None, table=None, status=None):
    d = x.q.shape[-1]
    kc = (x.k_cache if k_cache is None else k_cache).cuda()
    vc = (x.v_cache if v_cache is None else v_cache).cuda()
    bt = (x.block_table if table is None else table).cuda()
    o, lse = decode_paged_window(x.q.cuda(), kc, vc, bt, x.seq_lens.cuda(), x.max_seq_len, window=window,
                                 n_sink=n_sink, sinks=None if sinks is None else sinks.cuda(),
                                 scale=1 / math.sqrt(d), status=status)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def _check(x, window, n_sink, sinks, seqs=None, heads=None, poison=True, what=""):
    kc, vc = _poison_invisible(x, window, n_sink) if poison else (None, None)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = _run(x, window, n_sink, sinks, kc, vc, status=status)
    assert int(status.item()) == 0
    d, Hq = x.q.shape[-1], x.q.shape[1]
    seqs = range(x.q.shape[0]) if seqs is None else seqs
    heads = list(range(Hq)) if heads is None else heads
    for b in seqs:
        o_ref, l_ref = oracle.decode_rows_ref(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens, b, heads,
                                              1 / math.sqrt(d), window, n_sink, sinks)
        assert_parity(o[b, heads], o_ref, lse[b, heads], l_ref, what=f"{what} seq {b}")
    return o, lse


CASES = [  # (window, n_sink, learned sinks)
    (1, 0, False), (5, 0, True), (16, 0, False), (17, 1, False), (100, 4, True), (128, 0, True),
    (128, 33, True), (1000, 16, False), (0, 0, True),
]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("window,n_sink,with_sinks", CASES)
def test_mixed_lengths(d, window, n_sink, with_sinks):
    # lengths below, at and above the window; one long enough for several splits
    x = workloads.paged_decode_inputs(5, 8, 2, d, seq_lens=[1, 17, 130, 1200, 5000], block_size=16,
                                      seed=window * 7 + n_sink, extra_blocks=3, learned_sinks=with_sinks)
    _check(x, window, n_sink, x.sinks, what=f"d={d} w={window} s={n_sink}")


@pytest.mark.parametrize("bs", [32, 64, 128])
def test_block_sizes(bs):
    x = workloads.paged_decode_inputs(3, 8, 1, 128, seq_lens=[40, 700, 3001], block_size=bs, seed=bs,
                                      learned_sinks=True)
    _check(x, 100, 4, x.sinks, what=f"bs={bs}")


@pytest.mark.parametrize("window,n_sink,with_sinks", [(128, 0, True), (100, 4, True), (1000, 16, False)])
def test_paired_heads(window, n_sink, with_sinks):
    """32 query heads on one K/V head: the warp-pair CTAs with a window."""
    x = workloads.paged_decode_inputs(4, 32, 1, 128, seq_lens=[1, 130, 1200, 7000], block_size=16, seed=17,
                                      learned_sinks=with_sinks)
    _check(x, window, n_sink, x.sinks if with_sinks else None, what=f"paired w={window}")


def test_gptoss_shape_window128_with_sinks():
    """gpt-oss local layer: 64 query heads over 8 K/V heads, head_dim 64,
    window 128, one learned sink per head."""
    x = workloads.paged_decode_inputs(6, 64, 8, 64, len_range=(1, 3000), block_size=16, seed=11,
                                      learned_sinks=True)
    _check(x, 128, 0, x.sinks, what="gpt-oss")


def test_window_covering_everything_equals_plain_decode():
    """A window at least as long as every sequence hides nothing: the same
    kernel as the plain decode runs (this one-wave plan hands out its work at
    run time, so the results agree up to the rounding of the summation order)."""
    x = workloads.paged_decode_inputs(3, 8, 2, 128, seq_lens=[7, 300, 2000], block_size=16, seed=12)
    q, kc, vc, bt, sl = (t.cuda() for t in (x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens))
    o_ref, l_ref = decode_paged(q, kc, vc, bt, sl, x.max_seq_len)
    for window, n_sink in ((0, 0), (x.max_seq_len, 0), (x.max_seq_len + 5, 3)):
        o, lse = decode_paged_window(q, kc, vc, bt, sl, x.max_seq_len, window=window, n_sink=n_sink)
        assert (o.float() - o_ref.float()).abs().max().item() <= 2e-3, (window, n_sink)
        assert (lse - l_ref).abs().max().item() <= 1e-4, (window, n_sink)


def test_evicted_middle_blocks_are_never_read():
    """A rolling cache frees the blocks between the sink positions and the
    window: their table entries become -1 and their slots garbage. The result
    must not change."""
    window, n_sink, bs = 64, 4, 16
    x = workloads.paged_decode_inputs(3, 8, 2, 128, seq_lens=[50, 900, 4000], block_size=bs, seed=13,
                                      learned_sinks=True)
    o_ref, l_ref = _run(x, window, n_sink, x.sinks)
    table = x.block_table.clone()
    for b, n in enumerate(x.seq_lens.tolist()):
        vis = _visible_tokens(n, window, n_sink)
        for lb in range(-(-n // bs)):
            if not any(t in vis for t in range(lb * bs, min(n, lb * bs + bs))):
                table[b, lb] = -1
    assert (table == -1).sum() > (x.block_table == -1).sum()
    kc, vc = _poison_invisible(x, window, n_sink)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = _run(x, window, n_sink, x.sinks, kc, vc, table, status=status)
    assert int(status.item()) == 0
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)


@pytest.mark.parametrize("s", [-40.0, 40.0])
def test_extreme_sink_logits(s):
    x = workloads.paged_decode_inputs(2, 8, 2, 128, seq_lens=[33, 600], block_size=16, seed=14)
    sinks = torch.full((8,), s, dtype=torch.float32)
    o, lse = _check(x, 128, 2, sinks, what=f"sink={s}")
    if s > 0:  # all mass on the sink: O ~ 0, LSE ~ s
        assert float(o.float().abs().max()) < 1e-8
        assert float((lse - s).abs().max()) < 1e-5


def test_non_finite_sink_is_flagged():
    x = workloads.paged_decode_inputs(2, 8, 2, 128, seq_lens=[33, 600], block_size=16, seed=15,
                                      learned_sinks=True)
    sinks = x.sinks.clone()
    sinks[3] = float("nan")
    sinks[6] = float("inf")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = _run(x, 0, 0, sinks, status=status)
    assert int(status.item()) & 0x1
    for h in (3, 6):
        assert torch.isnan(o[:, h].float()).all() and torch.isnan(lse[:, h]).all()
    good = [h for h in range(8) if h not in (3, 6)]
    for b in range(2):
        o_ref, l_ref = oracle.decode_rows_ref(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens, b, good,
                                              1 / math.sqrt(128), 0, 0, sinks.double().nan_to_num(0.0))
        assert_parity(o[b, good], o_ref, lse[b, good], l_ref)


def test_invalid_visible_entry_is_flagged():
    x = workloads.paged_decode_inputs(2, 8, 2, 128, seq_lens=[300, 300], block_size=16, seed=16)
    x.block_table[0, 0] = 10 ** 6  # a sink block of sequence 0
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = _run(x, 64, 4, None, status=status)
    assert int(status.item()) & 0x1
    assert torch.isnan(o[0].float()).all()
    o_ref, l_ref = oracle.decode_rows_ref(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens, 1, range(8),
                                          1 / math.sqrt(128), 64, 4)
    assert_parity(o[1], o_ref, lse[1], l_ref)


@pytest.mark.parametrize("name", sorted(workloads.WINDOW_DECODE_WORKLOADS))
def test_full_size_sampled(name):
    cfg = dict(workloads.WINDOW_DECODE_WORKLOADS[name])
    B, Hq, Hkv, d = cfg.pop("B"), cfg.pop("Hq"), cfg.pop("Hkv"), cfg.pop("d")
    window, n_sink = cfg.pop("window"), cfg.pop("n_sink")
    x = workloads.paged_decode_inputs(B, Hq, Hkv, d, seed=0, **cfg)
    rng = np.random.default_rng(2)
    seqs = sorted(set([0, B - 1] + rng.integers(0, B, 2).tolist()))
    heads = sorted(set([0, Hq - 1] + rng.integers(0, Hq, 4).tolist()))
    _check(x, window, n_sink, x.sinks, seqs=seqs, heads=heads, poison=False, what=name)
    assert accounting.decode_window_kv_bytes(x.seq_lens.tolist(), Hkv, d, window, n_sink) > 0
