"""GPU parity of attn_prefill against the fp64 oracle (through the C ABI)."""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_softmax_attention_causal_b200 import prefill, workloads
from parity import assert_parity, to64

pytestmark = pytest.mark.gpu

MASK_IDS = {"full": oracle.MASK_FULL, "causal": oracle.MASK_CAUSAL, "window": oracle.MASK_SLIDING_WINDOW}


def _run(B, Hq, Hkv, N, d, mask, window=0, seed=0, scale=None):
    x = workloads.prefill_inputs(B, Hq, Hkv, N, d, seed)
    scale = scale if scale is not None else 1.0 / math.sqrt(d)
    q, k, v = (t.cuda() for t in (x.q, x.k, x.v))
    o, lse = prefill(q, k, v, mask=mask, window=window, scale=scale)
    torch.cuda.synchronize()
    return x, o.cpu(), lse.cpu(), scale


def _full_check(B, Hq, Hkv, N, d, mask, window=0, seed=0):
    x, o, lse, scale = _run(B, Hq, Hkv, N, d, mask, window, seed)
    o_ref, lse_ref = oracle.prefill_ref(x.q, x.k, x.v, MASK_IDS[mask], window, scale)
    return assert_parity(o, o_ref, lse, lse_ref, what=f"{B}x{Hq}/{Hkv}x{N}x{d} {mask} w={window}")


def test_tiny_causal_gqa_config():
    """B=1, Hq=4, Hkv=2, N=128, d=64, seed 0, scale 1/8, causal."""
    _full_check(1, 4, 2, 128, 64, "causal")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mask,window", [("causal", 0), ("full", 0), ("window", 1), ("window", 50),
                                         ("window", 130), ("window", 257), ("window", 1000)])
def test_ragged_multi_tile(d, mask, window):
    # N = 300: three 128-row tiles, the last one ragged (44 rows)
    _full_check(1, 4, 2, 300, d, mask, window, seed=1)


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 1), (6, 3)])
def test_head_maps(hq, hkv):
    _full_check(2, hq, hkv, 256, 128, "causal", seed=2)


@pytest.mark.parametrize("N", [1, 7, 129, 257, 640])
def test_sizes(N):
    _full_check(1, 2, 1, N, 128, "causal", seed=3)
    _full_check(1, 2, 1, N, 64, "full", seed=3)
    # small windows: the second query tile of an item may have no row before N
    _full_check(1, 2, 1, N, 128, "window", window=1, seed=3)
    _full_check(1, 2, 1, N, 64, "window", window=3, seed=3)


def test_causal_row0_is_v0_exactly():
    x, o, lse, scale = _run(2, 8, 2, 256, 128, "causal", seed=4)
    for h in range(8):
        assert torch.equal(o[:, h, 0], x.v[:, h // 4, 0])
    ref = (x.q[:, :, 0].double() * x.k[:, :, 0].double().repeat_interleave(4, dim=1)).sum(-1) * scale
    assert float((lse[:, :, 0].double() - ref).abs().max()) <= 1e-5


def test_equal_scores_give_mean_of_visible_values():
    B, Hq, Hkv, N, d, w = 1, 2, 1, 384, 128, 100
    x = workloads.prefill_inputs(B, Hq, Hkv, N, d, 5)
    q = torch.zeros_like(x.q).cuda()
    for mask, win in (("causal", 0), ("window", w)):
        o, lse = prefill(q, x.k.cuda(), x.v.cuda(), mask=mask, window=win)
        v = to64(x.v)[0, 0]
        i = np.arange(N)
        lo = np.maximum(0, i - win + 1) if mask == "window" else np.zeros(N, dtype=int)
        csum = np.concatenate([np.zeros((1, d)), np.cumsum(v, axis=0)])
        mean = (csum[i + 1] - csum[lo]) / (i + 1 - lo)[:, None]
        for h in range(Hq):
            assert_parity(o[0, h].cpu(), mean, lse[0, h].cpu(), np.log(i + 1 - lo), what=mask)


def test_wide_window_equals_causal_bitwise():
    x = workloads.prefill_inputs(1, 4, 2, 300, 128, 6)
    q, k, v = (t.cuda() for t in (x.q, x.k, x.v))
    oc, lc = prefill(q, k, v, mask="causal")
    for w in (300, 305, 600):
        ow, lw = prefill(q, k, v, mask="window", window=w)
        assert torch.equal(oc, ow) and torch.equal(lc, lw)


def test_deterministic_across_calls():
    x = workloads.prefill_inputs(1, 4, 1, 512, 128, 7)
    q, k, v = (t.cuda() for t in (x.q, x.k, x.v))
    o1, l1 = prefill(q, k, v, mask="causal")
    o2, l2 = prefill(q, k, v, mask="causal")
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_lse_optional_and_status_clean():
    x = workloads.prefill_inputs(1, 2, 2, 200, 64, 8)
    q, k, v = (t.cuda() for t in (x.q, x.k, x.v))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = prefill(q, k, v, mask="causal", return_lse=False, status=status)
    assert lse is None
    o2, _ = prefill(q, k, v, mask="causal")
    torch.cuda.synchronize()
    assert int(status.item()) == 0 and torch.equal(o, o2)


def test_bounded_wait_timeout_reports_status(monkeypatch):
    """A one-cycle wait budget makes pipeline waits give up: the call must come
    back with the timeout bit and NaN rows instead of hanging, and the context
    must stay usable (a normal call afterwards is correct)."""
    x = workloads.prefill_inputs(1, 2, 1, 1024, 128, 9)
    q, k, v = (t.cuda() for t in (x.q, x.k, x.v))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    monkeypatch.setenv("ATTN_WAIT_BUDGET_CYCLES", "1")
    o, _ = prefill(q, k, v, mask="causal", status=status)
    torch.cuda.synchronize()
    monkeypatch.delenv("ATTN_WAIT_BUDGET_CYCLES")
    st = int(status.item())
    # a one-cycle budget cannot cover the ring waits (a K/V slot is released
    # only after the P.V products of both query tiles), so waits must expire:
    # the timeout bit is set and the rows left unfinished are NaN, not garbage
    assert st & 0x2, f"status {st:#x}: no bounded wait expired under a one-cycle budget"
    assert torch.isnan(o.float()).any()
    o2, lse2 = prefill(q, k, v, mask="causal")
    o_ref, lse_ref = oracle.prefill_ref(x.q, x.k, x.v, oracle.MASK_CAUSAL, 0, 1 / math.sqrt(128))
    assert_parity(o2.cpu(), o_ref, lse2.cpu(), lse_ref)


# --------------------------------------------------------------------------
# full-size workloads, sampled rows (the oracle computes chosen rows directly)
# --------------------------------------------------------------------------
def _sample_rows(N, rng, n=24):
    fixed = [0, 1, 127, 128, 129, N // 2, N - 129, N - 128, N - 2, N - 1]
    extra = rng.integers(0, N, n - len(fixed)).tolist()
    return sorted(set(r for r in fixed + extra if 0 <= r < N))


@pytest.mark.parametrize("name", ["llama3_8b_causal_gqa", "long_causal_n32768", "long_window4096_n32768",
                                  "gqa_dial_prefill_mha", "gqa_dial_prefill_gqa8", "gqa_dial_prefill_mqa"])
def test_full_size_sampled(name):
    cfg = workloads.PREFILL_WORKLOADS[name]
    B, Hq, Hkv, N, d = cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["N"], cfg["d"]
    x, o, lse, scale = _run(B, Hq, Hkv, N, d, cfg["mask"], cfg["window"], seed=0)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    rng = np.random.default_rng(0)
    heads = sorted(set([0, Hq - 1, int(rng.integers(0, Hq))]))
    for b in sorted(set([0, B - 1])):
        for h in heads:
            rows = _sample_rows(N, rng)
            o_ref, l_ref = oracle.prefill_rows_ref(x.q, x.k, x.v, b, h, rows, MASK_IDS[cfg["mask"]], cfg["window"],
                                                   scale)
            assert_parity(o[b, h, rows], o_ref, lse[b, h, rows], l_ref, what=f"{name} b={b} h={h}")
