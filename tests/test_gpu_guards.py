"""Out-of-bounds write checks: every output, LSE, workspace and status word is
placed inside a larger buffer whose guard bytes on both sides hold a canary
pattern; after the call the canaries must be unchanged and the outputs must
still match the fp64 oracle. This is the write-side check for ragged tiles
(TMA stores of a last, partly filled query tile; partial MLA head blocks; the
split-partial workspace of the decode) that a memory checker would otherwise
give.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_softmax_attention_causal_b200 import (decode_paged, decode_paged_window, decode_window_workspace_bytes,
                                                  decode_workspace_bytes, mla_decode_paged,
                                                  mla_decode_workspace_bytes, paged_gather, prefill,
                                                  prefill_backward, prefill_backward_workspace_bytes, prefill_paged,
                                                  workloads)
from parity import assert_grad_parity, assert_parity

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side
CANARY = 0xA5
MASK_IDS = {"full": oracle.MASK_FULL, "causal": oracle.MASK_CAUSAL, "window": oracle.MASK_SLIDING_WINDOW}


class Guarded:
    """A tensor of `shape` and `dtype` in the middle of a canary-filled buffer."""

    def __init__(self, shape, dtype):
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((nbytes + 2 * GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        self.nbytes = nbytes
        self.t = self.raw[GUARD:GUARD + nbytes].view(dtype).view(shape)

    def check(self, what):
        torch.cuda.synchronize()
        lo = self.raw[:GUARD]
        hi = self.raw[GUARD + self.nbytes:]
        bad_lo = int((lo != CANARY).sum())
        bad_hi = int((hi != CANARY).sum())
        assert bad_lo == 0 and bad_hi == 0, f"{what}: {bad_lo} guard bytes changed below, {bad_hi} above"


def _ws(nbytes):
    g = Guarded((nbytes,), torch.uint8)
    return g


def _status():
    return Guarded((1,), torch.int32)


@pytest.mark.parametrize("d,mask,window,N", [(128, "causal", 0, 300), (64, "window", 50, 300), (128, "full", 0, 129),
                                             (64, "causal", 0, 1), (128, "window", 1, 257)])
def test_prefill_writes_stay_inside(d, mask, window, N):
    B, Hq, Hkv = 2, 4, 2
    x = workloads.prefill_inputs(B, Hq, Hkv, N, d, seed=40)
    o = Guarded((B, Hq, N, d), torch.bfloat16)
    lse = Guarded((B, Hq, N), torch.float32)
    st = _status()
    st.t.zero_()
    prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), mask=mask, window=window, out=o.t, lse=lse.t, status=st.t)
    for g, name in ((o, "O"), (lse, "LSE"), (st, "status")):
        g.check(f"prefill {name} N={N} d={d} {mask}")
    assert int(st.t.item()) == 0
    o_ref, l_ref = oracle.prefill_ref(x.q, x.k, x.v, MASK_IDS[mask], window, 1 / math.sqrt(d))
    assert_parity(o.t.cpu(), o_ref, lse.t.cpu(), l_ref, what="guarded prefill")


def test_prefill_paged_writes_stay_inside():
    B, Hq, Hkv, Nq, d = 2, 4, 1, 200, 128
    x = workloads.paged_prefill_inputs(B, Hq, Hkv, Nq, d, seq_lens=[300, 513], block_size=32, seed=41, extra_blocks=3)
    o = Guarded((B, Hq, Nq, d), torch.bfloat16)
    lse = Guarded((B, Hq, Nq), torch.float32)
    st = _status()
    st.t.zero_()
    prefill_paged(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.block_table.cuda(), x.seq_lens.cuda(),
                  x.max_seq_len, mask="causal", out=o.t, lse=lse.t, status=st.t)
    for g, name in ((o, "O"), (lse, "LSE"), (st, "status")):
        g.check(f"prefill_paged {name}")
    assert int(st.t.item()) == 0
    o_ref, l_ref = oracle.prefill_paged_ref(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens,
                                            oracle.MASK_CAUSAL, 0, 1 / math.sqrt(d))
    assert_parity(o.t.cpu(), o_ref, lse.t.cpu(), l_ref, what="guarded paged prefill")


@pytest.mark.parametrize("lens,Hq,Hkv", [([1, 700, 20000], 16, 4), ([131072], 32, 1), ([5, 3000], 8, 8)])
def test_decode_writes_stay_inside(lens, Hq, Hkv):
    d = 128
    x = workloads.paged_decode_inputs(len(lens), Hq, Hkv, d, seq_lens=lens, block_size=16, seed=42, extra_blocks=2)
    B = len(lens)
    o = Guarded((B, Hq, d), torch.bfloat16)
    lse = Guarded((B, Hq), torch.float32)
    ws = _ws(decode_workspace_bytes(B, Hq, Hkv, d, x.max_seq_len, 16))
    st = _status()
    st.t.zero_()
    decode_paged(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.block_table.cuda(), x.seq_lens.cuda(),
                 x.max_seq_len, out=o.t, lse=lse.t, workspace=ws.t, status=st.t)
    for g, name in ((o, "O"), (lse, "LSE"), (ws, "workspace"), (st, "status")):
        g.check(f"decode {name} {lens}")
    assert int(st.t.item()) == 0
    for b in range(B):
        heads = sorted(set([0, Hq // 2, Hq - 1]))
        o_ref, l_ref = oracle.decode_rows_ref(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens, b, heads,
                                              1 / math.sqrt(d))
        assert_parity(o.t[b, heads].cpu(), o_ref, lse.t[b, heads].cpu(), l_ref, what=f"guarded decode b={b}")


def test_decode_window_writes_stay_inside():
    B, Hq, Hkv, d, w, n_sink = 3, 8, 2, 64, 128, 4
    x = workloads.paged_decode_inputs(B, Hq, Hkv, d, seq_lens=[50, 1000, 9000], block_size=16, seed=43,
                                      learned_sinks=True)
    o = Guarded((B, Hq, d), torch.bfloat16)
    lse = Guarded((B, Hq), torch.float32)
    ws = _ws(decode_window_workspace_bytes(B, Hq, Hkv, d, x.max_seq_len, 16, w, n_sink))
    st = _status()
    st.t.zero_()
    decode_paged_window(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.block_table.cuda(), x.seq_lens.cuda(),
                        x.max_seq_len, window=w, n_sink=n_sink, sinks=x.sinks.cuda(), out=o.t, lse=lse.t,
                        workspace=ws.t, status=st.t)
    for g, name in ((o, "O"), (lse, "LSE"), (ws, "workspace"), (st, "status")):
        g.check(f"decode_window {name}")
    assert int(st.t.item()) == 0
    o_ref, l_ref = oracle.decode_paged_ref(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens, 1 / math.sqrt(d),
                                           window=w, n_sink=n_sink, sinks=x.sinks)
    assert_parity(o.t.cpu(), o_ref, lse.t.cpu(), l_ref, what="guarded windowed decode")


def test_mla_writes_stay_inside():
    B, H, dc, dr = 2, 20, 512, 64
    x = workloads.mla_decode_inputs(B, H, dc, dr, seq_lens=[100, 5000], block_size=16, seed=44)
    scale = 1 / math.sqrt(128 + dr)
    o = Guarded((B, H, dc), torch.bfloat16)
    lse = Guarded((B, H), torch.float32)
    ws = _ws(mla_decode_workspace_bytes(B, H, x.max_seq_len))
    st = _status()
    st.t.zero_()
    mla_decode_paged(x.q.cuda(), x.cache.cuda(), x.block_table.cuda(), x.seq_lens.cuda(), x.max_seq_len, scale,
                     out=o.t, lse=lse.t, workspace=ws.t, status=st.t)
    for g, name in ((o, "O"), (lse, "LSE"), (ws, "workspace"), (st, "status")):
        g.check(f"mla {name}")
    assert int(st.t.item()) == 0
    o_ref, l_ref = oracle.mla_decode_ref(x.q, x.cache, x.block_table, x.seq_lens, dc, scale)
    assert_parity(o.t.cpu(), o_ref, lse.t.cpu(), l_ref, what="guarded MLA decode")


@pytest.mark.parametrize("d,mask,window", [(128, "causal", 0), (64, "window", 70)])
def test_backward_writes_stay_inside(d, mask, window):
    B, Hq, Hkv, N = 1, 4, 2, 300
    x = workloads.prefill_inputs(B, Hq, Hkv, N, d, seed=45)
    gen = torch.Generator("cpu").manual_seed(46)
    d_o = torch.randn((B, Hq, N, d), generator=gen).to(torch.bfloat16)
    q, k, v, g = (t.cuda() for t in (x.q, x.k, x.v, d_o))
    o, lse = prefill(q, k, v, mask=mask, window=window)
    dq = Guarded((B, Hq, N, d), torch.bfloat16)
    dk = Guarded((B, Hkv, N, d), torch.bfloat16)
    dv = Guarded((B, Hkv, N, d), torch.bfloat16)
    ws = _ws(prefill_backward_workspace_bytes(B, Hq, N))
    st = _status()
    st.t.zero_()
    prefill_backward(q, k, v, o, lse, g, mask=mask, window=window, dq=dq.t, dk=dk.t, dv=dv.t, workspace=ws.t,
                     status=st.t)
    for gd, name in ((dq, "dQ"), (dk, "dK"), (dv, "dV"), (ws, "workspace"), (st, "status")):
        gd.check(f"backward {name} d={d} {mask}")
    assert int(st.t.item()) == 0
    r_q, r_k, r_v = oracle.prefill_backward_ref(x.q, x.k, x.v, d_o, MASK_IDS[mask], window, 1 / math.sqrt(d))
    assert_grad_parity(dq.t.cpu(), r_q, what="guarded dQ")
    assert_grad_parity(dk.t.cpu(), r_k, what="guarded dK")
    assert_grad_parity(dv.t.cpu(), r_v, what="guarded dV")


def test_paged_gather_writes_stay_inside():
    x = workloads.paged_decode_inputs(3, 4, 2, 128, seq_lens=[1, 33, 70], block_size=16, seed=47, extra_blocks=2)
    out = Guarded((3, 2, x.max_seq_len, 128), torch.bfloat16)
    paged_gather(x.k_cache.cuda(), x.block_table.cuda(), x.seq_lens.cuda(), x.max_seq_len, out=out.t)
    out.check("paged_gather out")
    ref = oracle.gather_paged_ref(x.k_cache, x.block_table, x.seq_lens, x.max_seq_len)
    assert np.array_equal(out.t.cpu().to(torch.float64).numpy(), ref)
