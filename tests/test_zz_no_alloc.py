"""attn_decode_paged_noalloc: the decode entry point for callers that cannot
allocate device memory (a host framework that owns all device memory, or a
decode loop that must not pay for an allocation). It keeps its split
partials in the library's static device array instead of a caller workspace.

Checked through the C ABI against attn_decode_paged (caller workspace) and
against the fp64 oracle on two calls in a row with different inputs, so the
second call runs on whatever the first left in the shared array. This file is
collected last on purpose.
"""

import ctypes
import math

import pytest
import torch

import oracle
from exact_softmax_attention_causal_b200 import _lib, decode_paged, decode_workspace_bytes, workloads
from parity import assert_parity

pytestmark = pytest.mark.gpu


def _noalloc(x, out, lse, status):
    q, kc, vc, bt, sl = x
    B, Hq, d = q.shape
    nb, bs, Hkv, _ = kc.shape
    return _lib.lib().attn_decode_paged_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()), ctypes.c_void_p(vc.data_ptr()),
        ctypes.c_void_p(bt.data_ptr()), ctypes.c_void_p(sl.data_ptr()), ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(lse.data_ptr()), B, Hq, Hkv, d, nb, bs, bt.shape[1], x_max_len(x), 1.0 / math.sqrt(d),
        ctypes.c_void_p(status.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def x_max_len(x):
    return x[3].shape[1] * x[2].shape[1]  # max_blocks_per_seq * block_size


def _inputs(seed, seq_lens, Hq=16, Hkv=4, d=128):
    xi = workloads.paged_decode_inputs(len(seq_lens), Hq, Hkv, d, seq_lens=seq_lens, block_size=16, seed=seed,
                                       extra_blocks=2)
    return xi, tuple(t.cuda() for t in (xi.q, xi.k_cache, xi.v_cache, xi.block_table, xi.seq_lens))


@pytest.mark.parametrize("first,second", [([1, 300, 4096, 17, 2048], [700, 5, 12000]),
                                          ([20000], [33, 33, 33, 33])])
def test_noalloc_matches_workspace_entry_point_twice(first, second):
    for seed, lens in ((1, first), (2, second)):
        xi, x = _inputs(seed, lens)
        q, kc, vc, bt, sl = x
        o_ref, l_ref = decode_paged(q, kc, vc, bt, sl, x_max_len(x))
        out = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(l_ref, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = _noalloc(x, out, lse, status)
        assert rc == _lib.ATTN_OK, rc
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert_parity(out.cpu(), o_ref.cpu(), lse.cpu(), l_ref.cpu(), what=f"noalloc call seed {seed}")
        # and against the fp64 oracle directly, so that a fault shared by the
        # two entry points' kernels cannot hide behind their agreement
        Hq = q.shape[1]
        heads = sorted(set([0, Hq // 2, Hq - 1]))
        for b in range(q.shape[0]):
            o64, l64 = oracle.decode_rows_ref(xi.q, xi.k_cache, xi.v_cache, xi.block_table, xi.seq_lens, b, heads,
                                              1.0 / math.sqrt(q.shape[2]))
            assert_parity(out[b, heads].cpu(), o64, lse[b, heads].cpu(), l64, what=f"noalloc vs oracle b={b}")


def test_noalloc_rejects_requests_beyond_its_scratch():
    # 256 sequences x 32 heads x 16 splits x 129 floats is about 68 MB > 32 MiB.
    # Every pointer is a real device buffer with valid contents (one cached
    # token per sequence, table entries 0), so even a call that got past the
    # size check would only read memory it owns.
    B, Hq, Hkv, d, max_len, bs = 256, 32, 8, 128, 32768, 16
    assert decode_workspace_bytes(B, Hq, Hkv, d, max_len, bs) > _lib.DECODE_NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, bs, Hkv, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    bt = torch.zeros((B, max_len // bs), dtype=torch.int32, device="cuda")
    sl = torch.ones((B,), dtype=torch.int32, device="cuda")
    out = torch.zeros_like(q)
    lse = torch.zeros((B, Hq), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    p = [ctypes.c_void_p(t.data_ptr()) for t in (q, kc, vc, bt, sl, out, lse, status)]
    rc = _lib.lib().attn_decode_paged_noalloc(p[0], p[1], p[2], p[3], p[4], p[5], p[6], B, Hq, Hkv, d, 1, bs,
                                              max_len // bs, max_len, 0.1, p[7],
                                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == _lib.ATTN_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert int(status.item()) == 0 and not bool(out.any())  # nothing ran
