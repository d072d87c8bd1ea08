"""attn_decode_paged_noalloc: the decode entry point for callers that cannot
allocate device memory (a host framework that owns all device memory, or a
decode loop that must not pay for an allocation). It keeps its split
partials in the library's static device array instead of a caller workspace.

Checked through the C ABI against attn_decode_paged (caller workspace) on two
calls in a row with different inputs, so the second call runs on whatever the
first left in the shared array. This file is collected last on purpose.
"""

import ctypes
import math

import pytest
import torch

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
    return tuple(t.cuda() for t in (xi.q, xi.k_cache, xi.v_cache, xi.block_table, xi.seq_lens))


@pytest.mark.parametrize("first,second", [([1, 300, 4096, 17, 2048], [700, 5, 12000]),
                                          ([20000], [33, 33, 33, 33])])
def test_noalloc_matches_workspace_entry_point_twice(first, second):
    for seed, lens in ((1, first), (2, second)):
        x = _inputs(seed, lens)
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


def test_noalloc_rejects_requests_beyond_its_scratch():
    # 256 sequences x 32 heads x 16 splits x 129 floats is about 68 MB > 32 MiB
    B, Hq, Hkv, d, max_len = 256, 32, 8, 128, 32768
    assert decode_workspace_bytes(B, Hq, Hkv, d, max_len, 16) > _lib.DECODE_NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: the call is rejected before any launch
    rc = _lib.lib().attn_decode_paged_noalloc(fake, fake, fake, fake, fake, fake, None, B, Hq, Hkv, d, 4096, 16,
                                              max_len // 16, max_len, 0.1, None, None)
    assert rc == _lib.ATTN_ERR_WORKSPACE
