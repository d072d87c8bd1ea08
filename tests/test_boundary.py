"""CPU checks of the C-ABI boundary: the library loads, exports every symbol
include/attn.h declares, rejects bad arguments before launching anything,
and plans decode splits on the host. No test here launches a kernel."""

import ctypes
import os
import re

import pytest

from exact_softmax_attention_causal_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", text)


def test_header_declares_expected_entry_points():
    names = declared_symbols()
    assert set(names) == set(_lib.SYMBOLS), names


def test_library_loads_and_exports_every_declared_symbol():
    lib = _lib.lib()
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert lib.attn_version() >= 100


def test_status_strings():
    lib = _lib.lib()
    for code in (0, -1, -2, -3, -4, -5, -6):
        s = lib.attn_status_string(code).decode()
        assert s and s != "unknown status"
    assert lib.attn_status_string(42).decode() == "unknown status"


FAKE = ctypes.c_void_p(0x10000)  # aligned, never dereferenced: every call below fails validation first
NULL = ctypes.c_void_p(0)


def _prefill(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=NULL, B=1, Hq=4, Hkv=2, N=128, d=64, mask=1, window=0,
             scale=0.125)
    a.update(kw)
    return _lib.lib().attn_prefill(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["N"],
                                   a["d"], a["mask"], a["window"], a["scale"], NULL, NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(q=NULL), _lib.ATTN_ERR_INVALID_ARG),
    (dict(o=NULL), _lib.ATTN_ERR_INVALID_ARG),
    (dict(B=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(N=-1), _lib.ATTN_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), _lib.ATTN_ERR_INVALID_ARG),
    (dict(mask=7), _lib.ATTN_ERR_INVALID_ARG),
    (dict(mask=2, window=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(scale=0.0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), _lib.ATTN_ERR_INVALID_ARG),
    (dict(q=ctypes.c_void_p(0x10008)), _lib.ATTN_ERR_INVALID_ARG),
    (dict(d=96), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(d=256), _lib.ATTN_ERR_UNSUPPORTED),
])
def test_prefill_rejects_bad_arguments(kw, code):
    assert _prefill(**kw) == code


def _decode(**kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, sl=FAKE, o=FAKE, lse=NULL, B=2, Hq=8, Hkv=2, d=128, nb=10, bs=16,
             mb=4, msl=64, scale=0.1, ws=FAKE, wsb=1 << 20)
    a.update(kw)
    return _lib.lib().attn_decode_paged(a["q"], a["kc"], a["vc"], a["bt"], a["sl"], a["o"], a["lse"], a["B"],
                                        a["Hq"], a["Hkv"], a["d"], a["nb"], a["bs"], a["mb"], a["msl"], a["scale"],
                                        a["ws"], a["wsb"], NULL, NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(q=NULL), _lib.ATTN_ERR_INVALID_ARG),
    (dict(bt=NULL), _lib.ATTN_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), _lib.ATTN_ERR_INVALID_ARG),
    (dict(mb=3), _lib.ATTN_ERR_INVALID_ARG),  # 3 blocks of 16 cannot hold 64 tokens
    (dict(nb=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(scale=-1.0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(bt=ctypes.c_void_p(0x10002)), _lib.ATTN_ERR_INVALID_ARG),
    (dict(d=80), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(bs=8, mb=8), _lib.ATTN_ERR_UNSUPPORTED),
])
def test_decode_rejects_bad_arguments(kw, code):
    assert _decode(**kw) == code


def _decode_window(**kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, sl=FAKE, sinks=NULL, o=FAKE, lse=NULL, B=2, Hq=8, Hkv=2, d=128, nb=10,
             bs=16, mb=4, msl=64, window=16, n_sink=4, scale=0.1, ws=FAKE, wsb=1 << 20)
    a.update(kw)
    return _lib.lib().attn_decode_paged_window(a["q"], a["kc"], a["vc"], a["bt"], a["sl"], a["sinks"], a["o"],
                                               a["lse"], a["B"], a["Hq"], a["Hkv"], a["d"], a["nb"], a["bs"], a["mb"],
                                               a["msl"], a["window"], a["n_sink"], a["scale"], a["ws"], a["wsb"],
                                               NULL, NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(q=NULL), _lib.ATTN_ERR_INVALID_ARG),
    (dict(window=-1), _lib.ATTN_ERR_INVALID_ARG),
    (dict(n_sink=-1), _lib.ATTN_ERR_INVALID_ARG),
    (dict(window=0, n_sink=1), _lib.ATTN_ERR_INVALID_ARG),  # sink positions only beside a finite window
    (dict(n_sink=65), _lib.ATTN_ERR_INVALID_ARG),           # n_sink > max_seq_len
    (dict(sinks=ctypes.c_void_p(0x10002)), _lib.ATTN_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), _lib.ATTN_ERR_INVALID_ARG),
    (dict(mb=3), _lib.ATTN_ERR_INVALID_ARG),
    (dict(d=80), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(bs=8, mb=8), _lib.ATTN_ERR_UNSUPPORTED),
])
def test_decode_window_rejects_bad_arguments(kw, code):
    assert _decode_window(**kw) == code


def test_decode_window_workspace_rejects_bad_sizes():
    lib = _lib.lib()
    assert lib.attn_decode_window_workspace_bytes(2, 8, 2, 80, 64, 16, 16, 0) == 0
    assert lib.attn_decode_window_workspace_bytes(2, 8, 2, 128, 64, 8, 16, 0) == 0
    assert lib.attn_decode_window_workspace_bytes(2, 8, 2, 128, 64, 16, -1, 0) == 0


def _mla(**kw):
    a = dict(q=FAKE, c=FAKE, bt=FAKE, sl=FAKE, o=FAKE, lse=NULL, B=2, H=128, dc=512, dr=64, nb=10, bs=16, mb=4, msl=64,
             scale=0.07, ws=FAKE, wsb=1 << 20)
    a.update(kw)
    return _lib.lib().attn_mla_decode_paged(a["q"], a["c"], a["bt"], a["sl"], a["o"], a["lse"], a["B"], a["H"],
                                            a["dc"], a["dr"], a["nb"], a["bs"], a["mb"], a["msl"], a["scale"],
                                            a["ws"], a["wsb"], NULL, NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(q=NULL), _lib.ATTN_ERR_INVALID_ARG),
    (dict(c=ctypes.c_void_p(0x10008)), _lib.ATTN_ERR_INVALID_ARG),
    (dict(H=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(mb=3), _lib.ATTN_ERR_INVALID_ARG),
    (dict(scale=0.0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(dc=256), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(dr=32), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(bs=48, mb=2), _lib.ATTN_ERR_UNSUPPORTED),
])
def test_mla_rejects_bad_arguments(kw, code):
    assert _mla(**kw) == code


def test_mla_workspace_rejects_unsupported_widths():
    assert _lib.lib().attn_mla_decode_workspace_bytes(2, 128, 256, 64, 1024) == 0


def _bwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, do=FAKE, lse=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, B=1, Hq=4, Hkv=2, N=256,
             d=128, mask=1, window=0, scale=0.1, ws=FAKE, wsb=1 << 20)
    a.update(kw)
    return _lib.lib().attn_prefill_backward(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"],
                                            a["dv"], a["B"], a["Hq"], a["Hkv"], a["N"], a["d"], a["mask"],
                                            a["window"], a["scale"], a["ws"], a["wsb"], NULL, NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(do=NULL), _lib.ATTN_ERR_INVALID_ARG),
    (dict(lse=NULL), _lib.ATTN_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), _lib.ATTN_ERR_INVALID_ARG),
    (dict(mask=2, window=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(dk=ctypes.c_void_p(0x10008)), _lib.ATTN_ERR_INVALID_ARG),
    (dict(d=96), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(ws=NULL), _lib.ATTN_ERR_WORKSPACE),
    (dict(wsb=100), _lib.ATTN_ERR_WORKSPACE),
    (dict(B=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(N=-1), _lib.ATTN_ERR_INVALID_ARG),
    (dict(mask=7), _lib.ATTN_ERR_INVALID_ARG),
    (dict(scale=0.0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), _lib.ATTN_ERR_INVALID_ARG),
    (dict(B=70000), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(Hq=70000, Hkv=2), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(B=1, Hq=4, N=1 << 29), _lib.ATTN_ERR_UNSUPPORTED),  # B * Hq * N = 2^31
])
def test_backward_rejects_bad_arguments(kw, code):
    assert _bwd(**kw) == code


def test_backward_workspace_is_two_floats_per_padded_row():
    assert _lib.lib().attn_prefill_backward_workspace_bytes(2, 8, 300) == 2 * (2 * 8 * 384 * 4)
    assert _lib.lib().attn_prefill_backward_workspace_bytes(0, 8, 300) == 0


def _prefill_paged(**kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, sl=FAKE, o=FAKE, lse=NULL, B=2, Hq=8, Hkv=2, Nq=64, d=128, nb=10,
             bs=16, mb=8, msl=128, mask=1, window=0, scale=0.1)
    a.update(kw)
    return _lib.lib().attn_prefill_paged(a["q"], a["kc"], a["vc"], a["bt"], a["sl"], a["o"], a["lse"], a["B"],
                                         a["Hq"], a["Hkv"], a["Nq"], a["d"], a["nb"], a["bs"], a["mb"], a["msl"],
                                         a["mask"], a["window"], a["scale"], NULL, NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(sl=NULL), _lib.ATTN_ERR_INVALID_ARG),
    (dict(Nq=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(msl=32), _lib.ATTN_ERR_INVALID_ARG),   # max_seq_len < Nq
    (dict(mb=7), _lib.ATTN_ERR_INVALID_ARG),     # 7 blocks of 16 cannot hold 128 tokens
    (dict(Hq=6, Hkv=4), _lib.ATTN_ERR_INVALID_ARG),
    (dict(mask=2, window=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(q=ctypes.c_void_p(0x10004)), _lib.ATTN_ERR_INVALID_ARG),
    (dict(d=96), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(bs=8, mb=16), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(bs=48, mb=3, msl=128), _lib.ATTN_ERR_UNSUPPORTED),
])
def test_prefill_paged_rejects_bad_arguments(kw, code):
    assert _prefill_paged(**kw) == code


def test_gather_rejects_bad_arguments():
    lib = _lib.lib()
    assert lib.attn_paged_gather(NULL, FAKE, FAKE, FAKE, 1, 1, 64, 4, 16, 2, 32, NULL, NULL) == _lib.ATTN_ERR_INVALID_ARG
    assert lib.attn_paged_gather(FAKE, FAKE, FAKE, FAKE, 1, 1, 64, 4, 16, 1, 32, NULL, NULL) == _lib.ATTN_ERR_INVALID_ARG


def _plan(B, Hq, Hkv, L, sms=148):
    c, s = ctypes.c_int(), ctypes.c_int()
    rc = _lib.lib().attn_decode_plan(B, Hq, Hkv, L, sms, ctypes.byref(c), ctypes.byref(s))
    return rc, c.value, s.value


@pytest.mark.parametrize("B,Hq,Hkv,L", [(64, 32, 8, 32768), (1, 32, 1, 131072), (1, 32, 8, 131072),
                                         (1, 32, 32, 131072), (3, 4, 2, 300), (1, 1, 1, 1)])
def test_decode_plan_covers_the_sequence(B, Hq, Hkv, L):
    rc, chunk, splits = _plan(B, Hq, Hkv, L)
    assert rc == _lib.ATTN_OK
    assert chunk % 16 == 0 and 16 <= chunk <= 4096
    assert splits == -(-L // chunk)
    # the 16-token sub-blocks are spread evenly: no split holds less than a sub-block less than another
    subs = -(-L // 16)
    assert subs - (splits - 1) * (chunk // 16) >= max(1, chunk // 16 - splits)
    # at least one (sequence, kv head, head chunk, split) CTA per SM of 148, unless chunks are small
    units = B * Hkv * -(-(Hq // Hkv) // 16) * splits
    assert units >= 148 or chunk <= 256


def test_decode_plan_examples():
    assert _plan(64, 32, 8, 32768)[1:] == (2048, 16)  # enough (sequence, head) units: 2048-token splits
    # few units: whole waves of two resident CTAs per SM (296 on 148 SMs)
    assert _plan(1, 32, 8, 131072)[1:] == (3552, 37)   # 8 units x 37 splits = 296 CTAs, one wave
    assert _plan(1, 32, 32, 131072)[1:] == (3552, 37)  # 32 units x 37 splits = 4 waves
    assert _plan(1, 32, 1, 131072)[1:] == (896, 147)   # 2 head chunks x 147 splits: one wave
    assert _plan(64, 32, 8, 4128)[1:] == (1376, 3)  # a 4096 window + 4 sinks: 258 sub-blocks in 3 even splits
    assert _plan(0, 32, 1, 131072)[0] == _lib.ATTN_ERR_INVALID_ARG
    assert _plan(1, 32, 3, 100)[0] == _lib.ATTN_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        _lib.lib()
