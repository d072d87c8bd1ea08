"""ctypes loader for libattn_b200.so (the C ABI declared in include/attn.h).

There is no fallback: if the library is missing or fails to load, every call
raises. Build it with ``python -m exact_softmax_attention_causal_b200.csrc.build``.
"""

from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libattn_b200.so")

# Exported symbols, as declared in include/attn.h.
SYMBOLS = (
    "attn_prefill",
    "attn_prefill_paged",
    "attn_decode_plan",
    "attn_decode_workspace_bytes",
    "attn_decode_paged",
    "attn_decode_paged_noalloc",
    "attn_decode_window_workspace_bytes",
    "attn_decode_paged_window",
    "attn_prefill_backward_workspace_bytes",
    "attn_prefill_backward",
    "attn_mla_decode_workspace_bytes",
    "attn_mla_decode_paged",
    "attn_paged_gather",
    "attn_status_string",
    "attn_version",
)

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = -1
ATTN_ERR_UNSUPPORTED = -2
ATTN_ERR_CUDA = -3
ATTN_ERR_DEVICE_CHECK = -4
ATTN_ERR_TIMEOUT = -5
ATTN_ERR_WORKSPACE = -6
DECODE_NOALLOC_SCRATCH_BYTES = 32 << 20
STATUS_BIT_DEVICE_CHECK = 0x1
STATUS_BIT_TIMEOUT = 0x2

_lock = threading.Lock()
_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t


def _declare(lib):
    lib.attn_prefill.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _vp, _vp]
    lib.attn_prefill.restype = _i
    lib.attn_prefill_paged.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                                       _i, _f, _vp, _vp]
    lib.attn_prefill_paged.restype = _i
    lib.attn_decode_plan.argtypes = [_i, _i, _i, _i, _i, ctypes.POINTER(_i), ctypes.POINTER(_i)]
    lib.attn_decode_plan.restype = _i
    lib.attn_decode_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i]
    lib.attn_decode_workspace_bytes.restype = _sz
    lib.attn_decode_paged.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _vp,
                                      _sz, _vp, _vp]
    lib.attn_decode_paged.restype = _i
    lib.attn_decode_paged_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f,
                                              _vp, _vp]
    lib.attn_decode_paged_noalloc.restype = _i
    lib.attn_decode_window_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i]
    lib.attn_decode_window_workspace_bytes.restype = _sz
    lib.attn_decode_paged_window.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                                             _i, _i, _f, _vp, _sz, _vp, _vp]
    lib.attn_decode_paged_window.restype = _i
    lib.attn_prefill_backward_workspace_bytes.argtypes = [_i, _i, _i]
    lib.attn_prefill_backward_workspace_bytes.restype = _sz
    lib.attn_prefill_backward.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f,
                                          _vp, _sz, _vp, _vp]
    lib.attn_prefill_backward.restype = _i
    lib.attn_mla_decode_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
    lib.attn_mla_decode_workspace_bytes.restype = _sz
    lib.attn_mla_decode_paged.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _vp, _sz,
                                          _vp, _vp]
    lib.attn_mla_decode_paged.restype = _i
    lib.attn_paged_gather.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp]
    lib.attn_paged_gather.restype = _i
    lib.attn_status_string.argtypes = [_i]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_version.argtypes = []
    lib.attn_version.restype = _i


def lib() -> ctypes.CDLL:
    """The loaded library; raises RuntimeError when it is not built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m exact_softmax_attention_causal_b200.csrc.build`")
            handle = ctypes.CDLL(LIB_PATH)
            _declare(handle)
            _lib = handle
        return _lib


class AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {lib().attn_status_string(code).decode()} (status {code})")


def check(code: int, where: str) -> None:
    if code != ATTN_OK:
        raise AttnError(code, where)
