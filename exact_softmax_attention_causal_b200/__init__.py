"""Exact softmax attention for NVIDIA B200 (sm_100a).

Causal / sliding-window / full grouped-query prefill (contiguous, or the
newest positions against a paged context) and paged single-token decode (whole
cache, or a sliding window with sink positions and learned sink logits),
computed by hand-written CUDA kernels behind the C ABI of
``include/attn.h``. This module is the thin Python binding: it checks tensor
dtypes, shapes and devices, allocates outputs with PyTorch (device memory
plumbing only) and passes raw pointers and the current CUDA stream to the
library. Every step of the computation runs in the library's kernels; there
is no CPU or PyTorch fallback, and calls raise if the library is not built.
"""

from __future__ import annotations

import ctypes
import math

import torch

from . import _lib
from ._lib import AttnError, STATUS_BIT_DEVICE_CHECK, STATUS_BIT_TIMEOUT  # noqa: F401

MASKS = {"full": 0, "causal": 1, "window": 2, "sliding_window": 2}

__all__ = ["prefill", "prefill_paged", "decode_paged", "decode_paged_window", "paged_gather", "decode_plan",
           "decode_workspace_bytes", "decode_window_workspace_bytes", "mla_decode_paged", "mla_decode_workspace_bytes",
           "prefill_backward", "prefill_backward_workspace_bytes",
           "AttnError", "version"]


def version() -> int:
    return int(_lib.lib().attn_version())


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype, ndim: int) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got {t.dim()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _need_out(t, name: str, dtype, shape) -> None:
    """A caller-provided output must be a contiguous CUDA tensor of the exact
    dtype and shape: the library writes shape-many elements at its address."""
    _need(t, name, dtype, len(shape))
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _need_buf(t, name: str) -> None:
    """Workspace / status buffers: contiguous CUDA memory (any dtype)."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if name == "status" and (t.dtype != torch.int32 or t.numel() < 1):
        raise TypeError("status must be an int32 CUDA tensor with at least one element")


def prefill(q, k, v, mask: str = "causal", window: int = 0, scale: float | None = None, out=None, lse=None,
            status=None, stream=None, return_lse: bool = True):
    """O = softmax(scale * Q K^T + M) V for every query row; returns (O, LSE).

    q [B, Hq, N, d], k/v [B, Hkv, N, d], bf16 CUDA tensors; O bf16 like q,
    LSE fp32 [B, Hq, N] (natural log). mask: "full", "causal" or "window"
    (keys i - window < j <= i).
    """
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, N, d] matching q")
    if mask not in MASKS:
        raise ValueError(f"mask must be one of {sorted(MASKS)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    _need_out(out, "out", torch.bfloat16, q.shape)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need_out(lse, "lse", torch.float32, (B, Hq, N))
    _need_buf(status, "status")
    rc = _lib.lib().attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N, d, MASKS[mask],
                                 int(window), float(scale), _ptr(status), _stream_handle(stream))
    _lib.check(rc, "attn_prefill")
    return out, lse


def prefill_backward_workspace_bytes(B: int, Hq: int, N: int) -> int:
    n = int(_lib.lib().attn_prefill_backward_workspace_bytes(B, Hq, N))
    if n == 0:
        raise AttnError(_lib.ATTN_ERR_INVALID_ARG, "attn_prefill_backward_workspace_bytes")
    return n


def prefill_backward(q, k, v, o, lse, d_o, mask: str = "causal", window: int = 0, scale: float | None = None,
                     dq=None, dk=None, dv=None, workspace=None, status=None, stream=None):
    """Gradients (dQ, dK, dV) of prefill() for the output gradient d_o, from the
    forward's inputs, output O and LSE. Shapes as in prefill(); bf16 results."""
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (d_o, "d_o")):
        _need(t, name, torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape or o.shape != q.shape or d_o.shape != q.shape:
        raise ValueError("k, v must be [B, Hkv, N, d]; o and d_o like q")
    if lse.shape != (B, Hq, N):
        raise ValueError("lse must be [B, Hq, N]")
    if mask not in MASKS:
        raise ValueError(f"mask must be one of {sorted(MASKS)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _need_out(dq, "dq", torch.bfloat16, q.shape)
    _need_out(dk, "dk", torch.bfloat16, k.shape)
    _need_out(dv, "dv", torch.bfloat16, v.shape)
    if workspace is None:
        workspace = torch.empty(prefill_backward_workspace_bytes(B, Hq, N), dtype=torch.uint8, device=q.device)
    _need_buf(workspace, "workspace")
    _need_buf(status, "status")
    rc = _lib.lib().attn_prefill_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(d_o), _ptr(lse), _ptr(dq), _ptr(dk),
                                          _ptr(dv), B, Hq, Hkv, N, d, MASKS[mask], int(window), float(scale),
                                          _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
                                          _stream_handle(stream))
    _lib.check(rc, "attn_prefill_backward")
    return dq, dk, dv


def prefill_paged(q, k_cache, v_cache, block_table, seq_lens, max_seq_len: int, mask: str = "causal",
                  window: int = 0, scale: float | None = None, out=None, lse=None, status=None, stream=None,
                  return_lse: bool = True):
    """Prefix (chunked) prefill: the newest Nq positions of every sequence attend
    to its seq_lens[b] cached tokens through the block table; returns (O, LSE).

    q [B, Hq, Nq, d] bf16; caches [num_blocks, block_size, Hkv, d] bf16;
    block_table [B, max_blocks] int32; seq_lens [B] int32 (each >= Nq).
    Query row i of sequence b sits at position seq_lens[b] - Nq + i.
    """
    _need(q, "q", torch.bfloat16, 4)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    B, Hq, Nq, d = q.shape
    num_blocks, block_size, Hkv, d2 = k_cache.shape
    if d2 != d or v_cache.shape != k_cache.shape:
        raise ValueError("caches must be [num_blocks, block_size, Hkv, d] matching q")
    if block_table.shape[0] != B or seq_lens.shape[0] != B:
        raise ValueError("block_table and seq_lens need one row per sequence")
    if mask not in MASKS:
        raise ValueError(f"mask must be one of {sorted(MASKS)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    _need_out(out, "out", torch.bfloat16, q.shape)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need_out(lse, "lse", torch.float32, (B, Hq, Nq))
    _need_buf(status, "status")
    rc = _lib.lib().attn_prefill_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens),
                                       _ptr(out), _ptr(lse), B, Hq, Hkv, Nq, d, num_blocks, block_size,
                                       block_table.shape[1], int(max_seq_len), MASKS[mask], int(window),
                                       float(scale), _ptr(status), _stream_handle(stream))
    _lib.check(rc, "attn_prefill_paged")
    return out, lse


def decode_plan(B: int, Hq: int, Hkv: int, max_seq_len: int, num_sms: int):
    """(chunk_tokens, num_splits) of the split-KV decode plan; host only."""
    chunk, splits = ctypes.c_int(0), ctypes.c_int(0)
    rc = _lib.lib().attn_decode_plan(B, Hq, Hkv, max_seq_len, num_sms, ctypes.byref(chunk), ctypes.byref(splits))
    _lib.check(rc, "attn_decode_plan")
    return chunk.value, splits.value


def decode_workspace_bytes(B: int, Hq: int, Hkv: int, d: int, max_seq_len: int, block_size: int) -> int:
    n = int(_lib.lib().attn_decode_workspace_bytes(B, Hq, Hkv, d, max_seq_len, block_size))
    if n == 0:
        raise AttnError(_lib.ATTN_ERR_INVALID_ARG, "attn_decode_workspace_bytes")
    return n


def decode_paged(q, k_cache, v_cache, block_table, seq_lens, max_seq_len: int, scale: float | None = None,
                 out=None, lse=None, workspace=None, status=None, stream=None, return_lse: bool = True):
    """One query token per sequence against its paged cache; returns (O, LSE).

    q [B, Hq, d] bf16; caches [num_blocks, block_size, Hkv, d] bf16;
    block_table [B, max_blocks] int32; seq_lens [B] int32.
    """
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    B, Hq, d = q.shape
    num_blocks, block_size, Hkv, d2 = k_cache.shape
    if d2 != d or v_cache.shape != k_cache.shape:
        raise ValueError("caches must be [num_blocks, block_size, Hkv, d] matching q")
    if block_table.shape[0] != B or seq_lens.shape[0] != B:
        raise ValueError("block_table and seq_lens need one row per sequence")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if workspace is None:
        nbytes = decode_workspace_bytes(B, Hq, Hkv, d, max_seq_len, block_size)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    _need_buf(workspace, "workspace")
    if out is None:
        out = torch.empty_like(q)
    _need_out(out, "out", torch.bfloat16, q.shape)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need_out(lse, "lse", torch.float32, (B, Hq))
    _need_buf(status, "status")
    rc = _lib.lib().attn_decode_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens),
                                      _ptr(out), _ptr(lse), B, Hq, Hkv, d, num_blocks, block_size,
                                      block_table.shape[1], int(max_seq_len), float(scale), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _ptr(status),
                                      _stream_handle(stream))
    _lib.check(rc, "attn_decode_paged")
    return out, lse


def decode_window_workspace_bytes(B: int, Hq: int, Hkv: int, d: int, max_seq_len: int, block_size: int, window: int,
                                  n_sink: int) -> int:
    n = int(_lib.lib().attn_decode_window_workspace_bytes(B, Hq, Hkv, d, max_seq_len, block_size, window, n_sink))
    if n == 0:
        raise AttnError(_lib.ATTN_ERR_INVALID_ARG, "attn_decode_window_workspace_bytes")
    return n


def decode_paged_window(q, k_cache, v_cache, block_table, seq_lens, max_seq_len: int, window: int = 0,
                        n_sink: int = 0, sinks=None, scale: float | None = None, out=None, lse=None, workspace=None,
                        status=None, stream=None, return_lse: bool = True):
    """Paged decode with a sliding window of `window` positions (0: none), the
    first `n_sink` positions kept visible, and optional learned per-head sink
    logits `sinks` (fp32 [Hq], appended to the scaled scores with no value).
    Returns (O [B, Hq, d] bf16, LSE [B, Hq] fp32, including the sink column).
    """
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    B, Hq, d = q.shape
    num_blocks, block_size, Hkv, d2 = k_cache.shape
    if d2 != d or v_cache.shape != k_cache.shape:
        raise ValueError("caches must be [num_blocks, block_size, Hkv, d] matching q")
    if block_table.shape[0] != B or seq_lens.shape[0] != B:
        raise ValueError("block_table and seq_lens need one row per sequence")
    if sinks is not None:
        _need(sinks, "sinks", torch.float32, 1)
        if sinks.shape[0] != Hq:
            raise ValueError("sinks needs one logit per query head")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if workspace is None:
        nbytes = decode_window_workspace_bytes(B, Hq, Hkv, d, max_seq_len, block_size, int(window), int(n_sink))
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    _need_buf(workspace, "workspace")
    if out is None:
        out = torch.empty_like(q)
    _need_out(out, "out", torch.bfloat16, q.shape)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need_out(lse, "lse", torch.float32, (B, Hq))
    _need_buf(status, "status")
    rc = _lib.lib().attn_decode_paged_window(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                             _ptr(seq_lens), _ptr(sinks), _ptr(out), _ptr(lse), B, Hq, Hkv, d,
                                             num_blocks, block_size, block_table.shape[1], int(max_seq_len),
                                             int(window), int(n_sink), float(scale), _ptr(workspace),
                                             workspace.numel() * workspace.element_size(), _ptr(status),
                                             _stream_handle(stream))
    _lib.check(rc, "attn_decode_paged_window")
    return out, lse


def mla_decode_workspace_bytes(B: int, H: int, max_seq_len: int, d_latent: int = 512, d_rope: int = 64) -> int:
    n = int(_lib.lib().attn_mla_decode_workspace_bytes(B, H, d_latent, d_rope, max_seq_len))
    if n == 0:
        raise AttnError(_lib.ATTN_ERR_INVALID_ARG, "attn_mla_decode_workspace_bytes")
    return n


def mla_decode_paged(q, cache, block_table, seq_lens, max_seq_len: int, scale: float, d_latent: int = 512, out=None,
                     lse=None, workspace=None, status=None, stream=None, return_lse: bool = True):
    """Absorbed MLA decode: q [B, H, d_latent + d_rope] (absorbed content query,
    then positional query), cache [num_blocks, block_size, d_latent + d_rope]
    (latent, then positional key), both bf16. Returns the latent output
    O [B, H, d_latent] bf16 (apply the value up-projection afterwards) and
    LSE [B, H] fp32. `scale` is 1 / sqrt(d_head + d_rope).
    """
    _need(q, "q", torch.bfloat16, 3)
    _need(cache, "cache", torch.bfloat16, 3)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    B, H, width = q.shape
    num_blocks, block_size, width2 = cache.shape
    if width2 != width or width <= d_latent:
        raise ValueError("q and cache rows must both be d_latent + d_rope wide")
    if block_table.shape[0] != B or seq_lens.shape[0] != B:
        raise ValueError("block_table and seq_lens need one row per sequence")
    d_rope = width - d_latent
    if workspace is None:
        workspace = torch.empty(mla_decode_workspace_bytes(B, H, max_seq_len, d_latent, d_rope), dtype=torch.uint8,
                                device=q.device)
    _need_buf(workspace, "workspace")
    if out is None:
        out = torch.empty((B, H, d_latent), dtype=torch.bfloat16, device=q.device)
    _need_out(out, "out", torch.bfloat16, (B, H, d_latent))
    if lse is None and return_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need_out(lse, "lse", torch.float32, (B, H))
    _need_buf(status, "status")
    rc = _lib.lib().attn_mla_decode_paged(_ptr(q), _ptr(cache), _ptr(block_table), _ptr(seq_lens), _ptr(out), _ptr(lse),
                                          B, H, d_latent, d_rope, num_blocks, block_size, block_table.shape[1],
                                          int(max_seq_len), float(scale), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _ptr(status),
                                          _stream_handle(stream))
    _lib.check(rc, "attn_mla_decode_paged")
    return out, lse


def paged_gather(cache, block_table, seq_lens, max_seq_len: int, out=None, status=None, stream=None):
    """Contiguous [B, Hkv, max_seq_len, d] copy of a paged cache (zeros past seq_len)."""
    _need(cache, "cache", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    num_blocks, block_size, Hkv, d = cache.shape
    B = block_table.shape[0]
    if out is None:
        out = torch.empty((B, Hkv, max_seq_len, d), dtype=cache.dtype, device=cache.device)
    _need_out(out, "out", torch.bfloat16, (B, Hkv, max_seq_len, d))
    _need_buf(status, "status")
    rc = _lib.lib().attn_paged_gather(_ptr(cache), _ptr(block_table), _ptr(seq_lens), _ptr(out), B, Hkv, d,
                                      num_blocks, block_size, block_table.shape[1], int(max_seq_len), _ptr(status),
                                      _stream_handle(stream))
    _lib.check(rc, "attn_paged_gather")
    return out
