"""Python binding of libfrt_attn.so (argument marshalling only).

Every call hands raw device pointers, sizes and the current CUDA stream to
the C ABI declared in include/frt_attn.h; all of the attention arithmetic
runs in the library's CUDA kernels.  There is no fallback: if the library is
missing or a call is rejected, this module raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfrt_attn.so")

EXPORTS = ("frt_attn_fwd", "frt_attn_fwd_ws", "frt_attn_decode_paged",
           "frt_attn_decode_paged_noalloc", "frt_attn_prefill_paged", "frt_attn_decode_paged_fp8",
           "frt_attn_fwd_strided", "frt_attn_merge_lse", "frt_read_device_error",
           "frt_debug_fp8_decode", "frt_debug_wait_timeout", "frt_version")

STATUS = {0: "FRT_OK", 1: "FRT_ERR_INVALID_ARG", 2: "FRT_ERR_UNSUPPORTED",
          3: "FRT_ERR_WORKSPACE", 4: "FRT_ERR_CUDA"}


class FrtError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m flash_attention_tiled_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.POINTER(ctypes.c_size_t)
    lib.frt_attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, F, P]
    lib.frt_attn_fwd_ws.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, F, P, Z, P]
    lib.frt_attn_decode_paged.argtypes = [P, P, P, P, I, P, I, I, P, P, I, I, I, I, F, I, P, Z, P]
    lib.frt_attn_decode_paged_noalloc.argtypes = [P, P, P, P, I, P, I, I, P, P, I, I, I, I, F,
                                                  I, P]
    lib.frt_attn_merge_lse.argtypes = [P, P, I, I, I, I, P, P, P]
    lib.frt_attn_prefill_paged.argtypes = [P, P, P, P, I, P, P, I, I, P, P, I, I, I, I, I, I, F,
                                           P]
    lib.frt_read_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint)]
    lib.frt_attn_decode_paged_fp8.argtypes = [P, P, P, P, P, P, I, P, I, I, P, P, I, I, I, I, F, I,
                                              P, Z, P]
    lib.frt_debug_fp8_decode.argtypes = [P, P, I, P]
    lib.frt_debug_wait_timeout.argtypes = [P, P]
    lib.frt_attn_fwd_strided.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, F, P, P, P, P, P]
    for name in EXPORTS[:-1]:
        getattr(lib, name).restype = ctypes.c_int
    lib.frt_version.restype = ctypes.c_char_p
    return lib


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def version() -> str:
    return _lib.frt_version().decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(fn: str, rc: int):
    if rc != 0:
        raise FrtError(fn, rc)


def _need(t: torch.Tensor, name: str, dtype, ndim: int):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _shape(t: torch.Tensor, name: str, shape):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _out(t, name: str, dtype, shape, device, contiguous: bool = True):
    """A caller-supplied output: right dtype, shape and device (the kernels
    write exactly that many elements)."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    _shape(t, name, shape)
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, the inputs on {device}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _same_device(device, **tensors):
    for name, t in tensors.items():
        if t.device != device:
            raise ValueError(f"{name} is on {t.device}, q on {device}")


# Workspaces, one per (device, stream).  A call writes every word of the
# workspace it later reads, and each kernel first waits for the one before it
# in the stream, so one buffer serves every later call on the same stream,
# whatever its shape.  It grows in powers of two when a call needs more; an
# outgrown buffer is kept alive (a captured CUDA graph may still use it), so
# all buffers together hold less than twice the largest need.
#
# The key is the raw stream handle.  Streams from torch's pool are never
# destroyed, so there a handle always names the same stream.  Two cases are
# the caller's to order: an external stream destroyed and replaced by a new
# one with the same handle (synchronise the old one first), and a CUDA graph
# captured on stream A replayed on another stream while eager calls run on A
# (the graph holds A's buffer; order the replay after A's calls).
_workspaces: dict = {}
_retired: list = []


def workspace(nbytes: int, device, stream_handle: int) -> torch.Tensor:
    key = (torch.device(device).index, stream_handle)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        size = 256
        while size < nbytes:
            size *= 2
        if ws is not None:
            _retired.append(ws)
        ws = torch.zeros(size, dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def _fwd_args(q, k, v, causal, scale, out, lse, return_lse):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, 4)
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    _shape(k, "k", (B, Hkv, Skv, D))
    _shape(v, "v", k.shape)
    _same_device(q.device, k=k, v=v)
    _out(out, "out", torch.bfloat16, q.shape, q.device)
    _out(lse, "lse", torch.float32, (B, Hq, Sq), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    return (B, Hq, Hkv, Sq, Skv, D), scale, out, lse


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
             scale: float | None = None, out: torch.Tensor | None = None,
             lse: torch.Tensor | None = None, return_lse: bool = True):
    """o, lse = attention(q [B,Hq,Sq,D], k/v [B,Hkv,Skv,D]) with bf16 tensors
    (frt_attn_fwd: no workspace; Sq = 1 runs the cluster-merged decode)."""
    (B, Hq, Hkv, Sq, Skv, D), scale, out, lse = _fwd_args(q, k, v, causal, scale, out, lse,
                                                          return_lse)
    _check("frt_attn_fwd", _lib.frt_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B,
                                             Hq, Hkv, Sq, Skv, D, int(causal), scale,
                                             _stream(q.device)))
    return out, lse


def attn_fwd_ws(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                scale: float | None = None, out: torch.Tensor | None = None,
                lse: torch.Tensor | None = None, return_lse: bool = True):
    """attn_fwd through frt_attn_fwd_ws: Sq = 1 runs the split-KV decode with a
    workspace (from this module's per-stream buffers) and its merge kernel."""
    (B, Hq, Hkv, Sq, Skv, D), scale, out, lse = _fwd_args(q, k, v, causal, scale, out, lse,
                                                          return_lse)
    stream = _stream(q.device)
    need = ctypes.c_size_t(0)
    _check("frt_attn_fwd_ws", _lib.frt_attn_fwd_ws(None, None, None, None, None, B, Hq, Hkv, Sq,
                                                   Skv, D, int(causal), scale, None,
                                                   ctypes.byref(need), stream))
    ws = None
    if need.value > 0:
        ws = workspace(need.value, q.device, stream.value)
        need = ctypes.c_size_t(ws.numel())
    _check("frt_attn_fwd_ws", _lib.frt_attn_fwd_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                                   _ptr(lse), B, Hq, Hkv, Sq, Skv, D, int(causal),
                                                   scale, _ptr(ws), ctypes.byref(need), stream))
    return out, lse


def attn_decode_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                      block_table: torch.Tensor, seq_lens: torch.Tensor,
                      scale: float | None = None, num_splits: int = 0,
                      out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                      return_lse: bool = True):
    """o, lse = decode attention of q [B,Hq,D] over pages [P,Hkv,ps,D] (bf16)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_pages, "k_pages", torch.bfloat16, 4)
    _need(v_pages, "v_pages", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    B, Hq, D = q.shape
    P, Hkv, ps, _ = k_pages.shape
    _shape(k_pages, "k_pages", (P, Hkv, ps, D))
    _shape(v_pages, "v_pages", k_pages.shape)
    _shape(block_table, "block_table", (B, block_table.shape[1]))
    _shape(seq_lens, "seq_lens", (B,))
    _same_device(q.device, k_pages=k_pages, v_pages=v_pages, block_table=block_table,
                 seq_lens=seq_lens)
    _out(out, "out", torch.bfloat16, q.shape, q.device)
    _out(lse, "lse", torch.float32, (B, Hq), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    stream = _stream(q.device)
    need = ctypes.c_size_t(0)
    _check("frt_attn_decode_paged", _lib.frt_attn_decode_paged(
        None, None, None, None, block_table.shape[1], None, ps, P, None, None, B, Hq, Hkv, D,
        scale, num_splits, None, ctypes.byref(need), stream))
    ws = workspace(need.value, q.device, stream.value)
    need = ctypes.c_size_t(ws.numel())
    _check("frt_attn_decode_paged", _lib.frt_attn_decode_paged(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), block_table.shape[1],
        _ptr(seq_lens), ps, P, _ptr(out), _ptr(lse), B, Hq, Hkv, D, scale, num_splits,
        _ptr(ws), ctypes.byref(need), stream))
    return out, lse


def attn_decode_paged_fp8(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                          k_scale: torch.Tensor, v_scale: torch.Tensor,
                          block_table: torch.Tensor, seq_lens: torch.Tensor,
                          scale: float | None = None, num_splits: int = 0,
                          out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                          return_lse: bool = True):
    """o, lse = decode attention of q [B,Hq,D] (bf16) over an FP8 cache: pages
    [P,Hkv,ps,D] of e4m3 codes (uint8), KV head h's values = code * scale[h]
    with k_scale / v_scale [Hkv] fp32."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_pages, "k_pages", torch.uint8, 4)
    _need(v_pages, "v_pages", torch.uint8, 4)
    _need(k_scale, "k_scale", torch.float32, 1)
    _need(v_scale, "v_scale", torch.float32, 1)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    B, Hq, D = q.shape
    P, Hkv, ps, _ = k_pages.shape
    _shape(k_pages, "k_pages", (P, Hkv, ps, D))
    _shape(v_pages, "v_pages", k_pages.shape)
    _shape(k_scale, "k_scale", (Hkv,))
    _shape(v_scale, "v_scale", (Hkv,))
    _shape(block_table, "block_table", (B, block_table.shape[1]))
    _shape(seq_lens, "seq_lens", (B,))
    _same_device(q.device, k_pages=k_pages, v_pages=v_pages, k_scale=k_scale, v_scale=v_scale,
                 block_table=block_table, seq_lens=seq_lens)
    _out(out, "out", torch.bfloat16, q.shape, q.device)
    _out(lse, "lse", torch.float32, (B, Hq), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    stream = _stream(q.device)
    need = ctypes.c_size_t(0)
    _check("frt_attn_decode_paged_fp8", _lib.frt_attn_decode_paged_fp8(
        None, None, None, None, None, None, block_table.shape[1], None, ps, P, None, None, B, Hq,
        Hkv, D, scale, num_splits, None, ctypes.byref(need), stream))
    ws = workspace(need.value, q.device, stream.value)
    need = ctypes.c_size_t(ws.numel())
    _check("frt_attn_decode_paged_fp8", _lib.frt_attn_decode_paged_fp8(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(k_scale), _ptr(v_scale), _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), ps, P, _ptr(out), _ptr(lse), B, Hq, Hkv, D, scale,
        num_splits, _ptr(ws), ctypes.byref(need), stream))
    return out, lse


def _strides3(t: torch.Tensor, name: str):
    if t.dtype != torch.bfloat16 or t.dim() != 4:
        raise ValueError(f"{name} must be a 4-dim bf16 tensor [B, H, S, D]")
    if t.stride(3) != 1:
        raise ValueError(f"{name}: the last (head-dim) axis must be contiguous")
    return (ctypes.c_int64 * 3)(t.stride(0), t.stride(1), t.stride(2))


def attn_fwd_strided(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                     scale: float | None = None, out: torch.Tensor | None = None,
                     lse: torch.Tensor | None = None, return_lse: bool = True):
    """attn_fwd for views in any layout: q [B,Hq,Sq,D], k/v [B,Hkv,Skv,D] with
    any batch/head/token strides (multiples of 8 elements) and a contiguous
    last axis, e.g. views into a fused QKV tensor.  `out` may be a strided
    view too (default: a new contiguous [B,Hq,Sq,D])."""
    qs, ks, vs = _strides3(q, "q"), _strides3(k, "k"), _strides3(v, "v")
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    _shape(k, "k", (B, Hkv, Skv, D))
    _shape(v, "v", k.shape)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if not t.is_cuda:
            raise TypeError(f"{n} must be a CUDA tensor")
    _same_device(q.device, k=k, v=v)
    _out(out, "out", torch.bfloat16, (B, Hq, Sq, D), q.device, contiguous=False)
    _out(lse, "lse", torch.float32, (B, Hq, Sq), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty((B, Hq, Sq, D), dtype=q.dtype, device=q.device)
    os_ = _strides3(out, "out")
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    _check("frt_attn_fwd_strided", _lib.frt_attn_fwd_strided(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Skv, D, int(causal), scale,
        qs, ks, vs, os_, _stream(q.device)))
    return out, lse


def debug_fp8_decode(codes: torch.Tensor) -> torch.Tensor:
    """The FP8 decode kernel's conversion of e4m3 codes (uint8, on the device)."""
    _need(codes, "codes", torch.uint8, 1)
    y = torch.empty(codes.shape, dtype=torch.float32, device=codes.device)
    _check("frt_debug_fp8_decode", _lib.frt_debug_fp8_decode(
        _ptr(codes), _ptr(y), codes.numel(), _stream(codes.device)))
    return y


def attn_decode_paged_noalloc(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                              block_table: torch.Tensor, seq_lens: torch.Tensor,
                              scale: float | None = None, num_splits: int = 0,
                              out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                              return_lse: bool = True):
    """attn_decode_paged without a workspace: the library's fixed per-device
    scratch buffer is used instead (see frt_attn_decode_paged_noalloc in
    include/frt_attn.h for its size limit and the rule that calls which may
    overlap on the device race)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_pages, "k_pages", torch.bfloat16, 4)
    _need(v_pages, "v_pages", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    B, Hq, D = q.shape
    P, Hkv, ps, _ = k_pages.shape
    _shape(k_pages, "k_pages", (P, Hkv, ps, D))
    _shape(v_pages, "v_pages", k_pages.shape)
    _shape(block_table, "block_table", (B, block_table.shape[1]))
    _shape(seq_lens, "seq_lens", (B,))
    _same_device(q.device, k_pages=k_pages, v_pages=v_pages, block_table=block_table,
                 seq_lens=seq_lens)
    _out(out, "out", torch.bfloat16, q.shape, q.device)
    _out(lse, "lse", torch.float32, (B, Hq), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _check("frt_attn_decode_paged_noalloc", _lib.frt_attn_decode_paged_noalloc(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), block_table.shape[1],
        _ptr(seq_lens), ps, P, _ptr(out), _ptr(lse), B, Hq, Hkv, D, scale, num_splits,
        _stream(q.device)))
    return out, lse


def attn_prefill_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                       block_table: torch.Tensor, seq_lens: torch.Tensor, q_lens: torch.Tensor,
                       causal: bool = True, scale: float | None = None,
                       out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                       return_lse: bool = True):
    """o, lse = chunked prefill of q [B,Hq,max_q,D] over pages [P,Hkv,16,D]."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k_pages, "k_pages", torch.bfloat16, 4)
    _need(v_pages, "v_pages", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    _need(q_lens, "q_lens", torch.int32, 1)
    B, Hq, max_q, D = q.shape
    P, Hkv, ps, _ = k_pages.shape
    _shape(k_pages, "k_pages", (P, Hkv, ps, D))
    _shape(v_pages, "v_pages", k_pages.shape)
    _shape(block_table, "block_table", (B, block_table.shape[1]))
    _shape(seq_lens, "seq_lens", (B,))
    _shape(q_lens, "q_lens", (B,))
    _same_device(q.device, k_pages=k_pages, v_pages=v_pages, block_table=block_table,
                 seq_lens=seq_lens, q_lens=q_lens)
    _out(out, "out", torch.bfloat16, q.shape, q.device)
    _out(lse, "lse", torch.float32, (B, Hq, max_q), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, max_q), dtype=torch.float32, device=q.device)
    _check("frt_attn_prefill_paged", _lib.frt_attn_prefill_paged(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), block_table.shape[1],
        _ptr(seq_lens), _ptr(q_lens), ps, P, _ptr(out), _ptr(lse), B, Hq, Hkv, max_q, D,
        int(causal), scale, _stream(q.device)))
    return out, lse


def merge_lse(o_parts: torch.Tensor, lse_parts: torch.Tensor, out: torch.Tensor | None = None,
              lse: torch.Tensor | None = None, return_lse: bool = True):
    """o [B,Hq,D] bf16, lse [B,Hq] = merge of o_parts [S,B,Hq,D], lse_parts [S,B,Hq] (fp32)."""
    _need(o_parts, "o_parts", torch.float32, 4)
    _need(lse_parts, "lse_parts", torch.float32, 3)
    S, B, Hq, D = o_parts.shape
    _shape(lse_parts, "lse_parts", (S, B, Hq))
    _same_device(o_parts.device, lse_parts=lse_parts)
    _out(out, "out", torch.bfloat16, (B, Hq, D), o_parts.device)
    _out(lse, "lse", torch.float32, (B, Hq), o_parts.device)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=o_parts.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=o_parts.device)
    _check("frt_attn_merge_lse", _lib.frt_attn_merge_lse(
        _ptr(o_parts), _ptr(lse_parts), S, B, Hq, D, _ptr(out), _ptr(lse),
        _stream(o_parts.device)))
    return out, lse


def read_device_error() -> int:
    """Read and clear the library's device-side error word (synchronises)."""
    flags = ctypes.c_uint(0)
    _check("frt_read_device_error", _lib.frt_read_device_error(ctypes.byref(flags)))
    return flags.value
