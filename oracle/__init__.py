"""CPU oracle for fused attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The CUDA library never calls it and shares no
code with it.

``attn_oracle.c`` holds the fp64 definition (full score matrix, explicit
softmax); this module builds it with gcc, loads it with ctypes and converts
arrays.  ``brute.py`` holds an independent pure-Python loop used to pin the C
code on tiny shapes.

Every function takes bf16 tensors (``torch.bfloat16``; their bit patterns are
handed to C, which widens them exactly) and returns float64 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libattn_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into libattn_oracle.so (plain gcc, IEEE fp64, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        lib.oracle_attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, D]
        lib.oracle_attn_fwd_rows.argtypes = [P, P, P, I, I, I, I, I, I, I, D, I, P, P, P]
        lib.oracle_attn_decode_paged.argtypes = [P, P, P, P, I, P, I, I, P, P,
                                                 I, I, I, I, D, P]
        lib.oracle_merge_lse.argtypes = [P, P, I, I, I, P, P]
        lib.oracle_attn_prefill_paged.argtypes = [P, P, P, P, I, P, P, I, I, P, P, I, I, I, I,
                                                  I, I, D]
        lib.oracle_attn_decode_paged_fp8.argtypes = [P, P, P, P, P, P, I, P, I, I, P, P, I, I, I, I,
                                                     D, P]
        lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_f64.restype = D
        for f in (lib.oracle_attn_fwd, lib.oracle_attn_fwd_rows,
                  lib.oracle_attn_decode_paged, lib.oracle_merge_lse,
                  lib.oracle_attn_prefill_paged, lib.oracle_attn_decode_paged_fp8):
            f.restype = I
        _lib = lib
    return _lib


def _bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> contiguous uint16 numpy array of its bit patterns."""
    if t.dtype != torch.bfloat16:
        raise TypeError(f"oracle inputs are bf16, got {t.dtype}")
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _i32(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().numpy()
    return np.ascontiguousarray(t, dtype=np.int32)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"{what}: oracle rejected the arguments (code {rc})")


def attn_fwd(q, k, v, causal: bool, scale: float):
    """q [B,Hq,Sq,D], k/v [B,Hkv,Skv,D] bf16 -> (o [B,Hq,Sq,D], lse [B,Hq,Sq]) fp64."""
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    qa, ka, va = _bits(q), _bits(k), _bits(v)
    o = np.zeros((B, Hq, Sq, D), np.float64)
    lse = np.zeros((B, Hq, Sq), np.float64)
    rc = _load().oracle_attn_fwd(_ptr(qa), _ptr(ka), _ptr(va), _ptr(o), _ptr(lse),
                                 B, Hq, Hkv, Sq, Skv, D, int(bool(causal)), float(scale))
    _check(rc, "attn_fwd")
    return o, lse


def attn_fwd_rows(q, k, v, causal: bool, scale: float, rows):
    """Sampled rows; rows are flat indices (b*Hq + h)*Sq + i.
    Returns (o [n,D], lse [n]) fp64."""
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    qa, ka, va = _bits(q), _bits(k), _bits(v)
    o = np.zeros((len(rows), D), np.float64)
    lse = np.zeros((len(rows),), np.float64)
    rc = _load().oracle_attn_fwd_rows(_ptr(qa), _ptr(ka), _ptr(va), B, Hq, Hkv, Sq, Skv, D,
                                      int(bool(causal)), float(scale), len(rows), _ptr(rows),
                                      _ptr(o), _ptr(lse))
    _check(rc, "attn_fwd_rows")
    return o, lse


def attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, scale: float,
                      heads_mask=None):
    """q [B,Hq,D]; k/v pages [P,Hkv,ps,D]; block_table [B,maxp] int32; seq_lens [B].
    Returns (o [B,Hq,D], lse [B,Hq]) fp64.  heads_mask [B,Hq] (optional) selects
    the rows to compute; the others stay 0."""
    B, Hq, D = q.shape
    P, Hkv, ps, _ = k_pages.shape
    bt, sl = _i32(block_table), _i32(seq_lens)
    maxp = bt.shape[1] if bt.ndim == 2 else 0
    qa, ka, va = _bits(q), _bits(k_pages), _bits(v_pages)
    o = np.zeros((B, Hq, D), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    mask = None
    if heads_mask is not None:
        mask = np.ascontiguousarray(np.asarray(heads_mask, dtype=bool).reshape(B, Hq),
                                    dtype=np.uint8)
    rc = _load().oracle_attn_decode_paged(_ptr(qa), _ptr(ka), _ptr(va), _ptr(bt), maxp,
                                          _ptr(sl), ps, P, _ptr(o), _ptr(lse), B, Hq, Hkv,
                                          D, float(scale),
                                          None if mask is None else _ptr(mask))
    _check(rc, "attn_decode_paged")
    return o, lse


def attn_prefill_paged(q, k_pages, v_pages, block_table, seq_lens, q_lens, causal: bool,
                       scale: float):
    """Chunked prefill over a paged cache: q [B,Hq,max_q,D]; pages [P,Hkv,ps,D];
    block_table [B,maxp]; seq_lens [B] (context incl. the chunk); q_lens [B].
    Returns (o [B,Hq,max_q,D], lse [B,Hq,max_q]) fp64; padding rows o=0, lse=-inf."""
    B, Hq, max_q, D = q.shape
    P, Hkv, ps, _ = k_pages.shape
    bt, sl, ql = _i32(block_table), _i32(seq_lens), _i32(q_lens)
    maxp = bt.shape[1]
    qa, ka, va = _bits(q), _bits(k_pages), _bits(v_pages)
    o = np.zeros((B, Hq, max_q, D), np.float64)
    lse = np.zeros((B, Hq, max_q), np.float64)
    rc = _load().oracle_attn_prefill_paged(_ptr(qa), _ptr(ka), _ptr(va), _ptr(bt), maxp,
                                           _ptr(sl), _ptr(ql), ps, P, _ptr(o), _ptr(lse), B, Hq,
                                           Hkv, max_q, D, int(bool(causal)), float(scale))
    _check(rc, "attn_prefill_paged")
    return o, lse


def e4m3_to_f64(code: int) -> float:
    """The oracle's FP8 e4m3 decoder for one code (0..255)."""
    return float(_load().oracle_e4m3_to_f64(int(code)))


def attn_decode_paged_fp8(q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens,
                          scale: float, heads_mask=None):
    """q [B,Hq,D] bf16; k/v pages [P,Hkv,ps,D] uint8 e4m3 codes; k_scale/v_scale [Hkv]
    fp32 (KV head h's value = code * scale[h]); block_table [B,maxp]; seq_lens [B].
    Returns (o [B,Hq,D], lse [B,Hq]) fp64."""
    B, Hq, D = q.shape
    P, Hkv, ps, _ = k_pages.shape
    bt, sl = _i32(block_table), _i32(seq_lens)
    maxp = bt.shape[1] if bt.ndim == 2 else 0
    qa = _bits(q)
    ka = np.ascontiguousarray(k_pages.detach().cpu().numpy(), dtype=np.uint8)
    va = np.ascontiguousarray(v_pages.detach().cpu().numpy(), dtype=np.uint8)
    ks = np.ascontiguousarray(np.asarray(k_scale.detach().cpu() if isinstance(k_scale, torch.Tensor)
                                         else k_scale, dtype=np.float32))
    vs = np.ascontiguousarray(np.asarray(v_scale.detach().cpu() if isinstance(v_scale, torch.Tensor)
                                         else v_scale, dtype=np.float32))
    o = np.zeros((B, Hq, D), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    mask = None
    if heads_mask is not None:
        mask = np.ascontiguousarray(np.asarray(heads_mask, dtype=bool).reshape(B, Hq),
                                    dtype=np.uint8)
    rc = _load().oracle_attn_decode_paged_fp8(_ptr(qa), _ptr(ka), _ptr(va), _ptr(ks), _ptr(vs),
                                              _ptr(bt), maxp, _ptr(sl), ps, P, _ptr(o), _ptr(lse),
                                              B, Hq, Hkv, D, float(scale),
                                              None if mask is None else _ptr(mask))
    _check(rc, "attn_decode_paged_fp8")
    return o, lse


def merge_lse(o_parts, lse_parts):
    """o_parts [S,...,D], lse_parts [S,...] (any float) -> (o [...,D], lse [...]) fp64."""
    op = np.ascontiguousarray(np.asarray(o_parts, dtype=np.float64))
    lp = np.ascontiguousarray(np.asarray(lse_parts, dtype=np.float64))
    S, D = op.shape[0], op.shape[-1]
    rows_shape = lp.shape[1:]
    n = int(np.prod(rows_shape)) if rows_shape else 1
    o = np.zeros(rows_shape + (D,), np.float64)
    lse = np.zeros(rows_shape, np.float64)
    rc = _load().oracle_merge_lse(_ptr(op), _ptr(lp), S, n, D, _ptr(o), _ptr(lse))
    _check(rc, "merge_lse")
    return o, lse


def threads() -> int:
    """Threads the OpenMP oracle uses (OMP_NUM_THREADS, else the usable cores)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env and env.isdigit():
        return int(env)
    return len(os.sched_getaffinity(0))
