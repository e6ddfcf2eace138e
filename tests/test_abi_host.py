"""Host-side checks of the C ABI (no GPU): the library loads, exports every
call that include/*.h declares, and rejects bad arguments before touching
the device."""
import ctypes
import glob
import os
import re

import pytest

from flash_attention_tiled_b200 import frt

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names += re.findall(r"FRT_API\s+[\w\s\*]*?\b(frt_\w+)\s*\(", text)
    return names


def test_every_declared_symbol_is_exported():
    declared = _declared()
    assert set(frt.EXPORTS) <= set(declared)
    for name in declared:
        assert hasattr(frt.lib(), name), name     # ctypes resolves it with dlsym


def test_version():
    assert re.fullmatch(r"\d+\.\d+\.\d+", frt.version())


NULL = None
Z = ctypes.c_size_t


def _fwd(B=1, Hq=2, Hkv=2, Sq=4, Skv=4, D=64, causal=0, scale=0.125, query=True):
    need = Z(0)
    return frt.lib().frt_attn_fwd_ws(NULL, NULL, NULL, NULL, NULL, B, Hq, Hkv, Sq, Skv, D, causal,
                                     scale, NULL, ctypes.byref(need), NULL), need.value


def _fwd14(q=NULL, k=NULL, v=NULL, o=NULL, lse=NULL, B=1, Hq=2, Hkv=2, Sq=4, Skv=4, D=64,
           causal=0, scale=0.125):
    return frt.lib().frt_attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, causal, scale, NULL)


def test_fwd_has_the_plugin_signature():
    # frt_attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, causal, scale, stream): the
    # plugin convention of the TensorRT analysis page, no workspace arguments
    text = open(os.path.join(ROOT, "include", "frt_attn.h")).read()
    m = re.search(r"FRT_API\s+frt_status\s+frt_attn_fwd\s*\(([^)]*)\)", text)
    params = [re.findall(r"(\w+)\s*$", p.strip())[0] for p in m.group(1).split(",")]
    assert params == ["q", "k", "v", "o", "lse", "B", "Hq", "Hkv", "Sq", "Skv", "D", "causal",
                      "scale", "stream"]
    assert len(frt.lib().frt_attn_fwd.argtypes) == 14


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=3, Hkv=2), 1),               # Hq % Hkv != 0
    (dict(Hkv=0), 1),
    (dict(B=-1), 1),
    (dict(Sq=-2), 1),
    (dict(causal=2), 1),
    (dict(scale=0.0), 1),
    (dict(scale=float("nan")), 1),
    (dict(scale=float("inf")), 1),
    (dict(D=96), 2),                      # head dim not built
    (dict(D=256), 2),
])
def test_fwd_rejects(kw, code):
    rc, _ = _fwd(**kw)
    assert rc == code
    assert _fwd14(**kw) == code      # the workspace-free entry checks the same


def test_fwd_prefill_needs_no_workspace():
    rc, need = _fwd(Sq=64, Skv=64)
    assert rc == 0 and need == 0


def _paged(B=1, Hq=8, Hkv=2, D=128, ps=16, num_pages=4, maxp=2, splits=0, scale=0.1):
    need = Z(0)
    return frt.lib().frt_attn_decode_paged(NULL, NULL, NULL, NULL, maxp, NULL, ps, num_pages,
                                           NULL, NULL, B, Hq, Hkv, D, scale, splits, NULL,
                                           ctypes.byref(need), NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=6, Hkv=4), 1), (dict(scale=-1.0), 1), (dict(splits=-1), 1), (dict(num_pages=-1), 1),
    (dict(maxp=-1), 1), (dict(D=80), 2), (dict(ps=8), 2), (dict(ps=32), 2), (dict(B=5000), 2),
])
def test_decode_rejects(kw, code):
    assert _paged(**kw) == code


def test_decode_workspace_query_with_explicit_splits():
    # with an explicit split count the size needs no device query
    need = Z(0)
    rc = frt.lib().frt_attn_decode_paged(NULL, NULL, NULL, NULL, 8, NULL, 16, 10, NULL, NULL, 2,
                                         64, 8, 128, 0.1, 37, NULL, ctypes.byref(need), NULL)
    assert rc == 0
    # partials for 37 + 16 slots of 16 rows x 128 fp32, their LSEs and a
    # piece range (two int32) per segment
    assert need.value >= (37 + 16) * 16 * 128 * 4 + (37 + 16) * 16 * 4 + 16 * 8


@pytest.mark.parametrize("S,B,Hq,D,code", [(0, 1, 1, 64, 1), (1, -1, 1, 64, 1), (2, 1, 0, 64, 1),
                                           (2, 1, 1, 32, 2)])
def test_merge_rejects(S, B, Hq, D, code):
    assert frt.lib().frt_attn_merge_lse(NULL, NULL, S, B, Hq, D, NULL, NULL, NULL) == code


def test_merge_empty_rows_is_a_noop():
    assert frt.lib().frt_attn_merge_lse(NULL, NULL, 3, 0, 4, 64, NULL, NULL, NULL) == 0


def _fp8(B=1, Hq=8, Hkv=2, D=128, page_size=16, scale=0.1, num_pages=10, splits=0,
         q=NULL, ks=NULL, vs=NULL):
    need = Z(0)
    fake = ctypes.c_void_p(256)            # aligned, never dereferenced: rejected first
    args = (q, fake if q else NULL, fake if q else NULL, ks, vs, fake if q else NULL, 4,
            fake if q else NULL, page_size, num_pages, fake if q else NULL, NULL, B, Hq, Hkv, D,
            scale, splits, NULL, ctypes.byref(need), NULL)
    return frt.lib().frt_attn_decode_paged_fp8(*args), need.value


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=3, Hkv=2), 1),
    (dict(D=64), 2),                      # the FP8 cache is built for D = 128
    (dict(page_size=8), 2),
    (dict(scale=0.0), 1),
    (dict(B=-1), 1),
    (dict(q=ctypes.c_void_p(256)), 1),    # a real call without scales
])
def test_decode_fp8_rejects(kw, code):
    rc, _ = _fp8(**kw)
    assert rc == code


def test_decode_fp8_workspace_query_matches_bf16():
    rc, need8 = _fp8(B=3, Hq=16, Hkv=4, splits=37)
    assert rc == 0
    need = Z(0)
    rc = frt.lib().frt_attn_decode_paged(NULL, NULL, NULL, NULL, 4, NULL, 16, 10, NULL, NULL, 3,
                                         16, 4, 128, 0.1, 37, NULL, ctypes.byref(need), NULL)
    assert rc == 0 and need.value == need8


def test_debug_fp8_decode_rejects():
    assert frt.lib().frt_debug_fp8_decode(NULL, NULL, -1, NULL) == 1
    assert frt.lib().frt_debug_fp8_decode(NULL, NULL, 0, NULL) == 0


def _strided(B=1, Hq=2, Hkv=2, Sq=4, Skv=4, D=64, causal=0, scale=0.125, qs=(512, 256, 64),
             ks=(512, 256, 64), vs=(512, 256, 64), os_=(512, 256, 64)):
    arr = lambda t: None if t is None else (ctypes.c_int64 * 3)(*t)
    return frt.lib().frt_attn_fwd_strided(NULL, NULL, NULL, NULL, NULL, B, Hq, Hkv, Sq, Skv, D,
                                          causal, scale, arr(qs), arr(ks), arr(vs), arr(os_), NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=3, Hkv=2), 1),
    (dict(D=96), 2),
    (dict(qs=(512, 256, 60)), 1),         # a token step that is not 16 bytes
    (dict(ks=(512, -256, 64)), 1),
    (dict(vs=(0, 256, 64)), 1),
    (dict(os_=None), 1),
    (dict(scale=-1.0), 1),
])
def test_fwd_strided_rejects(kw, code):
    assert _strided(**kw) == code


def test_fwd_strided_empty_is_a_noop():
    assert _strided(B=0) == 0 and _strided(Sq=0) == 0


# ------------------------------------------- real calls refused before launch
# Fake device addresses: these calls are rejected by the argument checks,
# which run before any CUDA call, so nothing is ever dereferenced.
A16 = ctypes.c_void_p(1 << 20)         # 16-byte aligned
ODD = ctypes.c_void_p((1 << 20) + 2)   # 2-byte aligned only


def _fwd_call(q=A16, k=A16, v=A16, o=A16, lse=NULL, B=1, Hq=2, Hkv=2, Sq=4, Skv=4, D=64):
    need = Z(0)
    rc = frt.lib().frt_attn_fwd_ws(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, 0, 0.125, NULL,
                                   ctypes.byref(need), NULL)
    rc14 = _fwd14(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D)
    assert rc14 == rc, (rc14, rc)
    return rc


@pytest.mark.parametrize("kw,code", [
    (dict(o=NULL), 1),
    (dict(k=NULL), 1),
    (dict(q=ODD), 1),
    (dict(o=ODD), 1),
    (dict(v=ODD), 1),
    (dict(lse=ODD), 1),
    (dict(Sq=1, q=ODD), 1),                     # the decode path checks the same
    (dict(Sq=1, o=NULL), 1),
    (dict(B=1 << 16, Hq=1 << 8, Hkv=1 << 8, Sq=1 << 8, Skv=1), 2),   # 2^32 query rows
])
def test_fwd_real_call_rejects(kw, code):
    assert _fwd_call(**kw) == code


def test_fwd_real_call_with_nothing_to_do():
    assert _fwd_call(B=0) == 0 and _fwd_call(Sq=0) == 0


def _paged_call(q=A16, kp=A16, vp=A16, bt=A16, sl=A16, o=A16, lse=NULL, B=1, Hq=8, Hkv=2,
                num_pages=4, maxp=2):
    need = Z(1 << 30)
    return frt.lib().frt_attn_decode_paged(q, kp, vp, bt, maxp, sl, 16, num_pages, o, lse, B, Hq,
                                           Hkv, 128, 0.1, 4, A16, ctypes.byref(need), NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(kp=NULL), 1),
    (dict(sl=NULL), 1),
    (dict(o=NULL), 1),
    (dict(bt=NULL), 1),
    (dict(bt=ctypes.c_void_p((1 << 20) + 2)), 1),   # int32 table not 4-byte aligned
    (dict(sl=ctypes.c_void_p((1 << 20) + 1)), 1),
    (dict(q=ODD), 1),
    (dict(lse=ODD), 1),
    (dict(num_pages=0), 1),
    (dict(num_pages=1 << 27, Hkv=2), 2),            # 2^32 cache rows
])
def test_decode_real_call_rejects(kw, code):
    assert _paged_call(**kw) == code


def _prefill_paged(q=A16, kp=A16, vp=A16, bt=A16, sl=A16, ql=A16, o=A16, lse=NULL, B=1, Hq=4,
                   Hkv=2, max_q=8, D=128, ps=16, num_pages=4, maxp=2, causal=1, scale=0.1):
    return frt.lib().frt_attn_prefill_paged(q, kp, vp, bt, maxp, sl, ql, ps, num_pages, o, lse,
                                            B, Hq, Hkv, max_q, D, causal, scale, NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=3), 1),
    (dict(max_q=-1), 1),
    (dict(causal=2), 1),
    (dict(scale=0.0), 1),
    (dict(maxp=-1), 1),
    (dict(D=80), 2),
    (dict(ps=32), 2),
    (dict(num_pages=1 << 27), 2),
    (dict(q=NULL), 1),
    (dict(ql=NULL), 1),
    (dict(bt=NULL), 1),
    (dict(maxp=0), 1),
    (dict(num_pages=0), 1),
    (dict(kp=ODD), 1),
    (dict(ql=ctypes.c_void_p((1 << 20) + 2)), 1),
])
def test_prefill_paged_rejects(kw, code):
    assert _prefill_paged(**kw) == code


def test_prefill_paged_with_nothing_to_do():
    assert _prefill_paged(B=0) == 0 and _prefill_paged(max_q=0) == 0


def test_noalloc_refuses_a_plan_larger_than_its_scratch():
    # 4000 parts of 16 rows x 128 fp32 partials do not fit the 16 MiB scratch:
    # refused with FRT_ERR_WORKSPACE before anything runs
    rc = frt.lib().frt_attn_decode_paged_noalloc(A16, A16, A16, A16, 2, A16, 16, 4, A16, NULL, 1,
                                                 8, 2, 128, 0.1, 4000, NULL)
    assert rc == 3


def test_noalloc_argument_checks():
    lib = frt.lib()
    assert lib.frt_attn_decode_paged_noalloc(A16, A16, A16, A16, 2, A16, 8, 4, A16, NULL, 1, 8, 2,
                                             128, 0.1, 4, NULL) == 2      # page size 8
    assert lib.frt_attn_decode_paged_noalloc(NULL, A16, A16, A16, 2, A16, 16, 4, A16, NULL, 1, 8,
                                             2, 128, 0.1, 4, NULL) == 1   # no q
    assert lib.frt_attn_decode_paged_noalloc(NULL, NULL, NULL, NULL, 2, NULL, 16, 4, NULL, NULL,
                                             0, 8, 2, 128, 0.1, 4, NULL) == 0   # empty batch


def test_merge_real_call_rejects_misaligned():
    lib = frt.lib()
    assert lib.frt_attn_merge_lse(ODD, A16, 2, 1, 4, 64, A16, NULL, NULL) == 1
    assert lib.frt_attn_merge_lse(A16, A16, 2, 1, 4, 64, ODD, NULL, NULL) == 1
    assert lib.frt_attn_merge_lse(A16, ctypes.c_void_p((1 << 20) + 1), 2, 1, 4, 64, A16, NULL,
                                  NULL) == 1
    assert lib.frt_attn_merge_lse(NULL, A16, 2, 1, 4, 64, A16, NULL, NULL) == 1


def test_diagnostic_entries_check_their_arguments():
    lib = frt.lib()
    assert lib.frt_read_device_error(None) == 1


def test_page_count_limits_are_checked():
    # B * max_pages_per_seq >= 2^31 (paged decode, bf16 and FP8) and
    # max_pages_per_seq * 16 >= 2^31 (chunked prefill) are refused
    assert _paged_call(B=1024, maxp=1 << 21) == 2
    need = Z(0)
    assert frt.lib().frt_attn_decode_paged_fp8(NULL, NULL, NULL, NULL, NULL, NULL, 1 << 21, NULL, 16,
                                               10, NULL, NULL, 1024, 8, 2, 128, 0.1, 4, NULL,
                                               ctypes.byref(need), NULL) == 2
    assert _prefill_paged(maxp=1 << 27) == 2
    # a sequence's token bound max_pages_per_seq * 16 >= 2^31 (paged decode)
    assert _paged_call(B=1, maxp=1 << 27) == 2
    assert frt.lib().frt_attn_decode_paged_fp8(NULL, NULL, NULL, NULL, NULL, NULL, 1 << 27, NULL, 16,
                                               10, NULL, NULL, 1, 8, 2, 128, 0.1, 4, NULL,
                                               ctypes.byref(need), NULL) == 2
