"""frt_attn_decode_paged_noalloc: the decode call for callers that cannot
allocate device memory (plugins handed fixed buffers, real-time loops that
must not call cudaMalloc mid-run).  It uses the library's fixed per-device
scratch buffer instead of a caller workspace.

Checked through the C ABI against frt_attn_decode_paged (the same kernel with
a caller-provided workspace), within the parity tolerance of the other GPU
tests, on two calls in a row: the first call looks up the buffer, the second
finds it holding the first call's leftovers and must still be right.  This
file sorts last so that a run stopping at the first failure has run every
other test already; it also passes on its own in a fresh process.
"""
import ctypes
import math

import pytest
import torch

from flash_attention_tiled_b200 import inputs

pytestmark = pytest.mark.gpu

MAX_ABS, LSE_ABS = 1e-2, 1e-3


@pytest.fixture(scope="module")
def frt():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from flash_attention_tiled_b200 import frt as f
    return f


def _noalloc_call(frt, d, out, lse, num_splits=0):
    B, Hq, D = d["q"].shape
    P, Hkv, ps, _ = d["k_pages"].shape
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return frt.lib().frt_attn_decode_paged_noalloc(
        p(d["q"]), p(d["k_pages"]), p(d["v_pages"]), p(d["block_table"]),
        d["block_table"].shape[1], p(d["seq_lens"]), ps, P, p(out), p(lse), B, Hq, Hkv, D,
        1.0 / math.sqrt(D), num_splits,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _close(a, b):
    return (a.float() - b.float()).abs().max().item()


def test_noalloc_matches_workspace_decode_twice(frt):
    cases = [
        inputs.paged(4, 64, 8, 128, seq_lens=[3000, 17, 9001, 1024], seed=41),
        inputs.paged(2, 32, 4, 128, seq_lens=[20000, 5], seed=42),   # other shape, reused buffer
    ]
    for x in cases:
        d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
        o_ref, l_ref = frt.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"],
                                             d["block_table"], d["seq_lens"])
        for _ in range(2):
            o = torch.full_like(d["q"], float("nan"))
            lse = torch.full_like(l_ref, float("nan"))
            assert _noalloc_call(frt, d, o, lse) == 0
            torch.cuda.synchronize()
            assert torch.isfinite(o).all() and torch.isfinite(lse).all()
            assert _close(o, o_ref) <= MAX_ABS
            assert _close(lse, l_ref) <= LSE_ABS
    assert frt.read_device_error() == 0


def test_noalloc_rejects_problems_beyond_its_buffer(frt):
    # 1024 sequences x 8 KV heads at D = 128 with 4096 partitions needs far
    # more than the fixed 16 MiB: rejected with FRT_ERR_WORKSPACE, nothing runs
    need = ctypes.c_size_t(0)
    rc = frt.lib().frt_attn_decode_paged(None, None, None, None, 1, None, 16, 1, None, None,
                                         1024, 64, 8, 128, 0.1, 4096, None, ctypes.byref(need),
                                         None)
    assert rc == 0 and need.value > (16 << 20)
    x = inputs.paged(1, 8, 8, 128, seq_lens=[16], seed=1)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    q = torch.zeros(1024, 64, 128, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty(1024, 64, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    bt = torch.zeros(1024, 1, dtype=torch.int32, device="cuda")
    sl = torch.ones(1024, dtype=torch.int32, device="cuda")
    P = d["k_pages"].shape[0]
    rc = frt.lib().frt_attn_decode_paged_noalloc(
        p(q), p(d["k_pages"]), p(d["v_pages"]), p(bt), 1, p(sl), 16, P, p(o), p(lse), 1024, 64,
        8, 128, 0.1, 4096, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 3   # FRT_ERR_WORKSPACE
