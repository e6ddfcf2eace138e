"""Block-table entries outside [0, num_pages).

The kernels check every entry a sequence uses before issuing its copy: an
out-of-range entry (negative, num_pages itself, or a value whose page-row
offset would wrap in 32-bit arithmetic) is never an address.  That page reads
as zeros and bit 2 of the device error word is set.  Expected results come
from the oracle on the same cache with one all-zero page appended and every
bad entry pointed at it; the other sequences must be unaffected."""
import math

import numpy as np
import pytest
import torch

import oracle
from flash_attention_tiled_b200 import inputs

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS, LSE_ABS = 1e-2, 1e-3, 1e-3
ERR_BAD_PAGE = 1 << 2


@pytest.fixture(scope="module")
def frt():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from flash_attention_tiled_b200 import frt as f
    f.read_device_error()   # start clean
    return f


def _compare(o_gpu, o_ref, lse_gpu, lse_ref, what):
    o = o_gpu.detach().float().cpu().double().numpy().reshape(o_ref.shape)
    fin_rows = np.isfinite(lse_ref)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    err = np.abs(o - o_ref)
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3g}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs err {err.mean():.3g}"
    lg = lse_gpu.detach().cpu().double().numpy().reshape(lse_ref.shape)
    assert np.array_equal(np.isneginf(lg), np.isneginf(lse_ref))
    assert np.abs(lg[fin_rows] - lse_ref[fin_rows]).max() <= LSE_ABS, f"{what}: lse"


def _corrupt(x, b, pages, num_pages):
    """Bad entries at the given logical pages of sequence b, and the oracle's
    view of them: the pool with one zero page appended, the entries pointing
    there."""
    bad = [-1, num_pages, 0x7FFFFFFF, 1 << 28, -(1 << 30)]
    bt = x["block_table"].clone()
    bt_ref = x["block_table"].clone()
    for i, pg in enumerate(pages):
        bt[b, pg] = bad[i % len(bad)]
        bt_ref[b, pg] = num_pages          # the appended zero page
    ref = dict(x)
    for key in ("k_pages", "v_pages"):
        ref[key] = torch.cat([x[key], torch.zeros_like(x[key][:1])])
    ref["block_table"] = bt_ref
    return bt, ref


def test_decode_bad_entries_read_zeros_and_are_reported(frt):
    lens = [700, 900, 333]
    x = inputs.paged(3, 16, 2, 128, seq_lens=lens, seed=21)
    P = x["k_pages"].shape[0]
    bt, ref = _corrupt(x, 1, [3, 10, 20, 40, 56], P)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    scale = 1 / math.sqrt(128)
    o, lse = frt.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], bt.cuda(), d["seq_lens"],
                                   scale=scale)
    torch.cuda.synchronize()
    assert frt.read_device_error() == ERR_BAD_PAGE
    o_ref, lse_ref = oracle.attn_decode_paged(ref["q"], ref["k_pages"], ref["v_pages"],
                                              ref["block_table"], ref["seq_lens"], scale)
    _compare(o, o_ref, lse, lse_ref, "decode with bad entries")
    # a clean call afterwards reports nothing
    frt.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"],
                          scale=scale)
    torch.cuda.synchronize()
    assert frt.read_device_error() == 0


def test_fp8_decode_bad_entries_read_zeros_and_are_reported(frt):
    lens = [500, 1200]
    x = inputs.paged_fp8(2, 16, 2, 128, seq_lens=lens, seed=22)
    P = x["k_pages"].shape[0]
    bt, ref = _corrupt(x, 0, [0, 7, 31], P)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    scale = 1 / math.sqrt(128)
    o, lse = frt.attn_decode_paged_fp8(d["q"], d["k_pages"], d["v_pages"], d["k_scale"],
                                       d["v_scale"], bt.cuda(), d["seq_lens"], scale=scale)
    torch.cuda.synchronize()
    assert frt.read_device_error() == ERR_BAD_PAGE
    o_ref, lse_ref = oracle.attn_decode_paged_fp8(ref["q"], ref["k_pages"], ref["v_pages"],
                                                  ref["k_scale"], ref["v_scale"],
                                                  ref["block_table"], ref["seq_lens"], scale)
    _compare(o, o_ref, lse, lse_ref, "fp8 decode with bad entries")


def test_chunked_prefill_bad_entries_read_zeros_and_are_reported(frt):
    B, Hq, Hkv, D = 2, 4, 2, 128
    lens, qlens = [300, 200], [100, 64]
    x = inputs.paged(B, Hq, Hkv, D, seq_lens=lens, seed=23)
    max_q = max(qlens)
    g = torch.Generator().manual_seed(5)
    q = torch.randn(B, Hq, max_q, D, generator=g).to(torch.bfloat16)
    ql = torch.tensor(qlens, dtype=torch.int32)
    P = x["k_pages"].shape[0]
    bt, ref = _corrupt(x, 0, [2, 15], P)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    o, lse = frt.attn_prefill_paged(q.cuda(), d["k_pages"], d["v_pages"], bt.cuda(),
                                    d["seq_lens"], ql.cuda(), causal=True, scale=0.1)
    torch.cuda.synchronize()
    assert frt.read_device_error() == ERR_BAD_PAGE
    o_ref, lse_ref = oracle.attn_prefill_paged(q, ref["k_pages"], ref["v_pages"],
                                               ref["block_table"], ref["seq_lens"], ql, True, 0.1)
    _compare(o, o_ref, lse, lse_ref, "chunked prefill with bad entries")
