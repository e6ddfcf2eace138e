"""Seeded random shapes through every attention entry point, against the fp64
oracle, at the bar of every parity test (max-abs 1e-2, mean-abs 1e-3, LSE
1e-3).  The shapes are drawn once from fixed seeds, so a failure names a case
that reproduces: batch 1-3, 1-4 KV heads with 1, 2, 4 or 8 query heads each,
head dimension 64 or 128, causal or not, query and key lengths from 1 to a
few hundred (single-token rows through the cluster decode included), ragged
paged caches with shuffled block tables, chunked prefill and the FP8 cache."""
import math
import random

import numpy as np
import pytest
import torch

import oracle
from flash_attention_tiled_b200 import inputs

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS, LSE_ABS = 1e-2, 1e-3, 1e-3


@pytest.fixture(scope="module")
def frt():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from flash_attention_tiled_b200 import frt as f
    return f


def _compare(o_gpu, o_ref, lse_gpu, lse_ref, what):
    o = o_gpu.detach().float().cpu().double().numpy().reshape(o_ref.shape)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    err = np.abs(o - o_ref)
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3g}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs err {err.mean():.3g}"
    lg = lse_gpu.detach().cpu().double().numpy().reshape(lse_ref.shape)
    assert np.array_equal(np.isneginf(lg), np.isneginf(lse_ref)), f"{what}: -inf rows differ"
    fin = np.isfinite(lse_ref)
    if fin.any():
        assert np.abs(lg[fin] - lse_ref[fin]).max() <= LSE_ABS, f"{what}: lse err"


def _dense_cases(n, seed):
    rng = random.Random(seed)
    out = []
    for _ in range(n):
        Hkv = rng.randint(1, 4)
        g = rng.choice([1, 2, 4, 8])
        Sq = rng.choice([1, 1, rng.randint(2, 300), rng.randint(300, 600)])
        out.append((rng.randint(1, 3), Hkv * g, Hkv, Sq, rng.randint(1, 900),
                    rng.choice([64, 128]), rng.random() < 0.5))
    return out


@pytest.mark.parametrize("case", _dense_cases(20, 7), ids=str)
def test_fwd_random_shapes(frt, case):
    B, Hq, Hkv, Sq, Skv, D, causal = case
    x = inputs.dense(B, Hq, Hkv, Sq, Skv, D, seed=hash(case) % 100003)
    d = {k: v.cuda() for k, v in x.items()}
    scale = 1.0 / math.sqrt(D)
    o, lse = frt.attn_fwd(d["q"], d["k"], d["v"], causal=causal, scale=scale)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], causal, scale)
    _compare(o, o_ref, lse, lse_ref, str(case))
    assert frt.read_device_error() == 0


def _paged_cases(n, seed):
    rng = random.Random(seed)
    out = []
    for _ in range(n):
        Hkv = rng.randint(1, 4)
        g = rng.choice([1, 2, 4, 8, 16])
        B = rng.randint(1, 4)
        lens = [rng.choice([0, rng.randint(1, 40), rng.randint(40, 3000)]) for _ in range(B)]
        out.append((tuple(lens), Hkv * g, Hkv, rng.choice([64, 128]), rng.choice([0, 0, 3, 50])))
    return out


@pytest.mark.parametrize("case", _paged_cases(16, 11), ids=str)
def test_paged_decode_random_shapes(frt, case):
    lens, Hq, Hkv, D, splits = case
    x = inputs.paged(len(lens), Hq, Hkv, D, seq_lens=list(lens), seed=sum(lens) % 9973)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    scale = 1.0 / math.sqrt(D)
    o, lse = frt.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"],
                                   d["seq_lens"], scale=scale, num_splits=splits)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_decode_paged(x["q"], x["k_pages"], x["v_pages"],
                                              x["block_table"], x["seq_lens"], scale)
    _compare(o, o_ref, lse, lse_ref, str(case))
    if D == 128 and sum(lens) > 0:   # (the FP8 cache's per-head scales need some token)
        x8 = inputs.paged_fp8(len(lens), Hq, Hkv, D, seq_lens=list(lens), seed=sum(lens) % 9973)
        d8 = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x8.items()}
        o8, l8 = frt.attn_decode_paged_fp8(d8["q"], d8["k_pages"], d8["v_pages"], d8["k_scale"],
                                           d8["v_scale"], d8["block_table"], d8["seq_lens"],
                                           scale=scale, num_splits=splits)
        torch.cuda.synchronize()
        r8, rl8 = oracle.attn_decode_paged_fp8(x8["q"], x8["k_pages"], x8["v_pages"],
                                               x8["k_scale"], x8["v_scale"], x8["block_table"],
                                               x8["seq_lens"], scale)
        _compare(o8, r8, l8, rl8, "fp8 " + str(case))
    assert frt.read_device_error() == 0


def _chunk_cases(n, seed):
    rng = random.Random(seed)
    out = []
    for _ in range(n):
        Hkv = rng.randint(1, 3)
        B = rng.randint(1, 3)
        lens = [rng.randint(1, 1200) for _ in range(B)]
        qlens = [rng.randint(0, min(L, 300)) for L in lens]
        out.append((tuple(lens), tuple(qlens), Hkv * rng.choice([1, 2, 4]), Hkv,
                    rng.choice([64, 128]), rng.random() < 0.8))
    return out


@pytest.mark.parametrize("case", _chunk_cases(10, 13), ids=str)
def test_chunked_prefill_random_shapes(frt, case):
    lens, qlens, Hq, Hkv, D, causal = case
    B = len(lens)
    x = inputs.paged(B, Hq, Hkv, D, seq_lens=list(lens), seed=sum(lens) % 7919)
    max_q = max(max(qlens), 1)
    g = torch.Generator().manual_seed(sum(qlens) + 1)
    q = torch.randn(B, Hq, max_q, D, generator=g).to(torch.bfloat16)
    ql = torch.tensor(qlens, dtype=torch.int32)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    scale = 1.0 / math.sqrt(D)
    o, lse = frt.attn_prefill_paged(q.cuda(), d["k_pages"], d["v_pages"], d["block_table"],
                                    d["seq_lens"], ql.cuda(), causal=causal, scale=scale)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_prefill_paged(q, x["k_pages"], x["v_pages"], x["block_table"],
                                               x["seq_lens"], ql, causal, scale)
    _compare(o, o_ref, lse, lse_ref, str(case))
    assert frt.read_device_error() == 0
