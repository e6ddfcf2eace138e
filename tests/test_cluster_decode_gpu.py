"""Single-token decode through frt_attn_fwd (the 14-argument, workspace-free
call): the decode kernel in cluster mode, whose CTAs merge their partial
results through distributed shared memory.  Compared with the fp64 oracle
at the bar of every parity test (max-abs 1e-2, mean-abs 1e-3, LSE 1e-3), and
with the split-KV path that takes a workspace (frt_attn_fwd_ws)."""
import ctypes
import math

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
    assert np.abs(lg - lse_ref).max() <= LSE_ABS, f"{what}: lse err"


def _dev(x):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


CASES = [  # B, Hq, Hkv, Skv, D
    (1, 32, 8, 4096, 128),     # the 4k GQA decode: 8 clusters of 16 CTAs
    (2, 8, 2, 1, 128),         # one key: a cluster of one CTA
    (2, 8, 2, 7, 128),
    (2, 8, 2, 16, 128),
    (2, 8, 2, 100, 128),       # 7 pages: fewer pages than the largest cluster
    (2, 8, 2, 1025, 128),      # ragged last page
    (1, 32, 1, 4096, 128),     # MQA: two groups of 16 query heads per KV head
    (1, 24, 2, 333, 128),      # 12 heads per KV head (two head tiles, one part-filled)
    (3, 16, 16, 1000, 64),     # g = 1, D = 64
    (5, 40, 4, 777, 64),       # g = 10, D = 64
    (1, 64, 8, 2000, 128),     # g = 8
    (300, 8, 1, 50, 128),      # 300 segments: one CTA each, no merge
    (1100, 4, 2, 20, 64),      # more sequences than the split path's limit of 1024
]


@pytest.mark.parametrize("case", CASES, ids=str)
def test_cluster_decode_matches_oracle(frt, case):
    B, Hq, Hkv, Skv, D = case
    x = inputs.dense(B, Hq, Hkv, 1, Skv, D, seed=B * 7 + Hq + Skv)
    d = _dev(x)
    scale = 1.0 / math.sqrt(D)
    o, lse = frt.attn_fwd(d["q"], d["k"], d["v"], scale=scale)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], False, scale)
    _compare(o, o_ref, lse, lse_ref, str(case))
    assert frt.read_device_error() == 0


def test_cluster_decode_agrees_with_the_workspace_path(frt):
    x = _dev(inputs.make("gqa_decode_4k"))
    o1, l1 = frt.attn_fwd(x["q"], x["k"], x["v"])
    o2, l2 = frt.attn_fwd_ws(x["q"], x["k"], x["v"])
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 2 ** -7
    assert (l1 - l2).abs().max().item() <= 1e-4


def test_cluster_decode_deterministic(frt):
    x = _dev(inputs.dense(2, 32, 4, 1, 5000, 128, seed=11))
    o1, l1 = frt.attn_fwd(x["q"], x["k"], x["v"])
    o2, l2 = frt.attn_fwd(x["q"], x["k"], x["v"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("t_star", [0, 15, 16, 255, 256, 2047, 4095])
def test_cluster_decode_one_visible_key_gives_its_value_row(frt, t_star):
    # all keys 0 except token t*, whose key makes p one-hot in fp32: every CTA
    # of the cluster but the one holding t* carries weight 2^-369 = 0, so the
    # merged output is v[t*] bit-exactly (a wrong page or CTA share -> wrong row)
    B, Hq, Hkv, Skv, D = 1, 32, 8, 4096, 128
    x = inputs.dense(B, Hq, Hkv, 1, Skv, D, seed=t_star)
    q = torch.zeros_like(x["q"])
    q[..., 0] = 1.0
    k = torch.zeros_like(x["k"])
    k[:, :, t_star, 0] = 256.0
    d = _dev({"q": q, "k": k, "v": x["v"]})
    o, _ = frt.attn_fwd(d["q"], d["k"], d["v"], scale=1.0)
    torch.cuda.synchronize()
    kvh = torch.arange(Hq) // (Hq // Hkv)
    assert torch.equal(o[0, :, 0].cpu(), x["v"][0, kvh, t_star])


def test_fwd_called_with_exactly_the_fourteen_plugin_arguments(frt):
    # q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, causal, scale, stream -- raw
    # device pointers through the C ABI, for a decode row and a causal prefill
    for (Sq, Skv, causal) in ((1, 3000, 0), (300, 300, 1)):
        x = inputs.dense(1, 8, 2, Sq, Skv, 128, seed=Sq + Skv)
        d = _dev(x)
        o = torch.empty_like(d["q"])
        lse = torch.empty((1, 8, Sq), device="cuda")
        stream = torch.cuda.current_stream().cuda_stream
        rc = frt.lib().frt_attn_fwd(
            ctypes.c_void_p(d["q"].data_ptr()), ctypes.c_void_p(d["k"].data_ptr()),
            ctypes.c_void_p(d["v"].data_ptr()), ctypes.c_void_p(o.data_ptr()),
            ctypes.c_void_p(lse.data_ptr()), 1, 8, 2, Sq, Skv, 128, causal, 1 / math.sqrt(128),
            ctypes.c_void_p(stream))
        assert rc == 0
        torch.cuda.synchronize()
        o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], bool(causal), 1 / math.sqrt(128))
        _compare(o, o_ref, lse, lse_ref, f"C ABI Sq={Sq}")
