"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Bar (all outputs are bf16 from fp32 accumulation): max |o - o_ref| <= 1e-2,
mean |o - o_ref| <= 1e-3, max |lse - lse_ref| <= 1e-3; index work (which
page, which slot) bit-exact.  The five named workloads run at full size and are
compared element by element, each with the launch configuration the
benchmark times.
"""
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


def _compare(o_gpu, o_ref, lse_gpu=None, lse_ref=None, what=""):
    o = o_gpu.detach().float().cpu().double().numpy().reshape(o_ref.shape)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    err = np.abs(o - o_ref)
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3g}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs err {err.mean():.3g}"
    if lse_gpu is not None:
        lg = lse_gpu.detach().cpu().double().numpy().reshape(lse_ref.shape)
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isneginf(lg), np.isneginf(lse_ref)), f"{what}: -inf rows differ"
        if fin.any():
            lerr = np.abs(lg[fin] - lse_ref[fin])
            assert lerr.max() <= LSE_ABS, f"{what}: lse err {lerr.max():.3g}"
    return err.max()


def _dev(x):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def _no_device_error(frt):
    assert frt.read_device_error() == 0


# ------------------------------------------------------------ named workloads
def test_tiny_causal(frt):
    w = inputs.WORKLOADS["tiny_causal"]
    x = inputs.make(w)
    d = _dev(x)
    o, lse = frt.attn_fwd(d["q"], d["k"], d["v"], causal=True, scale=w.scale)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], True, w.scale)
    _compare(o, o_ref, lse, lse_ref, "tiny_causal")
    # causal row 0 attends to key 0 alone: p = 1 exactly, so o = v[0] bit-exactly
    assert torch.equal(o[:, :, 0].cpu(), x["v"][:, :, 0])
    _no_device_error(frt)


@pytest.mark.parametrize("entry", ["attn_fwd", "attn_fwd_ws"])
def test_gqa_decode_contiguous(frt, entry):
    # attn_fwd: the cluster-merged decode (what the benchmark times);
    # attn_fwd_ws: the split-KV decode with a workspace and its merge kernel
    w = inputs.WORKLOADS["gqa_decode_4k"]
    x = inputs.make(w)
    d = _dev(x)
    o, lse = getattr(frt, entry)(d["q"], d["k"], d["v"], causal=False, scale=w.scale)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], False, w.scale)
    _compare(o, o_ref, lse, lse_ref, "gqa_decode_4k")
    _no_device_error(frt)


def test_llama3_prefill_full(frt):
    # every element of the 32 x 4096 x 128 output and every LSE of the launch
    # the benchmark times, against the oracle's full fp64 score matrices
    w = inputs.WORKLOADS["llama3_8b_prefill_4k"]
    x = inputs.make(w)
    d = _dev(x)
    o, lse = frt.attn_fwd(d["q"], d["k"], d["v"], causal=True, scale=w.scale)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], True, w.scale)
    _compare(o, o_ref, lse, lse_ref, "llama3 prefill (all rows)")
    # properties that hold at any size: row 0 of every head is v[0] exactly,
    # and every output lies in the convex hull of the values it attends
    kvh = torch.arange(w.Hq, device="cuda") // (w.Hq // w.Hkv)
    assert torch.equal(o[0, :, 0], d["v"][0, kvh, 0])
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    vmax = d["v"].float().abs().amax().item()
    assert o.float().abs().amax().item() <= vmax
    _no_device_error(frt)


def _paged_case(frt, x, scale, num_splits=0, what=""):
    d = _dev(x)
    o, lse = frt.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"],
                                   d["seq_lens"], scale=scale, num_splits=num_splits)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_decode_paged(x["q"], x["k_pages"], x["v_pages"],
                                              x["block_table"], x["seq_lens"], scale)
    _compare(o, o_ref, lse, lse_ref, what)
    return o, lse


def test_paged_gqa_decode(frt):
    w = inputs.WORKLOADS["paged_gqa_decode_b4"]
    _paged_case(frt, inputs.make(w), w.scale, what=w.name)
    _no_device_error(frt)


def test_long_splitkv_decode(frt):
    w = inputs.WORKLOADS["long_splitkv_decode_256k"]
    _paged_case(frt, inputs.make(w), w.scale, what=w.name)
    _no_device_error(frt)


# --------------------------------------------------------- prefill edge cases
PREFILL_CASES = [  # B, Hq, Hkv, Sq, Skv, D, causal
    (1, 2, 2, 128, 128, 64, False),
    (2, 4, 2, 200, 200, 128, True),     # ragged tail, GQA
    (1, 4, 1, 77, 333, 128, True),      # MQA, Sq < Skv (bottom-right)
    (1, 2, 2, 333, 77, 64, True),       # Sq > Skv: leading rows see no key
    (1, 2, 1, 256, 1000, 128, False),   # cross attention shape
    (2, 2, 2, 129, 129, 64, True),
    (1, 1, 1, 2, 1, 128, False),        # Skv = 1: o = v
    (1, 2, 2, 513, 513, 128, True),
]


@pytest.mark.parametrize("case", PREFILL_CASES, ids=str)
def test_prefill_edge(frt, case):
    B, Hq, Hkv, Sq, Skv, D, causal = case
    x = inputs.dense(B, Hq, Hkv, Sq, Skv, D, seed=sum(case) + 17)
    d = _dev(x)
    scale = 1.0 / math.sqrt(D)
    o, lse = frt.attn_fwd(d["q"], d["k"], d["v"], causal=causal, scale=scale)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], causal, scale)
    _compare(o, o_ref, lse, lse_ref, str(case))
    _no_device_error(frt)


def test_prefill_large_scores_rescale(frt):
    # scores spread over hundreds of log2 units force the lazy rescale path
    x = inputs.dense(1, 2, 2, 300, 300, 128, seed=5)
    x["q"] = (x["q"].float() * 6).to(torch.bfloat16)
    d = _dev(x)
    o, lse = frt.attn_fwd(d["q"], d["k"], d["v"], causal=True, scale=0.5)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], True, 0.5)
    _compare(o, o_ref, lse, lse_ref, "large scores")


def test_prefill_empty_keys(frt):
    x = inputs.dense(1, 2, 2, 5, 1, 64, seed=3)
    d = _dev(x)
    k0 = d["k"][:, :, :0].contiguous()
    v0 = d["v"][:, :, :0].contiguous()
    o = torch.full_like(d["q"], 7.0)
    o, lse = frt.attn_fwd(d["q"], k0, v0, causal=False, out=o)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_prefill_deterministic(frt):
    x = _dev(inputs.dense(1, 4, 2, 384, 384, 128, seed=9))
    o1, l1 = frt.attn_fwd(x["q"], x["k"], x["v"], causal=True)
    o2, l2 = frt.attn_fwd(x["q"], x["k"], x["v"], causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ---------------------------------------------------------- decode edge cases
DECODE_CASES = [  # lens, Hq, Hkv, D, num_splits
    ([1], 8, 8, 128, 0),
    ([15, 16, 17, 33], 8, 2, 128, 0),
    ([5000, 0, 300], 32, 4, 128, 0),      # an empty sequence
    ([4096], 32, 1, 128, 0),              # MQA, two head groups of 16
    ([1000, 2000], 16, 16, 64, 0),        # g = 1, D = 64
    ([3333, 77], 24, 2, 128, 1),          # one partition: no merge
    ([3333, 77], 24, 2, 128, 3),
    ([3333, 77], 24, 2, 128, 1000),       # more partitions than pages
]


@pytest.mark.parametrize("case", DECODE_CASES, ids=str)
def test_decode_edge(frt, case):
    lens, Hq, Hkv, D, splits = case
    x = inputs.paged(len(lens), Hq, Hkv, D, seq_lens=lens, seed=len(lens) * 31 + Hq)
    o, lse = _paged_case(frt, x, 1.0 / math.sqrt(D), splits, str(case))
    for b, n in enumerate(lens):
        if n == 0:
            assert torch.all(o[b] == 0) and torch.all(torch.isneginf(lse[b]))
    _no_device_error(frt)


@pytest.mark.parametrize("entry", ["attn_fwd", "attn_fwd_ws"])
def test_decode_contiguous_ragged(frt, entry):
    for Skv in (1, 7, 16, 100, 1025):
        x = inputs.dense(2, 8, 2, 1, Skv, 128, seed=Skv)
        d = _dev(x)
        o, lse = getattr(frt, entry)(d["q"], d["k"], d["v"])
        torch.cuda.synchronize()
        o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], False, 1 / math.sqrt(128))
        _compare(o, o_ref, lse, lse_ref, f"contiguous decode Skv={Skv}")


@pytest.mark.parametrize("t_star", [0, 15, 16, 17, 4095, 4096, 4099])
def test_decode_page_indexing_probe(frt, t_star):
    # all keys 0 except logical token t*, whose key makes p one-hot: the output
    # must be that token's value row bit-exactly (wrong page or slot -> wrong row)
    B, Hq, Hkv, D, n = 2, 8, 2, 128, 4100
    x = inputs.paged(B, Hq, Hkv, D, seq_lens=[n, n - 37], seed=t_star)
    q = torch.zeros_like(x["q"])
    q[:, :, 0] = 1.0
    kp = torch.zeros_like(x["k_pages"])
    for b in range(B):
        if t_star < int(x["seq_lens"][b]):
            phys = int(x["block_table"][b, t_star // 16])
            kp[phys, :, t_star % 16, 0] = 256.0   # score 256*scale' >> others
    x["q"], x["k_pages"] = q, kp
    d = _dev(x)
    o, _ = frt.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"],
                                 d["seq_lens"], scale=1.0)
    torch.cuda.synchronize()
    for b in range(B):
        if t_star >= int(x["seq_lens"][b]):
            continue
        phys = int(x["block_table"][b, t_star // 16])
        for h in range(Hq):
            assert torch.equal(o[b, h].cpu(), x["v_pages"][phys, h // (Hq // Hkv), t_star % 16])


def test_decode_deterministic(frt):
    x = _dev(inputs.paged(3, 16, 2, 128, seq_lens=[9000, 100, 20000], seed=4))
    args = (x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"])
    o1, l1 = frt.attn_decode_paged(*args)
    o2, l2 = frt.attn_decode_paged(*args)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_splits_agree(frt):
    # any partition of the keys merges to the same result (within fp32 rounding;
    # the LSE goes through the approximate exp2/log2 units, ~1e-5 relative)
    x = _dev(inputs.paged(2, 16, 2, 128, seq_lens=[7000, 3001], seed=8))
    args = (x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"])
    o1, l1 = frt.attn_decode_paged(*args, num_splits=1)
    for s in (2, 7, 148, 600):
        o2, l2 = frt.attn_decode_paged(*args, num_splits=s)
        torch.cuda.synchronize()
        assert (o1.float() - o2.float()).abs().max().item() <= 2 ** -7
        assert (l1 - l2).abs().max().item() <= 1e-4


# ------------------------------------------------------ FP8 (e4m3) KV cache
def test_fp8_conversion_matches_the_e4m3_definition(frt):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    y = frt.debug_fp8_decode(codes.cuda()).cpu()
    for c in range(256):
        ref = oracle.e4m3_to_f64(c)
        if math.isnan(ref):
            assert math.isnan(y[c].item()), c
        else:
            assert y[c].item() == ref, (c, y[c].item(), ref)


def _fp8_case(frt, x, scale, num_splits=0, what=""):
    d = _dev(x)
    o, lse = frt.attn_decode_paged_fp8(d["q"], d["k_pages"], d["v_pages"], d["k_scale"],
                                       d["v_scale"], d["block_table"], d["seq_lens"],
                                       scale=scale, num_splits=num_splits)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_decode_paged_fp8(x["q"], x["k_pages"], x["v_pages"],
                                                  x["k_scale"], x["v_scale"], x["block_table"],
                                                  x["seq_lens"], scale)
    _compare(o, o_ref, lse, lse_ref, what)
    return o, lse


@pytest.mark.parametrize("name", ["paged_gqa_decode_b4", "long_splitkv_decode_256k"])
def test_fp8_paged_decode_workloads(frt, name):
    # the named paged workloads with their cache stored as e4m3 (per-KV-head
    # power-of-two scales); NaN codes in the poison page and tail slots
    w = inputs.WORKLOADS[name]
    x = inputs.paged_fp8(w.B, w.Hq, w.Hkv, w.D, len_range=w.len_range, page_size=w.page_size,
                         seed=w.seed)
    _fp8_case(frt, x, w.scale, what=f"fp8 {name}")
    _no_device_error(frt)


FP8_CASES = [  # lens, Hq, Hkv, num_splits
    ([1], 8, 8, 0),
    ([15, 16, 17, 33], 8, 2, 0),
    ([5000, 0, 300], 32, 4, 0),           # an empty sequence
    ([4096], 32, 1, 0),                   # MQA, two head groups of 16
    ([3333, 77], 24, 2, 1),               # one partition: no merge
    ([3333, 77], 24, 2, 1000),            # more partitions than pages
]


@pytest.mark.parametrize("case", FP8_CASES, ids=str)
def test_fp8_decode_edge(frt, case):
    lens, Hq, Hkv, splits = case
    x = inputs.paged_fp8(len(lens), Hq, Hkv, 128, seq_lens=lens, seed=len(lens) * 17 + Hq)
    o, lse = _fp8_case(frt, x, 1.0 / math.sqrt(128), splits, f"fp8 {case}")
    for b, n in enumerate(lens):
        if n == 0:
            assert torch.all(o[b] == 0) and torch.all(torch.isneginf(lse[b]))
    _no_device_error(frt)


@pytest.mark.parametrize("t_star", [0, 17, 4095, 4099])
def test_fp8_decode_page_indexing_probe(frt, t_star):
    # keys 0 except token t*, whose key code is 448 on d 0: p is one-hot and o
    # must be that token's dequantised value row exactly
    B, Hq, Hkv, D, n = 2, 8, 2, 128, 4100
    x = inputs.paged_fp8(B, Hq, Hkv, D, seq_lens=[n, n - 37], seed=t_star)
    q = torch.zeros_like(x["q"])
    q[:, :, 0] = 1.0
    kp = torch.zeros_like(x["k_pages"])
    for b in range(B):
        if t_star < int(x["seq_lens"][b]):
            kp[int(x["block_table"][b, t_star // 16]), :, t_star % 16, 0] = 0x7E
    x["q"], x["k_pages"] = q, kp
    x["k_scale"] = torch.ones(Hkv)
    d = _dev(x)
    o, _ = frt.attn_decode_paged_fp8(d["q"], d["k_pages"], d["v_pages"], d["k_scale"],
                                     d["v_scale"], d["block_table"], d["seq_lens"], scale=1.0)
    torch.cuda.synchronize()
    for b in range(B):
        if t_star >= int(x["seq_lens"][b]):
            continue
        phys = int(x["block_table"][b, t_star // 16])
        for h in range(Hq):
            kvh = h // (Hq // Hkv)
            row = x["v_pages"][phys, kvh, t_star % 16].view(torch.float8_e4m3fn).float()
            ref = (row * x["v_scale"][kvh]).to(torch.bfloat16)
            assert torch.equal(o[b, h].cpu(), ref)


def test_fp8_decode_deterministic(frt):
    x = _dev(inputs.paged_fp8(3, 16, 2, 128, seq_lens=[9000, 100, 20000], seed=5))
    args = (x["q"], x["k_pages"], x["v_pages"], x["k_scale"], x["v_scale"], x["block_table"],
            x["seq_lens"])
    o1, l1 = frt.attn_decode_paged_fp8(*args)
    o2, l2 = frt.attn_decode_paged_fp8(*args)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("fp8", [False, True])
def test_decode_maximum_batch(frt, fp8):
    # the largest batch the decode plan holds (1024 sequences: 32 per lane of
    # the prefix scan), ragged lengths including a few empty sequences
    g = torch.Generator().manual_seed(41)
    lens = torch.randint(0, 40, (1024,), generator=g).tolist()
    make = inputs.paged_fp8 if fp8 else inputs.paged
    x = make(1024, 8, 2, 128, seq_lens=lens, seed=42)
    if fp8:
        o, lse = _fp8_case(frt, x, 1 / math.sqrt(128), what="fp8 B=1024")
    else:
        o, lse = _paged_case(frt, x, 1 / math.sqrt(128), what="B=1024")
    for b, n in enumerate(lens):
        if n == 0:
            assert torch.all(o[b] == 0) and torch.all(torch.isneginf(lse[b]))
    _no_device_error(frt)


def test_decode_workspace_shared_across_shapes(frt):
    # one workspace per stream serves calls of any shape: a small decode, a
    # larger one (the buffer grows; the old one is kept), the small one again
    s = torch.cuda.Stream()
    g = torch.Generator().manual_seed(50)
    big = torch.randint(0, 300, (40,), generator=g).tolist()   # 80 segments: a larger need
    sizes = []
    with torch.cuda.stream(s):
        for B, lens, seed in ((1, [40], 51), (40, big, 52), (1, [40], 53)):
            x = inputs.paged(B, 16, 2, 128, seq_lens=lens, seed=seed)
            _paged_case(frt, x, 1 / math.sqrt(128), what=f"B={B} on a shared workspace")
            keys = [k for k in frt._workspaces if k[1] == s.cuda_stream]
            assert len(keys) == 1
            sizes.append(frt._workspaces[keys[0]].numel())
    assert sizes[1] > sizes[0] and sizes[2] == sizes[1], sizes
    _no_device_error(frt)


def test_a_wait_nothing_ends_times_out_and_the_context_survives(frt):
    # failure detection without a fault: a wait on a barrier that nothing
    # arrives at gives up after its limit and reports it on the host
    import time
    lib = frt.lib()
    flags = ctypes.c_uint(0)
    torch.cuda.synchronize()
    assert lib.frt_read_device_error(ctypes.byref(flags)) == 0        # clear
    r = torch.zeros(4, dtype=torch.int32, device="cuda")
    t0 = time.time()
    assert lib.frt_debug_wait_timeout(ctypes.c_void_p(r.data_ptr()), None) == 0
    torch.cuda.synchronize()
    took = time.time() - t0
    assert r[0].item() == 2
    assert 1.0 < took < 60.0, took
    assert lib.frt_read_device_error(ctypes.byref(flags)) == 0 and (flags.value & 1)
    # the context still runs real work
    x = inputs.paged(1, 8, 2, 128, seq_lens=[100], seed=61)
    _paged_case(frt, x, 1 / math.sqrt(128), what="after a timed-out wait")
    _no_device_error(frt)


# ------------------------------------------------ binding argument checks
def test_binding_rejects_mismatched_tensors(frt):
    # wrong output shapes, dtypes or table sizes are refused before any kernel
    # could write or read outside a buffer
    x = _dev(inputs.dense(1, 4, 2, 64, 64, 64, seed=31))
    with pytest.raises(ValueError):
        frt.attn_fwd(x["q"], x["k"], x["v"], out=torch.empty(1, 4, 32, 64, dtype=torch.bfloat16,
                                                             device="cuda"))
    with pytest.raises(TypeError):
        frt.attn_fwd(x["q"], x["k"], x["v"], lse=torch.empty(1, 4, 64, dtype=torch.float16,
                                                             device="cuda"))
    with pytest.raises(ValueError):
        frt.attn_fwd(x["q"], x["k"], x["v"][:, :, :32].contiguous())
    p = _dev(inputs.paged(2, 8, 2, 128, seq_lens=[40, 50], seed=32))
    with pytest.raises(ValueError):
        frt.attn_decode_paged(p["q"], p["k_pages"], p["v_pages"], p["block_table"][:1],
                              p["seq_lens"])
    with pytest.raises(ValueError):
        frt.attn_decode_paged(p["q"], p["k_pages"], p["v_pages"], p["block_table"],
                              p["seq_lens"][:1])
    with pytest.raises(ValueError):
        frt.attn_decode_paged(p["q"], p["k_pages"], p["v_pages"], p["block_table"],
                              p["seq_lens"], lse=torch.empty(2, 4, device="cuda"))
    f = _dev(inputs.paged_fp8(2, 8, 2, 128, seq_lens=[40, 50], seed=33))
    with pytest.raises(ValueError):
        frt.attn_decode_paged_fp8(f["q"], f["k_pages"], f["v_pages"], f["k_scale"][:1],
                                  f["v_scale"], f["block_table"], f["seq_lens"])


# -------------------------------------------------- exact special cases
def test_single_visible_key_gives_v_exactly(frt):
    # one key: p = 1 and l = 1, so o is that key's value row, bit for bit
    x = inputs.dense(2, 4, 2, 3, 1, 128, seed=21)
    d = _dev(x)
    o, lse = frt.attn_fwd(d["q"], d["k"], d["v"], causal=False)          # tile kernel (Sq = 3)
    torch.cuda.synchronize()
    g = 4 // 2
    for h in range(4):
        assert torch.equal(o[:, h].cpu(), x["v"][:, h // g, :1].expand(-1, 3, -1))
    p = inputs.paged(3, 8, 2, 128, seq_lens=[1, 1, 1], seed=22)
    dp = _dev(p)
    o, _ = frt.attn_decode_paged(dp["q"], dp["k_pages"], dp["v_pages"], dp["block_table"],
                                 dp["seq_lens"])
    torch.cuda.synchronize()
    for b in range(3):
        phys = int(p["block_table"][b, 0])
        for h in range(8):
            assert torch.equal(o[b, h].cpu(), p["v_pages"][phys, h // 4, 0])


def test_gqa_equals_mha_with_repeated_kv_heads(frt):
    B, Hq, Hkv, S, D = 1, 8, 2, 300, 128
    x = inputs.dense(B, Hq, Hkv, S, S, D, seed=23)
    d = _dev(x)
    g = Hq // Hkv
    k_rep, v_rep = (t.repeat_interleave(g, dim=1).contiguous() for t in (d["k"], d["v"]))
    o1, l1 = frt.attn_fwd(d["q"], d["k"], d["v"], causal=True)
    o2, l2 = frt.attn_fwd(d["q"], k_rep, v_rep, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)        # same per-head arithmetic
    # decode: the head grouping changes the split plan, so compare within the bar
    q1 = d["q"][:, :, :1].contiguous()
    o1, l1 = frt.attn_fwd(q1, d["k"], d["v"])
    o2, l2 = frt.attn_fwd(q1, k_rep, v_rep)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= MAX_ABS
    assert (l1 - l2).abs().max().item() <= LSE_ABS


# --------------------------------------------------------- strided layouts
STRIDED_CASES = [  # B, Hq, Hkv, Sq, Skv, D, causal, fused
    (2, 4, 4, 300, 300, 128, True, "qkv"),     # fused [B,S,3,H,D] projection output, MHA
    (1, 8, 2, 257, 257, 64, True, "gqa"),      # fused [B,S,Hq+2Hkv,D], GQA
    (2, 4, 2, 130, 577, 128, False, "bshd"),   # cross attention, [B,S,H,D] tensors
    (3, 8, 2, 1, 999, 128, False, "bshd"),     # single-token rows, tile kernel
]


def _strided_inputs(case, seed):
    B, Hq, Hkv, Sq, Skv, D, causal, fused = case
    g = torch.Generator().manual_seed(seed)
    rnd = lambda *shape: torch.randn(*shape, generator=g).to(torch.bfloat16).cuda()
    if fused == "qkv":
        qkv = rnd(B, Sq, 3, Hq, D)
        q, k, v = (qkv[:, :, i].permute(0, 2, 1, 3) for i in range(3))
    elif fused == "gqa":
        x = rnd(B, Sq, Hq + 2 * Hkv, D)
        q = x[:, :, :Hq].permute(0, 2, 1, 3)
        k = x[:, :, Hq:Hq + Hkv].permute(0, 2, 1, 3)
        v = x[:, :, Hq + Hkv:].permute(0, 2, 1, 3)
    else:
        q = rnd(B, Sq, Hq, D).permute(0, 2, 1, 3)
        k = rnd(B, Skv, Hkv, D).permute(0, 2, 1, 3)
        v = rnd(B, Skv, Hkv, D).permute(0, 2, 1, 3)
    return q, k, v


@pytest.mark.parametrize("case", STRIDED_CASES, ids=str)
def test_strided_layouts(frt, case):
    B, Hq, Hkv, Sq, Skv, D, causal, fused = case
    q, k, v = _strided_inputs(case, seed=Sq + Skv)
    assert Sq == 1 or not q.is_contiguous()   # (a one-token view counts as contiguous)
    out_buf = torch.full((B, Sq, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = out_buf.permute(0, 2, 1, 3)                    # a strided output view
    o, lse = frt.attn_fwd_strided(q, k, v, causal=causal, out=out)
    torch.cuda.synchronize()
    qc, kc, vc = q.contiguous(), k.contiguous(), v.contiguous()
    o_ref, lse_ref = oracle.attn_fwd(qc.cpu(), kc.cpu(), vc.cpu(), causal, 1 / math.sqrt(D))
    _compare(out, o_ref, lse, lse_ref, f"strided {case}")
    if Sq > 1:
        # the same tile kernel on contiguous copies: bit-identical
        o2, l2 = frt.attn_fwd(qc, kc, vc, causal=causal)
        torch.cuda.synchronize()
        assert torch.equal(out.contiguous(), o2) and torch.equal(lse, l2)
    _no_device_error(frt)


# ------------------------------------------------------------------- merge
@pytest.mark.parametrize("S,B,Hq,D,empty", [(1, 2, 8, 128, 0.0), (5, 3, 16, 128, 0.3),
                                            (37, 1, 32, 128, 0.0), (4, 2, 4, 64, 0.5)])
def test_merge_lse(frt, S, B, Hq, D, empty):
    x = inputs.partials(S, B * Hq, D, seed=S * 100 + D, empty_frac=empty)
    op = x["o_parts"].reshape(S, B, Hq, D)
    lp = x["lse_parts"].reshape(S, B, Hq)
    o, lse = frt.merge_lse(op.cuda(), lp.cuda())
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.merge_lse(op.numpy(), lp.numpy())
    _compare(o, o_ref, lse, lse_ref, "merge")
    if S == 1:
        assert torch.equal(o.cpu(), op[0].to(torch.bfloat16))


def test_merge_all_empty_row(frt):
    op = torch.randn(3, 1, 2, 64)
    lp = torch.full((3, 1, 2), -math.inf)
    o, lse = frt.merge_lse(op.cuda(), lp.cuda())
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


# ------------------------------------------- chunked prefill over a paged cache
PAGED_PREFILL_CASES = [  # lens (context incl. chunk), q_lens, Hq, Hkv, D, causal
    ([300], [300], 4, 2, 128, True),                  # whole prompt through pages
    ([1000, 37, 4096], [200, 37, 129], 8, 2, 128, True),   # chunks after context
    ([513, 700], [1, 256], 4, 4, 64, True),           # D = 64, a one-token chunk
    ([900, 130], [300, 130], 4, 1, 128, False),       # non-causal, MQA
    ([2000], [640], 32, 8, 128, True),
]


@pytest.mark.parametrize("case", PAGED_PREFILL_CASES, ids=str)
def test_prefill_paged(frt, case):
    lens, qls, Hq, Hkv, D, causal = case
    x = inputs.paged(len(lens), Hq, Hkv, D, seq_lens=lens, seed=sum(lens) + Hq)
    max_q = max(qls)
    g = torch.Generator().manual_seed(7 + D)
    q = torch.randn(len(lens), Hq, max_q, D, generator=g).to(torch.bfloat16)
    for b, n in enumerate(qls):       # the padding rows hold NaN: they must not matter
        q[b, :, n:] = float("nan")
    ql = torch.tensor(qls, dtype=torch.int32)
    d = _dev(x)
    o, lse = frt.attn_prefill_paged(q.cuda(), d["k_pages"], d["v_pages"], d["block_table"],
                                    d["seq_lens"], ql.cuda(), causal=causal)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_prefill_paged(q, x["k_pages"], x["v_pages"], x["block_table"],
                                               x["seq_lens"], ql, causal, 1 / math.sqrt(D))
    _compare(o, o_ref, lse, lse_ref, str(case))
    _no_device_error(frt)


def test_prefill_paged_matches_contiguous_bitwise(frt):
    # the same sequence stored contiguously and in shuffled pages gives the same bits
    n, Hq, Hkv, D = 1000, 8, 2, 128
    x = inputs.paged(1, Hq, Hkv, D, seq_lens=[n], seed=77, poison=False)
    g = torch.Generator().manual_seed(3)
    q = torch.randn(1, Hq, n, D, generator=g).to(torch.bfloat16).cuda()
    d = _dev(x)
    pages = x["block_table"][0, : (n + 15) // 16].long()
    kc = x["k_pages"][pages].permute(1, 0, 2, 3).reshape(Hkv, -1, D)[:, :n][None].contiguous()
    vc = x["v_pages"][pages].permute(1, 0, 2, 3).reshape(Hkv, -1, D)[:, :n][None].contiguous()
    o1, l1 = frt.attn_fwd(q, kc.cuda(), vc.cuda(), causal=True)
    o2, l2 = frt.attn_prefill_paged(q, d["k_pages"], d["v_pages"], d["block_table"],
                                    d["seq_lens"], torch.tensor([n], dtype=torch.int32).cuda())
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
