"""The prefill kernel is persistent: one CTA per SM walks its share of the work
items (two 128-row query tiles of one KV head) in rounds, with barrier phases,
the K/V ring and tensor memory carried from item to item.  These cases aim at
that hand-over, against the fp64 oracle at the bar of every parity test:
item counts just below, at and above the number of SMs and at multiples of
it (CTAs with one, two and three items), items of different key-tile counts
in one CTA (causal GQA), row-pair items (odd heads per KV head), and chunked
prefills where many items have no query row at all (an item with no work
between two with work must still write its zeros and -inf LSEs and leave the
barrier phases of its CTA in step)."""
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


@pytest.fixture(scope="module")
def sms():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.cuda.get_device_properties(0).multi_processor_count


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


# items = B * (Hq / 2) * ceil(Sq / 128) with two query heads per KV head:
# one item per sequence below, so B sets the item count relative to the SMs
@pytest.mark.parametrize("delta", [-1, 0, 1, None, "2G+1", "3G-1"], ids=str)
@pytest.mark.parametrize("causal", [True, False])
def test_item_counts_around_the_sm_count(frt, sms, delta, causal):
    B = {None: sms // 2, "2G+1": 2 * sms + 1, "3G-1": 3 * sms - 1}.get(delta, None)
    if B is None:
        B = sms + delta
    Hq, Hkv, S, D = 2, 1, 100, 64
    x = inputs.dense(B, Hq, Hkv, S, S, D, seed=B * 3 + causal)
    d = {k: v.cuda() for k, v in x.items()}
    scale = 1.0 / math.sqrt(D)
    o, lse = frt.attn_fwd(d["q"], d["k"], d["v"], causal=causal, scale=scale)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], causal, scale)
    _compare(o, o_ref, lse, lse_ref, f"B{B} causal={causal}")
    assert frt.read_device_error() == 0


@pytest.mark.parametrize("case", [
    (3, 16, 4, 1100, 1100, 128),    # 216 items of 1-9 key tiles: CTAs with two of different sizes
    (2, 12, 4, 700, 900, 128),      # g = 3: row-pair items (256 rows), Sq < Skv
    (5, 8, 8, 520, 520, 64),        # MHA, D = 64
], ids=str)
def test_items_of_different_sizes_in_one_cta(frt, case):
    B, Hq, Hkv, Sq, Skv, D = case
    x = inputs.dense(B, Hq, Hkv, Sq, Skv, D, seed=sum(case))
    d = {k: v.cuda() for k, v in x.items()}
    scale = 1.0 / math.sqrt(D)
    o, lse = frt.attn_fwd(d["q"], d["k"], d["v"], causal=True, scale=scale)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], True, scale)
    _compare(o, o_ref, lse, lse_ref, str(case))
    assert frt.read_device_error() == 0


@pytest.mark.parametrize("seed", [1, 2])
def test_chunked_prefill_with_many_empty_items(frt, sms, seed):
    # more sequences than SMs, most with an empty chunk: every CTA meets items
    # with no work between items with work
    rng = random.Random(seed)
    B = 2 * sms + 3
    lens = [rng.randint(1, 300) for _ in range(B)]
    qls = [0 if rng.random() < 0.6 else rng.randint(1, min(L, 64)) for L in lens]
    qls[0] = max(qls[0], 1)
    Hq, Hkv, D = 4, 2, 64
    x = inputs.paged(B, Hq, Hkv, D, seq_lens=lens, seed=seed)
    max_q = max(qls)
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, max_q, D, generator=g).to(torch.bfloat16)
    for b, n in enumerate(qls):       # padding rows hold NaN: they must not matter
        q[b, :, n:] = float("nan")
    ql = torch.tensor(qls, dtype=torch.int32)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    o, lse = frt.attn_prefill_paged(q.cuda(), d["k_pages"], d["v_pages"], d["block_table"],
                                    d["seq_lens"], ql.cuda(), causal=True)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_prefill_paged(q, x["k_pages"], x["v_pages"], x["block_table"],
                                               x["seq_lens"], ql, True, 1 / math.sqrt(D))
    _compare(o, o_ref, lse, lse_ref, f"seed {seed}")
    assert frt.read_device_error() == 0
