"""The seeded input generators shared by the CUDA path and the oracle (CPU
only): they are deterministic, and the paged caches they build have the
structure the parity tests rely on -- every real page used once through the
block table, padding entries and tail slots poisoned with NaN."""
import math

import pytest
import torch

from flash_attention_tiled_b200 import inputs


def _same(a, b):
    return all(torch.equal(a[k], b[k]) if isinstance(a[k], torch.Tensor) else a[k] == b[k]
               for k in a)


def test_dense_is_seeded_bf16():
    a = inputs.dense(2, 4, 2, 5, 7, 64, seed=3)
    b = inputs.dense(2, 4, 2, 5, 7, 64, seed=3)
    c = inputs.dense(2, 4, 2, 5, 7, 64, seed=4)
    assert _same(a, b) and not torch.equal(a["q"], c["q"])
    assert a["q"].shape == (2, 4, 5, 64) and a["k"].shape == (2, 2, 7, 64)
    assert a["v"].shape == (2, 2, 7, 64)
    assert all(a[n].dtype == torch.bfloat16 for n in ("q", "k", "v"))


@pytest.mark.parametrize("lens,ps", [([13, 4, 9], 4), ([0, 33, 16, 1], 16), ([40], 16)])
def test_paged_block_table_uses_every_real_page_once(lens, ps):
    x = inputs.paged(len(lens), 8, 2, 32, seq_lens=lens, page_size=ps, seed=7)
    pages = [(n + ps - 1) // ps for n in lens]
    real = sum(pages)
    assert x["k_pages"].shape == (real + 1, 2, ps, 32) and x["poison_page"] == real
    bt = x["block_table"]
    assert bt.dtype == torch.int32 and bt.shape == (len(lens), max(1, max(pages)))
    used = torch.cat([bt[b, :n] for b, n in enumerate(pages)])
    assert sorted(used.tolist()) == list(range(real))          # a permutation of the real pages
    for b, n in enumerate(pages):
        assert torch.all(bt[b, n:] == real)                    # padding points at the poison page
    assert x["seq_lens"].tolist() == lens and x["seq_lens"].dtype == torch.int32


def test_paged_poison_and_tails_are_nan_real_slots_finite():
    lens, ps = [13, 4, 9, 0], 4
    x = inputs.paged(len(lens), 4, 2, 16, seq_lens=lens, page_size=ps, seed=8)
    for name in ("k_pages", "v_pages"):
        pg = x[name].float()
        assert torch.all(torch.isnan(pg[x["poison_page"]]))
        for b, n in enumerate(lens):
            for t in range(((n + ps - 1) // ps) * ps):
                phys = int(x["block_table"][b, t // ps])
                row = pg[phys, :, t % ps]
                assert torch.all(torch.isfinite(row)) if t < n else torch.all(torch.isnan(row))


def test_paged_is_seeded():
    a = inputs.paged(3, 8, 2, 32, seq_lens=[5, 17, 30], seed=11)
    b = inputs.paged(3, 8, 2, 32, seq_lens=[5, 17, 30], seed=11)
    c = inputs.paged(3, 8, 2, 32, seq_lens=[5, 17, 30], seed=12)
    eq = lambda t, u: torch.equal(torch.nan_to_num(t.float()), torch.nan_to_num(u.float()))
    assert all(eq(a[k], b[k]) for k in ("q", "k_pages", "v_pages", "block_table"))
    assert not eq(a["q"], c["q"]) and not torch.equal(a["block_table"], c["block_table"])


def test_paged_fp8_codes_round_trip_within_e4m3_precision():
    lens, ps, Hkv = [7, 9, 16], 4, 2
    x = inputs.paged_fp8(len(lens), 4, Hkv, 8, seq_lens=lens, page_size=ps, seed=13)
    ref = inputs.paged(len(lens), 4, Hkv, 8, seq_lens=lens, page_size=ps, seed=13, poison=False)
    assert torch.equal(x["q"], ref["q"]) and torch.equal(x["block_table"], ref["block_table"])
    for name, sname in (("k_pages", "k_scale"), ("v_pages", "v_scale")):
        sc = x[sname]
        assert sc.shape == (Hkv,) and sc.dtype == torch.float32
        assert all(math.log2(s) == int(math.log2(s)) for s in sc.tolist())   # powers of two
        codes = x[name]
        assert codes.dtype == torch.uint8
        vals = codes.view(torch.float8_e4m3fn).float() * sc.view(1, Hkv, 1, 1)
        real = ref[name].float()
        for b, n in enumerate(lens):
            for t in range(n):
                phys = int(x["block_table"][b, t // ps])
                got, want = vals[phys, :, t % ps], real[phys, :, t % ps]
                assert torch.all(torch.isfinite(got))
                # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 in the normal
                # range, absolute <= half the smallest subnormal step below it
                tol = torch.maximum(want.abs() * 2.0 ** -4, sc.view(Hkv, 1) * 2.0 ** -10)
                assert torch.all((got - want).abs() <= tol)
        assert torch.all(codes[x["poison_page"]] == inputs.E4M3_NAN)
        assert codes[: x["poison_page"]].view(torch.float8_e4m3fn).float().abs().nan_to_num(0).max() <= 448


def test_workload_recipes():
    w = inputs.WORKLOADS
    assert {n: w[n].seed for n in w} == {
        "tiny_causal": 1001, "gqa_decode_4k": 1002, "llama3_8b_prefill_4k": 1003,
        "paged_gqa_decode_b4": 1004, "long_splitkv_decode_256k": 1005}
    x = inputs.make("paged_gqa_decode_b4")
    lens = x["seq_lens"].tolist()
    assert len(lens) == 4 and all(1024 <= n <= 32768 for n in lens)
    assert x["page_size"] == 16 and x["q"].shape == (4, 64, 128)
    y = inputs.make("tiny_causal")
    assert y["q"].shape == (1, 2, 128, 64)


def test_partials_mark_empty_parts_with_minus_infinity():
    p = inputs.partials(5, 64, 32, seed=2, empty_frac=0.3)
    assert p["o_parts"].shape == (5, 64, 32) and p["lse_parts"].shape == (5, 64)
    empty = torch.isneginf(p["lse_parts"])
    assert 0 < int(empty.sum()) < 5 * 64
    assert torch.all(torch.isfinite(p["lse_parts"][~empty]))
