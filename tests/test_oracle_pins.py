"""Pins of the CPU oracle against what the mathematics fixes (no GPU).

Each check is chosen so that a plausible slip in the oracle (a dropped or
misplaced scale, a wrong sign in the exponent, a transposed operand, an
off-by-one in the causal limit, the wrong KV head for a query head, a wrong
page or slot in the gather, a missing normaliser, log2 instead of ln in the
LSE, a merge that ignores the weights) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from flash_attention_tiled_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def _expr(s):
    if isinstance(s, (int, float)):
        return float(s)
    s = s.strip()
    if s in ("-inf", "inf", "nan"):
        return float(s)
    assert s.startswith("log(") and s.endswith(")"), s
    return math.log(float(s[4:-1]))


def _nested(x, f):
    return [_nested(e, f) for e in x] if isinstance(x, list) else f(x)


def _bf16(x):
    return torch.tensor(_nested(x, _expr), dtype=torch.float64).to(torch.bfloat16)


def _lists(t):
    return t.to(torch.float64).tolist()


def _rand(shape, seed, dist=1.0):
    g = torch.Generator().manual_seed(seed)
    return (dist * torch.randn(shape, generator=g)).to(torch.bfloat16)


# ---------------------------------------------------------------- golden cases
def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("case", _golden()["dense"], ids=lambda c: c["name"])
def test_golden_dense(case):
    q, k, v = _bf16(case["q"]), _bf16(case["k"]), _bf16(case["v"])
    scale = _expr(case["scale_expr"])
    o, lse = oracle.attn_fwd(q, k, v, case["causal"], scale)
    np.testing.assert_allclose(o, np.array(case["o"], dtype=np.float64), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, np.array(_nested(case["lse_expr"], _expr)), rtol=0,
                               atol=1e-12)
    ob, lb = brute.attn_fwd(_lists(q), _lists(k), _lists(v), case["causal"], scale)
    np.testing.assert_allclose(np.array(ob), np.array(case["o"], dtype=np.float64), atol=1e-12)
    np.testing.assert_allclose(np.array(lb), np.array(_nested(case["lse_expr"], _expr)),
                               atol=1e-12)


@pytest.mark.parametrize("case", _golden()["paged"], ids=lambda c: c["name"])
def test_golden_paged(case):
    q, kp, vp = _bf16(case["q"]), _bf16(case["k_pages"]), _bf16(case["v_pages"])
    bt = torch.tensor(case["block_table"], dtype=torch.int32)
    sl = torch.tensor(case["seq_lens"], dtype=torch.int32)
    scale = _expr(case["scale_expr"])
    o, lse = oracle.attn_decode_paged(q, kp, vp, bt, sl, scale)
    np.testing.assert_allclose(o, np.array(case["o"], dtype=np.float64), atol=1e-12)
    np.testing.assert_allclose(lse, np.array(_nested(case["lse_expr"], _expr)), atol=1e-12)
    ob, lb = brute.attn_decode_paged(_lists(q), _lists(kp), _lists(vp), bt.tolist(),
                                     sl.tolist(), scale)
    np.testing.assert_allclose(np.array(ob), np.array(case["o"], dtype=np.float64), atol=1e-12)


@pytest.mark.parametrize("case", _golden()["merge"], ids=lambda c: c["name"])
def test_golden_merge(case):
    o, lse = oracle.merge_lse(np.array(case["o_parts"], dtype=np.float64),
                              np.array(_nested(case["lse_parts_expr"], _expr)))
    np.testing.assert_allclose(o, np.array(case["o"], dtype=np.float64), atol=1e-12)
    np.testing.assert_allclose(lse, np.array(_nested(case["lse_expr"], _expr)), atol=1e-12)


# ------------------------------------------------------ brute force, tiny shapes
TINY = [  # B, Hq, Hkv, Sq, Skv, D, causal
    (1, 1, 1, 1, 1, 1, False),
    (1, 2, 2, 5, 5, 4, True),
    (2, 4, 2, 7, 7, 8, True),
    (1, 4, 1, 3, 9, 8, True),      # MQA, Sq < Skv (bottom-right)
    (2, 2, 1, 9, 4, 3, True),      # Sq > Skv: first rows see no key
    (1, 3, 3, 6, 17, 5, False),
    (2, 4, 4, 17, 17, 8, True),
]


@pytest.mark.parametrize("shape", TINY, ids=str)
def test_c_oracle_matches_brute_force(shape):
    B, Hq, Hkv, Sq, Skv, D, causal = shape
    q = _rand((B, Hq, Sq, D), 1)
    k = _rand((B, Hkv, Skv, D), 2)
    v = _rand((B, Hkv, Skv, D), 3)
    scale = 1.0 / math.sqrt(D)
    o, lse = oracle.attn_fwd(q, k, v, causal, scale)
    ob, lb = brute.attn_fwd(_lists(q), _lists(k), _lists(v), causal, scale)
    np.testing.assert_allclose(o, np.array(ob), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(np.array(lb)))
    fin = np.isfinite(lse)
    np.testing.assert_allclose(lse[fin], np.array(lb)[fin], rtol=0, atol=1e-12)
    # sampled rows agree with the full computation
    rows = np.arange(B * Hq * Sq)[::3]
    orow, lrow = oracle.attn_fwd_rows(q, k, v, causal, scale, rows)
    np.testing.assert_array_equal(orow, o.reshape(-1, D)[rows])
    np.testing.assert_array_equal(lrow, lse.reshape(-1)[rows])


@pytest.mark.parametrize("lens,Hq,Hkv,ps", [([5, 1, 12], 4, 2, 4), ([16, 9], 2, 1, 16),
                                            ([7], 3, 3, 2), ([0, 3], 2, 2, 4)])
def test_c_oracle_paged_matches_brute_force(lens, Hq, Hkv, ps):
    D = 6
    x = inputs.paged(len(lens), Hq, Hkv, D, seq_lens=lens, page_size=ps, seed=11)
    scale = 0.37
    o, lse = oracle.attn_decode_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"],
                                      x["seq_lens"], scale)
    ob, lb = brute.attn_decode_paged(_lists(x["q"]), _lists(x["k_pages"]),
                                     _lists(x["v_pages"]), x["block_table"].tolist(),
                                     x["seq_lens"].tolist(), scale)
    np.testing.assert_allclose(o, np.array(ob), rtol=0, atol=1e-12)
    lb = np.array(lb)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(lb))
    fin = np.isfinite(lb)
    np.testing.assert_allclose(lse[fin], lb[fin], atol=1e-12)
    assert np.isfinite(o).all()           # NaN poison never reached


# ---------------------------------------------------------------- closed forms
def test_single_key_returns_its_value():
    q, k, v = _rand((2, 4, 3, 8), 4), _rand((2, 2, 1, 8), 5), _rand((2, 2, 1, 8), 6)
    o, lse = oracle.attn_fwd(q, k, v, False, 0.3)
    vv = v.double().numpy()
    for h in range(4):
        np.testing.assert_array_equal(o[:, h], np.broadcast_to(vv[:, h // 2], o[:, h].shape))
    s = 0.3 * np.einsum("bhid,bhjd->bhij", q.double().numpy(),
                        np.repeat(k.double().numpy(), 2, axis=1))[..., 0]
    np.testing.assert_allclose(lse, s, atol=1e-12)


def test_identical_keys_average_visible_values():
    B, H, S, D = 1, 2, 9, 4
    q = _rand((B, H, S, D), 7)
    k = _rand((B, H, 1, D), 8).expand(B, H, S, D).contiguous()
    v = _rand((B, H, S, D), 9)
    vv = v.double().numpy()
    o, lse = oracle.attn_fwd(q, k, v, True, 0.5)
    s = 0.5 * np.einsum("bhid,bhd->bhi", q.double().numpy(), k[:, :, 0].double().numpy())
    for i in range(S):
        np.testing.assert_allclose(o[:, :, i], vv[:, :, : i + 1].mean(axis=2), atol=1e-12)
        np.testing.assert_allclose(lse[:, :, i], s[:, :, i] + math.log(i + 1), atol=1e-12)
    o2, _ = oracle.attn_fwd(q, k, v, False, 0.5)
    np.testing.assert_allclose(o2, np.broadcast_to(vv.mean(axis=2, keepdims=True), o2.shape),
                               atol=1e-12)


def test_causal_row0_is_first_value():
    q, k, v = _rand((1, 3, 6, 8), 10), _rand((1, 3, 6, 8), 11), _rand((1, 3, 6, 8), 12)
    o, lse = oracle.attn_fwd(q, k, v, True, 0.25)
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0].double().numpy())
    s00 = 0.25 * (q[:, :, 0].double() * k[:, :, 0].double()).sum(-1).numpy()
    np.testing.assert_allclose(lse[:, :, 0], s00, atol=1e-12)


def test_weights_sum_to_one():
    # with every value row equal to 1 the output is exactly sum_j p_ij = 1
    q, k = _rand((2, 4, 11, 8), 13, 3.0), _rand((2, 2, 11, 8), 14, 3.0)
    v = torch.ones((2, 2, 11, 8), dtype=torch.bfloat16)
    for causal in (False, True):
        o, _ = oracle.attn_fwd(q, k, v, causal, 0.35)
        np.testing.assert_allclose(o, 1.0, atol=1e-12)


def test_gqa_equals_mha_with_repeated_kv():
    g = 4
    q = _rand((2, 8, 5, 8), 15)
    k, v = _rand((2, 2, 7, 8), 16), _rand((2, 2, 7, 8), 17)
    o, lse = oracle.attn_fwd(q, k, v, True, 0.3)
    o2, lse2 = oracle.attn_fwd(q, k.repeat_interleave(g, 1), v.repeat_interleave(g, 1), True,
                               0.3)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)


def test_shift_invariance_and_lse_shift():
    # k_j + u for all j adds scale*q.u to every score of the row: o unchanged, lse shifted
    q = torch.tensor([[[[1.0, -2.0, 0.5, 0.0]]]], dtype=torch.bfloat16)
    gen = torch.Generator().manual_seed(18)
    k = (torch.randint(-8, 9, (1, 1, 6, 4), generator=gen) / 4.0).to(torch.bfloat16)
    v = _rand((1, 1, 6, 4), 19)
    u = torch.tensor([0.5, 0.25, 2.0, -3.0])
    k2 = (k.double() + u.double()).to(torch.bfloat16)
    assert torch.equal(k2.double(), k.double() + u.double())   # exact in bf16
    o, lse = oracle.attn_fwd(q, k, v, False, 0.7)
    o2, lse2 = oracle.attn_fwd(q, k2, v, False, 0.7)
    np.testing.assert_allclose(o2, o, atol=1e-12)
    np.testing.assert_allclose(lse2 - lse, 0.7 * float(q[0, 0, 0].double() @ u.double()),
                               atol=1e-12)


def test_noncausal_key_permutation_invariance():
    q, k, v = _rand((1, 2, 4, 8), 20), _rand((1, 2, 13, 8), 21), _rand((1, 2, 13, 8), 22)
    perm = torch.randperm(13, generator=torch.Generator().manual_seed(0))
    o, lse = oracle.attn_fwd(q, k, v, False, 0.3)
    o2, lse2 = oracle.attn_fwd(q, k[:, :, perm], v[:, :, perm], False, 0.3)
    np.testing.assert_allclose(o2, o, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, atol=1e-12)


def test_causal_prefix_is_shorter_attention():
    # row i of causal attention equals non-causal attention over keys 0..i
    q, k, v = _rand((1, 2, 8, 8), 23), _rand((1, 2, 8, 8), 24), _rand((1, 2, 8, 8), 25)
    o, lse = oracle.attn_fwd(q, k, v, True, 0.3)
    for i in range(8):
        oi, li = oracle.attn_fwd(q[:, :, i:i + 1], k[:, :, : i + 1], v[:, :, : i + 1], False,
                                 0.3)
        np.testing.assert_allclose(o[:, :, i:i + 1], oi, atol=1e-12)
        np.testing.assert_allclose(lse[:, :, i:i + 1], li, atol=1e-12)


def test_rows_without_visible_key():
    q, k, v = _rand((1, 1, 5, 4), 26), _rand((1, 1, 2, 4), 27), _rand((1, 1, 2, 4), 28)
    o, lse = oracle.attn_fwd(q, k, v, True, 1.0)   # offset -3: rows 0..2 see nothing
    assert np.all(o[0, 0, :3] == 0) and np.all(np.isneginf(lse[0, 0, :3]))
    assert np.all(np.isfinite(lse[0, 0, 3:]))


# ---------------------------------------------------------------------- paging
def test_paged_equals_contiguous_on_gathered_cache():
    B, Hq, Hkv, D, ps = 3, 4, 2, 8, 4
    x = inputs.paged(B, Hq, Hkv, D, seq_lens=[13, 4, 9], page_size=ps, seed=29)
    o, lse = oracle.attn_decode_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"],
                                      x["seq_lens"], 0.4)
    for b in range(B):
        n = int(x["seq_lens"][b])
        pages = x["block_table"][b, : (n + ps - 1) // ps].long()
        kc = x["k_pages"][pages].permute(1, 0, 2, 3).reshape(Hkv, -1, D)[:, :n]
        vc = x["v_pages"][pages].permute(1, 0, 2, 3).reshape(Hkv, -1, D)[:, :n]
        oc, lc = oracle.attn_fwd(x["q"][b][None, :, None], kc[None].contiguous(),
                                 vc[None].contiguous(), False, 0.4)
        np.testing.assert_array_equal(o[b], oc[0, :, 0])
        np.testing.assert_array_equal(lse[b], lc[0, :, 0])


@pytest.mark.parametrize("t_star", [0, 3, 4, 15, 16, 17, 29])
def test_paged_one_hot_probe(t_star):
    # all keys zero except logical position t*, where k = c*q: p is one-hot at t*
    B, Hq, Hkv, D, ps, n = 1, 1, 1, 4, 4, 30
    x = inputs.paged(B, Hq, Hkv, D, seq_lens=[n], page_size=ps, seed=30)
    q = torch.tensor([[[1.0, 2.0, -1.0, 0.5]]], dtype=torch.bfloat16)
    kp = torch.zeros_like(x["k_pages"])
    phys = int(x["block_table"][0, t_star // ps])
    kp[phys, 0, t_star % ps] = (64 * q[0, 0].double()).to(torch.bfloat16)
    o, _ = oracle.attn_decode_paged(q, kp, x["v_pages"], x["block_table"], x["seq_lens"], 1.0)
    np.testing.assert_allclose(o[0, 0], x["v_pages"][phys, 0, t_star % ps].double().numpy(),
                               rtol=0, atol=1e-30 + 1e-12)


# ----------------------------------------------------------------------- merge
def test_merge_of_key_partition_equals_full_attention():
    q, k, v = _rand((1, 4, 1, 8), 31), _rand((1, 2, 40, 8), 32), _rand((1, 2, 40, 8), 33)
    o, lse = oracle.attn_fwd(q, k, v, False, 0.3)
    bounds = [0, 7, 8, 23, 40]
    parts = [oracle.attn_fwd(q, k[:, :, a:b], v[:, :, a:b], False, 0.3)
             for a, b in zip(bounds[:-1], bounds[1:])]
    om, lm = oracle.merge_lse(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    np.testing.assert_allclose(om, o, atol=1e-12)
    np.testing.assert_allclose(lm, lse, atol=1e-12)
    # permuting the parts changes nothing; one part is the identity
    order = [2, 0, 3, 1]
    om2, lm2 = oracle.merge_lse(np.stack([parts[i][0] for i in order]),
                                np.stack([parts[i][1] for i in order]))
    np.testing.assert_allclose(om2, om, atol=1e-12)
    np.testing.assert_allclose(lm2, lm, atol=1e-12)
    o1, l1 = oracle.merge_lse(o[None], lse[None])
    np.testing.assert_allclose(o1, o, atol=1e-15)
    np.testing.assert_allclose(l1, lse, atol=1e-15)


def test_merge_all_empty_row():
    o, lse = oracle.merge_lse(np.ones((3, 2, 4)), np.full((3, 2), -np.inf))
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_oracle_rejects_bad_shapes():
    q = _rand((1, 3, 2, 4), 34)
    k = _rand((1, 2, 2, 4), 35)
    with pytest.raises(ValueError):
        oracle.attn_fwd(q, k, k, False, 0.5)      # Hq % Hkv != 0
    with pytest.raises(ValueError):
        oracle.attn_fwd(q, q, q, False, -1.0)     # scale <= 0


# ------------------------------------------------- chunked prefill, paged cache
def _chunk_case(lens, q_lens, Hq, Hkv, D, ps, seed):
    x = inputs.paged(len(lens), Hq, Hkv, D, seq_lens=lens, page_size=ps, seed=seed)
    max_q = max(q_lens)
    q = _rand((len(lens), Hq, max_q, D), seed + 1)
    return x, q, torch.tensor(q_lens, dtype=torch.int32)


@pytest.mark.parametrize("causal", [True, False])
def test_paged_prefill_matches_brute_force(causal):
    x, q, ql = _chunk_case([9, 5, 13], [4, 5, 1], 4, 2, 6, 4, 40)
    o, lse = oracle.attn_prefill_paged(q, x["k_pages"], x["v_pages"], x["block_table"],
                                       x["seq_lens"], ql, causal, 0.41)
    ob, lb = brute.attn_prefill_paged(_lists(q), _lists(x["k_pages"]), _lists(x["v_pages"]),
                                      x["block_table"].tolist(), x["seq_lens"].tolist(),
                                      ql.tolist(), causal, 0.41)
    np.testing.assert_allclose(o, np.array(ob), rtol=0, atol=1e-12)
    lb = np.array(lb)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(lb))
    fin = np.isfinite(lb)
    np.testing.assert_allclose(lse[fin], lb[fin], atol=1e-12)
    assert np.isfinite(o).all()


def test_paged_prefill_equals_contiguous_on_gathered_cache():
    ps, D, Hq, Hkv = 4, 8, 4, 2
    x, q, ql = _chunk_case([14, 7], [6, 7], Hq, Hkv, D, ps, 50)
    o, lse = oracle.attn_prefill_paged(q, x["k_pages"], x["v_pages"], x["block_table"],
                                       x["seq_lens"], ql, True, 0.3)
    for b in range(2):
        n, nq = int(x["seq_lens"][b]), int(ql[b])
        pages = x["block_table"][b, : (n + ps - 1) // ps].long()
        kc = x["k_pages"][pages].permute(1, 0, 2, 3).reshape(Hkv, -1, D)[:, :n]
        vc = x["v_pages"][pages].permute(1, 0, 2, 3).reshape(Hkv, -1, D)[:, :n]
        oc, lc = oracle.attn_fwd(q[b:b + 1, :, :nq].contiguous(), kc[None].contiguous(),
                                 vc[None].contiguous(), True, 0.3)
        np.testing.assert_array_equal(o[b, :, :nq], oc[0])
        np.testing.assert_array_equal(lse[b, :, :nq], lc[0])
        assert np.all(o[b, :, nq:] == 0) and np.all(np.isneginf(lse[b, :, nq:]))


def test_paged_prefill_of_one_token_is_decode():
    x, q, ql = _chunk_case([30, 17, 1], [1, 1, 1], 8, 2, 8, 16, 60)
    o, lse = oracle.attn_prefill_paged(q, x["k_pages"], x["v_pages"], x["block_table"],
                                       x["seq_lens"], ql, True, 0.25)
    od, ld = oracle.attn_decode_paged(q[:, :, 0].contiguous(), x["k_pages"], x["v_pages"],
                                      x["block_table"], x["seq_lens"], 0.25)
    np.testing.assert_array_equal(o[:, :, 0], od)
    np.testing.assert_array_equal(lse[:, :, 0], ld)


# ------------------------------------------------------------- FP8 KV cache
def _torch_e4m3(code: int) -> float:
    return torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).float().item()


def test_e4m3_decoder_matches_torch_for_every_code():
    for c in range(256):
        got, ref, br = oracle.e4m3_to_f64(c), _torch_e4m3(c), brute.e4m3(c)
        if math.isnan(ref):
            assert math.isnan(got) and math.isnan(br), c
        else:
            assert got == ref == br, (c, got, ref, br)
            assert math.copysign(1.0, got) == math.copysign(1.0, ref), c


@pytest.mark.parametrize("code,value", [(0x38, 1.0), (0x40, 2.0), (0x7E, 448.0), (0xFE, -448.0),
                                        (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9),
                                        (0x08, 2.0 ** -6), (0x3C, 1.5), (0xB8, -1.0)])
def test_e4m3_closed_forms(code, value):
    # e4m3: bias 7, 3 mantissa bits; 0x08 is the smallest normal, 0x7E the largest
    assert oracle.e4m3_to_f64(code) == value


def test_e4m3_nan_and_signed_zero():
    assert math.isnan(oracle.e4m3_to_f64(0x7F)) and math.isnan(oracle.e4m3_to_f64(0xFF))
    z = oracle.e4m3_to_f64(0x80)
    assert z == 0.0 and math.copysign(1.0, z) == -1.0


def _fp8_lists(x):
    return (x["q"].double().tolist(), x["k_pages"].tolist(), x["v_pages"].tolist(),
            x["block_table"].tolist(), x["seq_lens"].tolist())


def test_fp8_paged_decode_matches_brute_force():
    x = inputs.paged_fp8(2, 4, 2, 8, seq_lens=[7, 9], page_size=4, seed=11)
    # any scales, not only powers of two; the scales are fp32, so the brute
    # force gets the same fp32 values
    ks = torch.tensor([0.37, 1.9], dtype=torch.float32)
    vs = torch.tensor([0.61, 0.23], dtype=torch.float32)
    o, l = oracle.attn_decode_paged_fp8(x["q"], x["k_pages"], x["v_pages"], ks, vs,
                                        x["block_table"], x["seq_lens"], 0.35)
    ks, vs = ks.double().tolist(), vs.double().tolist()
    q, kp, vp, bt, sl = _fp8_lists(x)
    ob, lb = brute.attn_decode_paged_fp8(q, kp, vp, ks, vs, bt, sl, 0.35)
    assert np.allclose(o, np.array(ob), rtol=0, atol=1e-12)
    assert np.allclose(l, np.array(lb), rtol=0, atol=1e-12)
    assert np.isfinite(o).all()                  # NaN codes in the tails are never read


def test_fp8_paged_decode_equals_bf16_decode_on_the_dequantised_cache():
    # with power-of-two scales every dequantised value is exact in bf16, so the
    # FP8 path must reproduce the (separately pinned) bf16 oracle
    x = inputs.paged_fp8(3, 8, 2, 32, seq_lens=[40, 1, 23], page_size=16, seed=12)
    deq = {}
    for name, sname in (("k_pages", "k_scale"), ("v_pages", "v_scale")):
        vals = x[name].view(torch.float8_e4m3fn).double() * x[sname].double().view(1, -1, 1, 1)
        deq[name] = vals.to(torch.bfloat16)
        # exact (the NaN codes of the poison page and tail slots stay NaN)
        assert torch.allclose(deq[name].double(), vals, rtol=0, atol=0, equal_nan=True)
    o8, l8 = oracle.attn_decode_paged_fp8(x["q"], x["k_pages"], x["v_pages"], x["k_scale"],
                                          x["v_scale"], x["block_table"], x["seq_lens"], 0.2)
    ob, lb = oracle.attn_decode_paged(x["q"], deq["k_pages"], deq["v_pages"], x["block_table"],
                                      x["seq_lens"], 0.2)
    assert np.allclose(o8, ob, rtol=0, atol=1e-12)
    assert np.allclose(l8, lb, rtol=0, atol=1e-12)


def test_fp8_scale_enters_linearly():
    # doubling k_scale doubles every score; doubling v_scale doubles o and
    # leaves the LSE alone
    x = inputs.paged_fp8(1, 2, 1, 16, seq_lens=[19], page_size=16, seed=13)
    args = (x["block_table"], x["seq_lens"])
    ks, vs = x["k_scale"], x["v_scale"]
    o1, l1 = oracle.attn_decode_paged_fp8(x["q"], x["k_pages"], x["v_pages"], ks, vs, *args, 0.5)
    o2, l2 = oracle.attn_decode_paged_fp8(x["q"], x["k_pages"], x["v_pages"], ks * 2, vs, *args, 0.25)
    o3, l3 = oracle.attn_decode_paged_fp8(x["q"], x["k_pages"], x["v_pages"], ks, vs * 2, *args, 0.5)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)
    assert np.allclose(2 * o1, o3, atol=1e-12) and np.allclose(l1, l3, atol=1e-12)
