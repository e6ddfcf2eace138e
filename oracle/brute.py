"""Brute-force attention by per-element Python loops -- TEST INFRASTRUCTURE ONLY.

A second, independent statement of the same definition as ``attn_oracle.c``,
arranged differently on purpose so that the two can pin each other on tiny
shapes: every output element is its own ratio

    o[b,h,i,d] = sum_j e^{s_ij} v[j,d] / sum_j e^{s_ij},   lse = log sum_j e^{s_ij}

over the visible keys j, with no running or subtracted maximum (inputs here are
tiny, so nothing overflows), exact summation (``math.fsum``), and, for the
paged cache, each key located through the block table at the moment it is
used instead of a gather into a contiguous copy.  Definition as on the
"Real-time inference optimisation" page (llmapi-app.pages.dev), section
"Flash Attention optimisation"; causal masking and GQA as listed on the
"FlashRT-HF-kernels" page (zingnex.cn), section "Attention optimisation".
Inputs are nested Python lists of floats (or anything indexable).
"""
from __future__ import annotations

import math


def _visible(i: int, j: int, Sq: int, Skv: int, causal: bool) -> bool:
    return (not causal) or (j - (Skv - Sq) <= i)


def attn_fwd(q, k, v, causal: bool, scale: float):
    """q[B][Hq][Sq][D], k/v[B][Hkv][Skv][D] -> (o[B][Hq][Sq][D], lse[B][Hq][Sq])."""
    B, Hq = len(q), len(q[0])
    Sq, D = len(q[0][0]), (len(q[0][0][0]) if len(q[0][0]) else 0)
    Hkv, Skv = len(k[0]), len(k[0][0])
    group = Hq // Hkv
    o = [[[[0.0] * D for _ in range(Sq)] for _ in range(Hq)] for _ in range(B)]
    lse = [[[-math.inf] * Sq for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            kvh = h // group
            for i in range(Sq):
                weights, keys = [], []
                for j in range(Skv):
                    if not _visible(i, j, Sq, Skv, causal):
                        continue
                    s = scale * math.fsum(q[b][h][i][d] * k[b][kvh][j][d] for d in range(D))
                    weights.append(math.exp(s))
                    keys.append(j)
                if not keys:
                    continue
                den = math.fsum(weights)
                for d in range(D):
                    num = math.fsum(w * v[b][kvh][j][d] for w, j in zip(weights, keys))
                    o[b][h][i][d] = num / den
                lse[b][h][i] = math.log(den)
    return o, lse


def attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, scale: float):
    """q[B][Hq][D]; k/v pages [P][Hkv][ps][D]; block_table[B][maxp]; seq_lens[B]."""
    B, Hq, D = len(q), len(q[0]), len(q[0][0])
    Hkv, ps = len(k_pages[0]), len(k_pages[0][0])
    group = Hq // Hkv
    o = [[[0.0] * D for _ in range(Hq)] for _ in range(B)]
    lse = [[-math.inf] * Hq for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            kvh = h // group
            weights, rows = [], []
            for t in range(seq_lens[b]):
                page = block_table[b][t // ps]
                key = k_pages[page][kvh][t % ps]
                s = scale * math.fsum(q[b][h][d] * key[d] for d in range(D))
                weights.append(math.exp(s))
                rows.append(v_pages[page][kvh][t % ps])
            if not rows:
                continue
            den = math.fsum(weights)
            for d in range(D):
                o[b][h][d] = math.fsum(w * r[d] for w, r in zip(weights, rows)) / den
            lse[b][h] = math.log(den)
    return o, lse


def attn_prefill_paged(q, k_pages, v_pages, block_table, seq_lens, q_lens, causal: bool,
                       scale: float):
    """q[B][Hq][max_q][D]; pages [P][Hkv][ps][D]; each sequence's last q_lens[b]
    tokens are the queries, bottom-right causal.  Padding rows: o = 0, lse = -inf."""
    B, Hq, max_q, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv, ps = len(k_pages[0]), len(k_pages[0][0])
    group = Hq // Hkv
    o = [[[[0.0] * D for _ in range(max_q)] for _ in range(Hq)] for _ in range(B)]
    lse = [[[-math.inf] * max_q for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        n, nq = seq_lens[b], q_lens[b]
        for h in range(Hq):
            kvh = h // group
            for i in range(nq):
                weights, rows = [], []
                for t in range(n):
                    if causal and t > i + (n - nq):
                        continue
                    page = block_table[b][t // ps]
                    key = k_pages[page][kvh][t % ps]
                    s = scale * math.fsum(q[b][h][i][d] * key[d] for d in range(D))
                    weights.append(math.exp(s))
                    rows.append(v_pages[page][kvh][t % ps])
                if not rows:
                    continue
                den = math.fsum(weights)
                for d in range(D):
                    o[b][h][i][d] = math.fsum(w * r[d] for w, r in zip(weights, rows)) / den
                lse[b][h][i] = math.log(den)
    return o, lse


def e4m3(code: int) -> float:
    """FP8 e4m3 ("fn": no infinities) code -> float, as an integer significand
    times a power of two: subnormals m * 2^-9, normals (8 + m) * 2^(e - 10),
    NaN for exponent 15 with mantissa 7."""
    sign = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 0xF, code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return sign * math.ldexp(m, -9)
    return sign * math.ldexp(8 + m, e - 10)


def attn_decode_paged_fp8(q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens,
                          scale: float):
    """As attn_decode_paged with e4m3 codes in the pages: the value of a cached
    element of KV head h is e4m3(code) * scale[h], decoded where it is used."""
    B, Hq, D = len(q), len(q[0]), len(q[0][0])
    Hkv, ps = len(k_pages[0]), len(k_pages[0][0])
    group = Hq // Hkv
    o = [[[0.0] * D for _ in range(Hq)] for _ in range(B)]
    lse = [[-math.inf] * Hq for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            kvh = h // group
            weights, rows = [], []
            for t in range(seq_lens[b]):
                page = block_table[b][t // ps]
                key = [e4m3(c) * k_scale[kvh] for c in k_pages[page][kvh][t % ps]]
                s = scale * math.fsum(q[b][h][d] * key[d] for d in range(D))
                weights.append(math.exp(s))
                rows.append([e4m3(c) * v_scale[kvh] for c in v_pages[page][kvh][t % ps]])
            if not rows:
                continue
            den = math.fsum(weights)
            for d in range(D):
                o[b][h][d] = math.fsum(w * r[d] for w, r in zip(weights, rows)) / den
            lse[b][h] = math.log(den)
    return o, lse
