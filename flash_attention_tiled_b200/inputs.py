"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws random numbers and lays them out; it holds none of the
attention arithmetic, so both the CUDA path and the CPU oracle can be fed from
it without sharing any of the method.

Recipe (same for every workload): a CPU ``torch.Generator`` seeded with the
workload's seed draws, in this order, the sequence lengths (paged workloads
only), the physical-page permutation (paged only), then Q, K and V as fp32
N(0, 1), each rounded once to bf16 (round-to-nearest-even).  Paged caches get
one extra physical page filled with NaN that every unused block-table entry
points at, and the unused tail slots of each sequence's last page are NaN as
well, so a kernel that reads past a sequence's end poisons its output.
"""
from __future__ import annotations

import dataclasses
import math

import torch

PAGE_SIZE = 16


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Skv: int            # contiguous workloads: keys per sequence; paged: max length bound
    D: int
    causal: bool
    paged: bool
    seed: int
    len_range: tuple | None = None   # paged: inclusive Uniform[lo, hi] sequence lengths
    page_size: int = PAGE_SIZE

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


# The five workloads, in order: a tiny causal self-attention, a single-token GQA
# decode over a contiguous cache, a Llama-3-8B-shaped causal prefill, a paged
# GQA decode with mixed lengths, and a long-context paged split-KV decode.
WORKLOADS = {
    "tiny_causal": Workload("tiny_causal", 1, 2, 2, 128, 128, 64, True, False, 1001),
    "gqa_decode_4k": Workload("gqa_decode_4k", 1, 32, 8, 1, 4096, 128, False, False, 1002),
    "llama3_8b_prefill_4k": Workload("llama3_8b_prefill_4k", 1, 32, 8, 4096, 4096, 128,
                                     True, False, 1003),
    "paged_gqa_decode_b4": Workload("paged_gqa_decode_b4", 4, 64, 8, 1, 32768, 128, False,
                                    True, 1004, len_range=(1024, 32768)),
    "long_splitkv_decode_256k": Workload("long_splitkv_decode_256k", 1, 32, 4, 1, 262144,
                                         128, False, True, 1005,
                                         len_range=(262144, 262144)),
}


def _bf16_normal(shape, gen) -> torch.Tensor:
    return torch.randn(shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def dense(B, Hq, Hkv, Sq, Skv, D, seed) -> dict:
    """Contiguous Q [B,Hq,Sq,D], K and V [B,Hkv,Skv,D], bf16 on the CPU."""
    gen = torch.Generator("cpu").manual_seed(seed)
    q = _bf16_normal((B, Hq, Sq, D), gen)
    k = _bf16_normal((B, Hkv, Skv, D), gen)
    v = _bf16_normal((B, Hkv, Skv, D), gen)
    return {"q": q, "k": k, "v": v}


def paged(B, Hq, Hkv, D, seq_lens=None, len_range=None, page_size=PAGE_SIZE, seed=0,
          poison=True) -> dict:
    """A paged KV cache with a shuffled block table.

    Returns q [B,Hq,D], k_pages / v_pages [num_pages,Hkv,page_size,D] (bf16),
    block_table [B,max_pages] int32, seq_lens [B] int32 and the poison page id.
    Sequence b's logical page p lives in physical page block_table[b][p]; the
    real pages are consecutive chunks of one seeded permutation, and the last
    physical page (num_pages-1) is the NaN poison page.
    """
    gen = torch.Generator("cpu").manual_seed(seed)
    if seq_lens is None:
        lo, hi = len_range
        seq_lens = torch.randint(lo, hi + 1, (B,), generator=gen, dtype=torch.int64)
    seq_lens = torch.as_tensor(seq_lens, dtype=torch.int64).reshape(B)
    pages_per_seq = [(int(n) + page_size - 1) // page_size for n in seq_lens]
    real_pages = sum(pages_per_seq)
    num_pages = real_pages + 1
    poison_page = real_pages
    perm = torch.randperm(real_pages, generator=gen)
    max_pages = max(1, max(pages_per_seq) if pages_per_seq else 1)
    block_table = torch.full((B, max_pages), poison_page, dtype=torch.int32)
    start = 0
    for b, n in enumerate(pages_per_seq):
        block_table[b, :n] = perm[start:start + n].to(torch.int32)
        start += n
    q = _bf16_normal((B, Hq, D), gen)
    k_pages = _bf16_normal((num_pages, Hkv, page_size, D), gen)
    v_pages = _bf16_normal((num_pages, Hkv, page_size, D), gen)
    if poison:
        nan = float("nan")
        k_pages[poison_page] = nan
        v_pages[poison_page] = nan
        for b in range(B):
            n = int(seq_lens[b])
            tail = n % page_size
            if n > 0 and tail:
                last = int(block_table[b, pages_per_seq[b] - 1])
                k_pages[last, :, tail:, :] = nan
                v_pages[last, :, tail:, :] = nan
    return {"q": q, "k_pages": k_pages, "v_pages": v_pages, "block_table": block_table,
            "seq_lens": seq_lens.to(torch.int32), "poison_page": poison_page,
            "page_size": page_size}


# e4m3 code that is NaN (sign 0, exponent 15, mantissa 7)
E4M3_NAN = 0x7F
E4M3_MAX = 448.0


def paged_fp8(B, Hq, Hkv, D, seq_lens=None, len_range=None, page_size=PAGE_SIZE, seed=0,
              poison=True) -> dict:
    """A paged FP8 (e4m3) KV cache: the bf16 cache of `paged` with the same
    seed, stored per KV head as e4m3 codes of value / scale with a power-of-two
    scale (the smallest with |value| / scale <= 448 over that head's real
    tokens).  Returns the fields of `paged` with k_pages / v_pages as uint8
    codes, plus k_scale / v_scale [Hkv] fp32.  The poison page and the tail
    slots hold the NaN code."""
    x = paged(B, Hq, Hkv, D, seq_lens=seq_lens, len_range=len_range, page_size=page_size,
              seed=seed, poison=False)
    real = x["k_pages"].shape[0] - 1            # the last physical page is the poison page
    out = dict(x)
    for name, sname in (("k_pages", "k_scale"), ("v_pages", "v_scale")):
        t = x[name].float()
        amax = t[:real].abs().amax(dim=(0, 2, 3)).clamp_min(1e-30)          # [Hkv]
        sc = torch.exp2(torch.ceil(torch.log2(amax / E4M3_MAX)))
        codes = (t / sc.view(1, Hkv, 1, 1)).to(torch.float8_e4m3fn).view(torch.uint8)
        out[name] = codes.contiguous()
        out[sname] = sc.to(torch.float32)
    if poison:
        pp = x["poison_page"]
        for name in ("k_pages", "v_pages"):
            out[name][pp] = E4M3_NAN
        lens = x["seq_lens"]
        for b in range(B):
            n = int(lens[b])
            tail = n % page_size
            if n > 0 and tail:
                last = int(x["block_table"][b, (n + page_size - 1) // page_size - 1])
                out["k_pages"][last, :, tail:, :] = E4M3_NAN
                out["v_pages"][last, :, tail:, :] = E4M3_NAN
    return out


def make(workload: Workload | str) -> dict:
    """The seeded inputs of one named workload (CPU tensors)."""
    w = WORKLOADS[workload] if isinstance(workload, str) else workload
    if w.paged:
        return paged(w.B, w.Hq, w.Hkv, w.D, len_range=w.len_range, page_size=w.page_size,
                     seed=w.seed)
    return dense(w.B, w.Hq, w.Hkv, w.Sq, w.Skv, w.D, w.seed)


def partials(S, rows, D, seed, empty_frac=0.0) -> dict:
    """Random partial results for the log-sum-exp merge: o_parts [S,rows,D] fp32
    ~ N(0, 1/4) (a partial attention output is a convex combination of value
    rows, so it is smaller than one value row), lse_parts [S,rows] fp32
    ~ N(0, 4); a fraction of the parts is marked empty (lse = -inf)."""
    gen = torch.Generator("cpu").manual_seed(seed)
    o_parts = 0.5 * torch.randn((S, rows, D), generator=gen, dtype=torch.float32)
    lse_parts = 2.0 * torch.randn((S, rows), generator=gen, dtype=torch.float32)
    if empty_frac > 0:
        drop = torch.rand((S, rows), generator=gen) < empty_frac
        lse_parts[drop] = -math.inf
    return {"o_parts": o_parts, "lse_parts": lse_parts}
