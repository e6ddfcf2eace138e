"""B200 (sm_100a) fused attention for low-batch inference.

The compute path is the CUDA library ``libfrt_attn.so`` (C ABI in
``include/frt_attn.h``); ``flash_attention_tiled_b200.frt`` is its thin
Python binding:

    from flash_attention_tiled_b200 import frt
    o, lse = frt.attn_fwd(q, k, v, causal=True)              # prefill / decode
    o, lse = frt.attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens)
    o, lse = frt.merge_lse(o_parts, lse_parts)

``flash_attention_tiled_b200.inputs`` holds the seeded synthetic workloads.
The binding is imported on first use so that the input generators can be
used without the CUDA library.
"""
import importlib

__all__ = ["frt", "inputs", "build"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
