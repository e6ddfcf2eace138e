"""The oracle's pins reject plausible slips (CPU only).

Each case plants one mistake in a copy of ``oracle/attn_oracle.c`` (a wrong
causal limit or alignment, a dropped scale, exp2 for exp, a missing softmax
normaliser, a wrong LSE, a transposed or reversed operand, the wrong KV head
for a query head, a wrong slot or KV head in the page gather, a wrong e4m3
exponent bias, a lost FP8 scale, a merge without its weights), builds the copy
into a temporary library, points the oracle's wrapper at it and runs the pins
of ``test_oracle_pins.py`` until one fails.  A slip that no pin notices would
mean the pins do not fix that part of the definition.  Every substitution
keeps all memory accesses in bounds, so a planted copy can only compute wrong
numbers.  The real oracle is not touched.
"""
import inspect
import itertools

import pytest

import oracle
import test_oracle_pins as pins

# (name, exact text in attn_oracle.c, replacement); each text occurs once
MUTATIONS = [
    ("causal limit off by one",
     "int visible = !causal || ((long long)j <= (long long)i + offset);",
     "int visible = !causal || ((long long)j < (long long)i + offset);"),
    ("top-left causal alignment",
     "const long long offset = (long long)Skv - (long long)Sq;",
     "const long long offset = 0;"),
    ("scale dropped", "srow[j] = scale * dot;", "srow[j] = dot;"),
    ("exp2 instead of exp",
     "double p = (srow[j] == -INFINITY) ? 0.0 : exp(srow[j] - m);",
     "double p = (srow[j] == -INFINITY) ? 0.0 : exp2(srow[j] - m);"),
    ("softmax normaliser missing", "double w = srow[j] / l;", "double w = srow[j];"),
    ("LSE without the row max", "lseh[i - i0] = m + log(l);", "lseh[i - i0] = log(l);"),
    ("LSE in log2", "lseh[i - i0] = m + log(l);", "lseh[i - i0] = m + log2(l);"),
    ("K operand reversed along d",
     "widen_bf16(kh[(size_t)j * D + d])",
     "widen_bf16(kh[(size_t)j * D + (D - 1 - d)])"),
    ("V operand reversed along d",
     "orow[d] += w * widen_bf16(vh[(size_t)j * D + d]);",
     "orow[d] += w * widen_bf16(vh[(size_t)j * D + (D - 1 - d)]);"),
    ("GQA head interleaved instead of grouped",
     "const int b = (int)(bh / Hq), h = (int)(bh % Hq), kvh = h / g;",
     "const int b = (int)(bh / Hq), h = (int)(bh % Hq), kvh = h % Hkv;"),
    ("page slot off by one", "const int slot = t % page_size;",
     "const int slot = (t + 1) % page_size;"),
    ("wrong KV head in the page gather",
     "const size_t src = (((size_t)phys * Hkv + kvh) * page_size + slot) * D;",
     "const size_t src = (((size_t)phys * Hkv + (Hkv - 1 - kvh)) * page_size + slot) * D;"),
    ("chunked prefill ignores causal",
     "lse + ((size_t)b * Hq + h) * max_q, ql, len, D, causal, scale, 0, ql, s);",
     "lse + ((size_t)b * Hq + h) * max_q, ql, len, D, 0, scale, 0, ql, s);"),
    ("e4m3 exponent bias 8", "ldexp(1.0 + (double)m / 8.0, e - 7)",
     "ldexp(1.0 + (double)m / 8.0, e - 8)"),
    ("e4m3 subnormal exponent", "ldexp((double)m / 8.0, 1 - 7)", "ldexp((double)m / 8.0, -7)"),
    ("FP8 K scale dropped",
     "kc[dst + d] = oracle_e4m3_to_f64(k_pages[src + d]) * (double)k_scale[kvh];",
     "kc[dst + d] = oracle_e4m3_to_f64(k_pages[src + d]);"),
    ("FP8 V dequantised with K's scale", "(double)v_scale[kvh]", "(double)k_scale[kvh]"),
    ("FP8 decode scale dropped", "s[j] = scale * dot;", "s[j] = dot;"),
    ("merge weights not normalised", "const double w = exp(ls - lse_r);",
     "const double w = exp(ls - m);"),
    ("merge LSE in log2", "const double lse_r = m + log(total);",
     "const double lse_r = m + log2(total);"),
]


def _pin_calls():
    """Every test function of the pins module with each of its parameter sets,
    in the module's order; functions that need fixtures are left out."""
    calls = []
    for name, fn in vars(pins).items():
        if not name.startswith("test_") or not callable(fn):
            continue
        grids = []
        for mark in getattr(fn, "pytestmark", []):
            if mark.name != "parametrize":
                continue
            argnames, argvalues = mark.args[0], mark.args[1]
            names = ([a.strip() for a in argnames.split(",")] if isinstance(argnames, str)
                     else list(argnames))
            sets = []
            for v in argvalues:
                if hasattr(v, "values") and hasattr(v, "marks"):   # pytest.param(...)
                    v = v.values
                elif len(names) == 1:
                    v = (v,)
                sets.append(dict(zip(names, v)))
            grids.append(sets)
        params = set(inspect.signature(fn).parameters)
        for combo in itertools.product(*grids):
            kw = {}
            for d in combo:
                kw.update(d)
            if params <= set(kw):
                calls.append((name, fn, kw))
    return calls


PIN_CALLS = _pin_calls()


def test_pins_are_collected():
    names = {n for n, _, _ in PIN_CALLS}
    assert len(names) >= 20 and "test_c_oracle_matches_brute_force" in names


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_a_pin_rejects_the_planted_slip(tmp_path, monkeypatch, name, old, new):
    with open(oracle._SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"{name}: the text to replace must occur once"
    mutant = tmp_path / "attn_oracle_mutant.c"
    mutant.write_text(src.replace(old, new))
    monkeypatch.setattr(oracle, "_SRC", str(mutant))
    monkeypatch.setattr(oracle, "_LIB_PATH", str(tmp_path / "libattn_oracle_mutant.so"))
    monkeypatch.setattr(oracle, "_lib", None)
    oracle.build(force=True)   # a copy that does not compile is not a caught slip
    caught = None
    for pin, fn, kw in PIN_CALLS:
        try:
            fn(**kw)
        except (Exception, pytest.fail.Exception):
            caught = pin
            break
    assert caught is not None, f"no pin notices the planted slip: {name}"
