"""The oracle's pins must catch plausible mistakes in the oracle itself.

Each case plants one mistake in a copy of oracle/oracle.c (on the CPU), builds
it into a temporary library, points the oracle wrapper at it and runs the pin
tests: at least one pin must fail.  The unmutated oracle passes all of them
(tests/test_oracle_pins.py).
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTATIONS = {
    "relu_dropped": ("I += wj * (x > 0.0 ? x : 0.0);", "I += wj * x;"),
    "relu_sign_flipped": ("I += wj * (x > 0.0 ? x : 0.0);", "I += wj * (x < 0.0 ? x : 0.0);"),
    "weight_index_swapped": ("double x = 0.0, wj = (double)a->w[(size_t)r * H + j];",
                             "double x = 0.0, wj = (double)a->w[(size_t)j * a->R + r % a->R];"),
    "key_scale_ignored": ("double sc = a->k_scale ? (double)a->k_scale[krow0] : 1.0;", "double sc = 1.0;"),
    "tie_break_reversed": ("return a->i < b->i ? -1 : (a->i > b->i ? 1 : 0);",
                           "return a->i > b->i ? -1 : (a->i < b->i ? 1 : 0);"),
    "topk_unsorted_output": ("qsort(p, (size_t)m, sizeof(vi_pair), cmp_pos);", ""),
    "e4m3_truncates": ("n = nearbyint(a / step);", "n = floor(a / step);"),
    "e4m3_bias_off_by_one": ("return s | (uint8_t)(((E + 7) << 3) | ((int)n - 8));",
                             "return s | (uint8_t)(((E + 8) << 3) | ((int)n - 8));"),
    "quant_scale_inverted": ("s = amax > 0.0f ? amax / 448.0f : 1.0f;", "s = amax > 0.0f ? 448.0f / amax : 1.0f;"),
    "absorb_transposed": ("(double)orc_bf16_to_f32(wdec[((size_t)j * d + e) * dc + c]);",
                          "(double)orc_bf16_to_f32(wdec[((size_t)j * dc + c) * d + e]);"),
    "causal_exclusive": ("if (a->causal) n = (long long)r + 1 + a->causal_offset;",
                         "if (a->causal) n = (long long)r + a->causal_offset;"),
    "hs_padding_scored": ("            if (s < 0) {\n                if (J->cand_scores)",
                          "            if (s < -1000000) {\n                if (J->cand_scores)"),
}

PIN_TESTS = [name for name in dir(pins) if name.startswith("test_")]


def _build(tmp_path, name, old, new):
    src = open(SRC).read()
    assert old in src, name
    mutated = src.replace(old, new, 1)
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-pthread", str(c),
                           "-o", str(so), "-lm"])
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(tmp_path, monkeypatch, name):
    old, new = MUTATIONS[name]
    so = _build(tmp_path, name, old, new)
    saved = oracle._lib
    monkeypatch.setattr(oracle, "_LIB", so)
    monkeypatch.setattr(oracle, "_SRC", so)  # keeps build() from rebuilding over it
    oracle._lib = None
    caught = []
    try:
        for t in PIN_TESTS:
            fn = getattr(pins, t)
            try:
                if "tmp_path" in fn.__code__.co_varnames[:fn.__code__.co_argcount]:
                    continue
                if fn.__code__.co_argcount:
                    continue  # parametrised pins are covered by their plain siblings
                fn()
            except (AssertionError, ValueError, IndexError):
                caught.append(t)
    finally:
        oracle._lib = saved
    assert caught, f"no pin caught the mutation {name}"


# The consumer's oracle is numpy code: mutate its source text instead of oracle.c.
PY_MUTATIONS = {
    "attn_softmax_over_heads": ("logits.max(axis=1, keepdims=True)", "logits.max(axis=0, keepdims=True)",
                                "p.sum(axis=1, keepdims=True)", "p.sum(axis=0, keepdims=True)"),
    "attn_scale_dropped": ("logits = scale * (q[b] @ keys.T)", "logits = (q[b] @ keys.T)"),
    "attn_value_wrong_slice": ("out[b] = p @ keys[:, :dv]", "out[b] = p @ keys[:, -dv:]"),
    "attn_pads_kept": ("s = s[(s >= 0) & (s < cache.shape[0])]", "s = s[s < cache.shape[0]]"),
    "attn_not_normalised": ("p = p / p.sum(axis=1, keepdims=True)", "p = p"),
}


@pytest.mark.parametrize("name", sorted(PY_MUTATIONS))
def test_pins_catch_python_oracle_mutation(monkeypatch, name):
    import inspect
    import textwrap
    reps = PY_MUTATIONS[name]
    src = textwrap.dedent(inspect.getsource(oracle.sparse_attention))
    for old, new in zip(reps[::2], reps[1::2]):
        assert old in src, (name, old)
        src = src.replace(old, new)
    ns = dict(vars(oracle))
    exec(compile(src, f"<{name}>", "exec"), ns)
    monkeypatch.setattr(oracle, "sparse_attention", ns["sparse_attention"])
    failed = []
    for t in [n for n in PIN_TESTS if "sparse_attention" in n]:
        try:
            getattr(pins, t)()
        except Exception:
            failed.append(t)
    assert failed, f"no pin caught {name}"
