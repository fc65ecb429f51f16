"""The pins catch plausible mistakes: each test plants one mistake in a copy of the oracle's C source
(on the CPU, in a temporary directory), builds it, and checks that at least one pin fails on it.
The real oracle is never modified.
"""
import json
import math
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle
from helpers import golden_case_arrays, random_paged_case
from test_oracle_attention import CASES, sdpa_reference

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "pa_oracle.c")

# (name, text to replace, replacement): a dropped term, a wrong sign, a wrong index, a transposed or
# mis-mapped operand, a wrong constant.
MUTANTS = [
    ("logical_block_index", "t / a->block_size];\n    int off = t % a->block_size;\n    if (blk",
     "t % a->block_size];\n    int off = t % a->block_size;\n    if (blk"),
    ("offset_within_block", "int off = t % a->block_size;\n    if (blk", "int off = t / a->block_size;\n    if (blk"),
    ("softmax_sign", "denom += exp(z[t] - m)", "denom += exp(m - z[t])"),
    ("no_max_shift_in_weights", "double w = exp(z[t] - m) / denom;", "double w = exp(z[t]) / denom;"),
    ("gqa_head_mapping", "const int kvh = h / G;", "const int kvh = h % a->num_kv_heads;"),
    ("scale_dropped", "z[t] = a->scale * dot;", "z[t] = dot;"),
    ("layout_head_and_offset_swapped",
     "size_t k_base = (((size_t)blk * a->block_size + off) * a->num_kv_heads + kvh) * d;",
     "size_t k_base = (((size_t)blk * a->num_kv_heads + kvh) * a->block_size + off) * d;"),
    ("fp8_subnormal_exponent", "v = ldexp((double)mantissa, -9);", "v = ldexp((double)mantissa, -10);"),
    ("fp8_bias", "v = ldexp(1.0 + mantissa / 8.0, exponent - 7);", "v = ldexp(1.0 + mantissa / 8.0, exponent - 8);"),
    ("fp8_ties_away", "pick = (lo % 2 == 0) ? lo : hi;", "pick = hi;"),
    ("fp8_k_scale_dropped", "(element(a->key_cache, a->kv_dtype, k_base + i) * ks);",
     "(element(a->key_cache, a->kv_dtype, k_base + i));"),
    ("bf16_bias", "v = ldexp(1.0 + fraction / 128.0, exponent - 127);", "v = ldexp(1.0 + fraction / 128.0, exponent - 126);"),
]


def run_pins():
    """A compact selection of the pins; returns the names of those that fail."""
    failed = []
    for case in CASES:
        try:
            out = oracle.paged_attention(**golden_case_arrays(case))
            if not np.allclose(out, np.array(case["expected"]), rtol=0, atol=1e-12):
                failed.append("golden:" + case["name"])
        except Exception:
            failed.append("golden-error:" + case["name"])
    rng = np.random.default_rng(0)
    inputs, q, Ks, Vs = random_paged_case(rng, [33, 7, 64], 8, 2, 32, 8, "bf16")
    try:
        out = oracle.paged_attention(scale=0.3, **inputs)
        if not np.allclose(out, sdpa_reference(q, Ks, Vs, 0.3, 2), rtol=0, atol=1e-12):
            failed.append("sdpa")
    except Exception:
        failed.append("sdpa-error")
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_double(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    if not np.array_equal(np.nan_to_num(ours, nan=7.0), np.nan_to_num(ref, nan=7.0)):
        failed.append("e4m3-decode")
    pos = ref[:0x7F]
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    lower = np.arange(0x7E, dtype=np.uint8)
    if not np.array_equal(oracle.e4m3_from_float(mids), np.where(lower % 2 == 0, lower, lower + 1)):
        failed.append("e4m3-ties")
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    bf = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    if not np.array_equal(np.nan_to_num(oracle.bf16_to_double(bits), nan=7.0), np.nan_to_num(bf, nan=7.0)):
        failed.append("bf16-decode")
    return failed


def test_unmutated_oracle_passes_the_selection():
    assert run_pins() == []


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, old, new):
    text = open(SRC).read()
    # The mistakes are planted in the codecs and the decode definition, which come before the
    # decode worker; later functions (prefill, cache operations) are left as they are.
    cut = text.index("static void* attention_worker(")
    head, tail = text[:cut], text[cut:]
    assert head.count(old) == 1, f"mutation anchor for {name} not unique"
    src = tmp_path / "mutant.c"
    src.write_text(head.replace(old, new) + tail)
    lib = tmp_path / f"libmutant_{name}.so"
    subprocess.run(["gcc", "-std=c11", "-O1", "-fPIC", "-shared", "-pthread", "-o", str(lib), str(src), "-lm"],
                   check=True)
    with oracle.use_library(str(lib)):
        failed = run_pins()
    assert failed, f"planted mistake {name} went unnoticed"
