"""Pins for the oracle's paged prefill attention (CPU only).

* A chunk of one token per sequence is decode: equal to the decode oracle (itself pinned).
* PyTorch's scaled_dot_product_attention in float64 on the logical contiguous K/V, with an explicit
  causal mask aligned to the END of the context (a chunk continues its sequence), grouped heads
  expanded by the library.
* Closed forms: the first token of a whole prompt attends only to itself, so its output is v_0;
  with all keys equal the weights are uniform over the prefix, so the output is the mean of v_0..v_p.
* Block placement does not matter (a permuted pool and table give the same output).
* Negative control: attention without the causal rule differs, and so does a mask aligned to the
  start of the context.
* FP8 caches (per kv head and per (block, kv head) scales): equal to the same SDPA on K/V that this
  test decodes itself (torch's float8 decode times the scale of the token's physical block), and
  one-token chunks equal the decode oracle bit for bit.
* Planted mistakes in a copy of the C source (off-by-one in the causal bound, the chunk placed at the
  start of the context, the row index of the query, a per-block scale read at the logical block, the
  value scale taken from the keys') fail these pins.
"""
import os
import shutil
import subprocess
import zlib

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from helpers import bits16, logical_fp8, random_paged_case

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "pa_oracle.c")


def chunk_case(rng, lens, qlens, H, Hkv, d, bs, dtype="bf16"):
    """Paged cache of the full contexts, plus query chunks (the last qlens[s] positions)."""
    inputs, _, Ks, Vs = random_paged_case(rng, lens, H, Hkv, d, bs, dtype)
    T = int(sum(qlens))
    q = torch.from_numpy(rng.standard_normal((T, H, d))).to(torch.bfloat16 if dtype == "bf16" else torch.float16)
    q_start = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    inputs = dict(inputs, query_bits=bits16(q), q_start=q_start)
    return inputs, q.to(torch.float64), Ks, Vs


def sdpa_causal_end_aligned(q, Ks, Vs, q_start, scale, H, Hkv):
    out = []
    for s in range(len(Ks)):
        n = q_start[s + 1] - q_start[s]
        if n == 0:
            continue
        L = Ks[s].shape[0]
        qs = q[q_start[s]:q_start[s + 1]].permute(1, 0, 2).unsqueeze(0)       # [1, H, n, d]
        k = Ks[s].permute(1, 0, 2).unsqueeze(0)                                # [1, Hkv, L, d]
        v = Vs[s].permute(1, 0, 2).unsqueeze(0)
        pos = torch.arange(L - n, L).unsqueeze(1)                              # query positions
        mask = torch.arange(L).unsqueeze(0) <= pos                             # [n, L]
        o = F.scaled_dot_product_attention(qs, k, v, attn_mask=mask, scale=scale, enable_gqa=(H != Hkv))
        out.append(o[0].permute(1, 0, 2))
    return torch.cat(out).numpy()


CASES = [
    # (bs, H, Hkv, d, lens, qlens)
    (16, 8, 8, 64, [17, 40, 100], [17, 5, 64]),
    (8, 8, 2, 32, [9, 64, 65, 3], [1, 64, 20, 3]),
    (4, 6, 3, 16, [13, 5, 30], [13, 0, 7]),
    (32, 4, 1, 128, [70, 33], [70, 1]),
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_matches_library_sdpa_with_end_aligned_causal_mask(case, dtype):
    bs, H, Hkv, d, lens, qlens = case
    rng = np.random.default_rng(zlib.crc32(repr((case, dtype)).encode()))
    inputs, q, Ks, Vs = chunk_case(rng, lens, qlens, H, Hkv, d, bs, dtype)
    out = oracle.paged_prefill(scale=0.2, **inputs)
    ref = sdpa_causal_end_aligned(q, Ks, Vs, inputs["q_start"], 0.2, H, Hkv)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_one_token_chunks_equal_decode():
    rng = np.random.default_rng(1)
    lens = [1, 9, 31, 64]
    inputs, q, _, _ = chunk_case(rng, lens, [1] * 4, 8, 2, 32, 8)
    pre = oracle.paged_prefill(scale=0.3, **inputs)
    dec_inputs = {k: v for k, v in inputs.items() if k != "q_start"}
    dec = oracle.paged_attention(scale=0.3, **dec_inputs)
    assert np.array_equal(pre, dec)


def test_closed_forms():
    rng = np.random.default_rng(2)
    L, H, d, bs = 12, 2, 8, 4
    inputs, q, Ks, Vs = chunk_case(rng, [L], [L], H, H, d, bs)
    out = oracle.paged_prefill(scale=0.5, **inputs)
    np.testing.assert_allclose(out[0], Vs[0][0].numpy(), rtol=0, atol=1e-15)        # first token: v_0
    # All keys equal: uniform weights over each prefix.
    kc = inputs["key_cache"]
    tables = inputs["block_tables"]
    k0 = kc[tables[0, 0], 0].copy()
    for t in range(L):
        kc[tables[0, t // bs], t % bs] = k0
    out = oracle.paged_prefill(scale=0.5, **inputs)
    for p in range(L):
        np.testing.assert_allclose(out[p], Vs[0][:p + 1].mean(0).numpy(), rtol=0, atol=1e-14)


def test_placement_invariance():
    rng = np.random.default_rng(3)
    inputs, *_ = chunk_case(rng, [30, 21], [11, 21], 4, 2, 16, 4)
    out = oracle.paged_prefill(scale=0.25, **inputs)
    perm = rng.permutation(inputs["key_cache"].shape[0])
    inv = np.argsort(perm)
    moved = dict(inputs, key_cache=inputs["key_cache"][perm].copy(), value_cache=inputs["value_cache"][perm].copy(),
                 block_tables=inv[inputs["block_tables"]].astype(np.int32))
    assert np.array_equal(oracle.paged_prefill(scale=0.25, **moved), out)


def test_negative_controls():
    rng = np.random.default_rng(4)
    lens, qlens = [40, 25], [16, 25]
    inputs, q, Ks, Vs = chunk_case(rng, lens, qlens, 4, 4, 16, 8)
    out = oracle.paged_prefill(scale=0.25, **inputs)
    # No causal rule: every query sees the whole context.
    full = []
    for s in range(2):
        qs = q[inputs["q_start"][s]:inputs["q_start"][s + 1]].permute(1, 0, 2).unsqueeze(0)
        o = F.scaled_dot_product_attention(qs, Ks[s].permute(1, 0, 2).unsqueeze(0),
                                           Vs[s].permute(1, 0, 2).unsqueeze(0), scale=0.25)
        full.append(o[0].permute(1, 0, 2))
    assert np.max(np.abs(out - torch.cat(full).numpy())) > 1e-3
    # Mask aligned to the start of the context (the library's own is_causal convention).
    s0 = q[:16].permute(1, 0, 2).unsqueeze(0)
    o = F.scaled_dot_product_attention(s0, Ks[0].permute(1, 0, 2).unsqueeze(0), Vs[0].permute(1, 0, 2).unsqueeze(0),
                                       scale=0.25, is_causal=True)
    assert np.max(np.abs(out[:16] - o[0].permute(1, 0, 2).numpy())) > 1e-3


FP8_FORMATS = ["fp8_e4m3", "fp8_e4m3_block"]


def fp8_chunk_case(rng, lens, qlens, H, Hkv, d, bs, fmt):
    """Query chunks over an FP8 cache quantised by the oracle's encoder (itself pinned against torch's
    float8 cast), with random scales per kv head or per (block, kv head)."""
    inputs, q, _, _ = chunk_case(rng, lens, qlens, H, Hkv, d, bs)
    NB = inputs["key_cache"].shape[0]
    shape = (NB, Hkv) if fmt == "fp8_e4m3_block" else (Hkv,)
    ks = rng.uniform(0.002, 0.02, shape).astype(np.float32)
    vs = rng.uniform(0.002, 0.02, shape).astype(np.float32)
    quant = oracle.quantize_e4m3_blocks if fmt == "fp8_e4m3_block" else oracle.quantize_e4m3
    kc = quant(inputs["key_cache"], "bf16", ks)
    vc = quant(inputs["value_cache"], "bf16", vs)
    return dict(inputs, key_cache=kc, value_cache=vc, kv_dtype=fmt, k_scale=ks, v_scale=vs), q


def fp8_sdpa_reference(inputs, q, lens, bs, scale, H, Hkv):
    t = inputs["block_tables"]
    Ks = [logical_fp8(inputs["key_cache"], inputs["k_scale"], t, s, L, bs) for s, L in enumerate(lens)]
    Vs = [logical_fp8(inputs["value_cache"], inputs["v_scale"], t, s, L, bs) for s, L in enumerate(lens)]
    return sdpa_causal_end_aligned(q, Ks, Vs, inputs["q_start"], scale, H, Hkv)


@pytest.mark.parametrize("case", CASES[:3])
@pytest.mark.parametrize("fmt", FP8_FORMATS)
def test_fp8_caches_match_sdpa_on_self_decoded_kv(case, fmt):
    bs, H, Hkv, d, lens, qlens = case
    rng = np.random.default_rng(zlib.crc32(repr((case, fmt)).encode()))
    inputs, q = fp8_chunk_case(rng, lens, qlens, H, Hkv, d, bs, fmt)
    out = oracle.paged_prefill(scale=0.2, **inputs)
    np.testing.assert_allclose(out, fp8_sdpa_reference(inputs, q, lens, bs, 0.2, H, Hkv), rtol=0, atol=1e-12)


@pytest.mark.parametrize("fmt", FP8_FORMATS)
def test_fp8_one_token_chunks_equal_decode(fmt):
    rng = np.random.default_rng(11)
    inputs, _ = fp8_chunk_case(rng, [1, 9, 31, 64], [1] * 4, 8, 2, 32, 8, fmt)
    pre = oracle.paged_prefill(scale=0.3, **inputs)
    dec = oracle.paged_attention(scale=0.3, **{k: v for k, v in inputs.items() if k != "q_start"})
    assert np.array_equal(pre, dec)


MUTANTS = [
    ("causal_off_by_one", "for (int t = 0; t <= p; ++t) {\n    int blk = a->block_tables[(size_t)s * a->max_blocks_per_seq + t / a->block_size];\n    if (blk",
     "for (int t = 0; t < p; ++t) {\n    int blk = a->block_tables[(size_t)s * a->max_blocks_per_seq + t / a->block_size];\n    if (blk"),
    ("chunk_at_start", "const int p = a->context_lens[s] - n + j;", "const int p = j;"),
    ("query_row", "const size_t q_base = ((size_t)row * a->num_heads + h) * d;\n  double* o",
     "const size_t q_base = ((size_t)j * a->num_heads + h) * d;\n  double* o"),
    ("block_scale_logical_index",
     "t % a->block_size) * a->num_kv_heads + kvh) * d;\n"
     "    const double ks = kv_scale(a->k_scale, a->kv_dtype, blk, a->num_kv_heads, kvh);",
     "t % a->block_size) * a->num_kv_heads + kvh) * d;\n"
     "    const double ks = kv_scale(a->k_scale, a->kv_dtype, t / a->block_size, a->num_kv_heads, kvh);"),
    ("value_scale_from_keys",
     "t % a->block_size) * a->num_kv_heads + kvh) * d;\n"
     "    const double vs = kv_scale(a->v_scale, a->kv_dtype, blk, a->num_kv_heads, kvh);",
     "t % a->block_size) * a->num_kv_heads + kvh) * d;\n"
     "    const double vs = kv_scale(a->k_scale, a->kv_dtype, blk, a->num_kv_heads, kvh);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS)
def test_planted_mistakes_fail_the_pins(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, name
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-shared", "-fPIC", "-fno-fast-math", "-ffp-contract=off", "-o", str(so),
                    str(mutant), "-lm", "-lpthread"], check=True)
    failures = 0
    with oracle.use_library(str(so)):
        for case in CASES[:2]:
            bs, H, Hkv, d, lens, qlens = case
            rng = np.random.default_rng(zlib.crc32(repr((case, "bf16")).encode()))
            inputs, q, Ks, Vs = chunk_case(rng, lens, qlens, H, Hkv, d, bs)
            try:
                out = oracle.paged_prefill(scale=0.2, **inputs)
                if not np.allclose(out, sdpa_causal_end_aligned(q, Ks, Vs, inputs["q_start"], 0.2, H, Hkv),
                                   rtol=0, atol=1e-12):
                    failures += 1
            except Exception:
                failures += 1
            rng = np.random.default_rng(zlib.crc32(repr((case, "fp8_e4m3_block")).encode()))
            inputs, q = fp8_chunk_case(rng, lens, qlens, H, Hkv, d, bs, "fp8_e4m3_block")
            try:
                out = oracle.paged_prefill(scale=0.2, **inputs)
                if not np.allclose(out, fp8_sdpa_reference(inputs, q, lens, bs, 0.2, H, Hkv), rtol=0, atol=1e-12):
                    failures += 1
            except Exception:
                failures += 1
    assert failures > 0, f"mutant {name} passed every pin"
