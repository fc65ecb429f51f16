"""Pins for the oracle's paged attention (CPU only).

Each check ties the oracle to something other than itself:
  * hand-derived golden cases (tests/golden/attention_hand_cases.json);
  * PyTorch's scaled_dot_product_attention in float64 on contiguous logical K/V that never went
    through the oracle's block-table gather (the test writes tokens into blocks itself);
  * closed forms: one token gives its value exactly; equal keys or a zero scale give the mean of V;
    a dominant key gives its value;
  * invariants: permuting physical blocks changes nothing (bit for bit); shared prefix blocks give
    the same output as private copies;
  * the tutorial page's per-block loop ("企业官网建设流程全解析", sec. 2.2) agrees with the definition
    when the context fits in one block and disagrees as soon as it spans two (negative control).
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from helpers import bits16, golden_case_arrays, random_paged_case

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
CASES = json.load(open(os.path.join(GOLDEN, "attention_hand_cases.json")))["cases"]


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_golden_hand_cases(case):
    out = oracle.paged_attention(**golden_case_arrays(case))
    np.testing.assert_allclose(out, np.array(case["expected"]), rtol=0, atol=1e-12)


def sdpa_reference(q, Ks, Vs, scale, num_kv_heads):
    """Library attention per sequence on the logical K/V (float64, grouped-query heads)."""
    outs = []
    for s in range(q.shape[0]):
        L = Ks[s].shape[0]
        H = q.shape[1]
        if L == 0:
            outs.append(torch.zeros(H, q.shape[2], dtype=torch.float64))
            continue
        qs = q[s].unsqueeze(1).unsqueeze(0)            # [1, H, 1, d]
        k = Ks[s].permute(1, 0, 2).unsqueeze(0)       # [1, Hkv, L, d]
        v = Vs[s].permute(1, 0, 2).unsqueeze(0)
        o = F.scaled_dot_product_attention(qs, k, v, scale=scale, enable_gqa=(H != num_kv_heads))
        outs.append(o[0, :, 0, :])
    return torch.stack(outs).numpy()


@pytest.mark.parametrize("bs,H,Hkv,d,lens", [
    (16, 8, 8, 64, [1, 17, 33, 100]),
    (8, 8, 2, 32, [9, 8, 7, 64, 65]),
    (32, 4, 1, 16, [31, 32, 33, 0, 1]),
    (4, 6, 3, 8, [1, 2, 3, 4, 5, 13]),
])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_matches_library_sdpa_on_logical_kv(bs, H, Hkv, d, lens, dtype):
    rng = np.random.default_rng(hash((bs, H, Hkv, d, len(lens), dtype)) % (2 ** 32))
    inputs, q, Ks, Vs = random_paged_case(rng, lens, H, Hkv, d, bs, dtype)
    scale = 1.0 / math.sqrt(d)
    out = oracle.paged_attention(scale=scale, **inputs)
    ref = sdpa_reference(q, Ks, Vs, scale, Hkv)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_fp8_matches_library_sdpa_on_dequantised_kv():
    rng = np.random.default_rng(5)
    lens, H, Hkv, d, bs = [40, 3, 17], 8, 2, 32, 16
    inputs, q, Ks, Vs = random_paged_case(rng, lens, H, Hkv, d, bs, "bf16")
    kc_codes = rng.integers(0, 256, inputs["key_cache"].shape, dtype=np.uint8)
    vc_codes = rng.integers(0, 256, inputs["key_cache"].shape, dtype=np.uint8)
    kc_codes[(kc_codes & 0x7F) == 0x7F] = 0x38   # keep the random cache free of NaN codes
    vc_codes[(vc_codes & 0x7F) == 0x7F] = 0x38
    ks = np.array([0.01, 0.02], np.float32)
    vs = np.array([0.03, 0.005], np.float32)
    out = oracle.paged_attention(inputs["query_bits"], "bf16", kc_codes, vc_codes, "fp8_e4m3",
                                 inputs["block_tables"], inputs["context_lens"], 0.125, ks, vs)
    dec = lambda c: torch.from_numpy(c.copy()).view(torch.float8_e4m3fn).to(torch.float64)
    Kd, Vd = dec(kc_codes), dec(vc_codes)
    Ks2, Vs2 = [], []
    for s, L in enumerate(lens):
        rows_k, rows_v = [], []
        for t in range(L):
            blk = inputs["block_tables"][s, t // bs]
            rows_k.append(Kd[blk, t % bs] * torch.from_numpy(ks.astype(np.float64))[:, None])
            rows_v.append(Vd[blk, t % bs] * torch.from_numpy(vs.astype(np.float64))[:, None])
        Ks2.append(torch.stack(rows_k))
        Vs2.append(torch.stack(rows_v))
    ref = sdpa_reference(q, Ks2, Vs2, 0.125, Hkv)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_single_token_returns_its_value_exactly():
    rng = np.random.default_rng(1)
    inputs, q, Ks, Vs = random_paged_case(rng, [1, 1], 4, 2, 16, 8, "bf16")
    out = oracle.paged_attention(scale=0.3, **inputs)
    for s in range(2):
        for h in range(4):
            assert np.array_equal(out[s, h], Vs[s][0, h // 2].numpy())


def test_equal_keys_and_zero_scale_give_mean_of_values():
    rng = np.random.default_rng(2)
    inputs, q, Ks, Vs = random_paged_case(rng, [37], 2, 1, 8, 8, "bf16")
    mean = Vs[0][:, 0].mean(dim=0).numpy()
    out0 = oracle.paged_attention(scale=0.0, **inputs)
    np.testing.assert_allclose(out0[0, 0], mean, rtol=0, atol=1e-13)
    kc = inputs["key_cache"].copy()
    kc[:] = bits16(torch.tensor([0.75], dtype=torch.bfloat16))[0]
    inputs["key_cache"] = kc
    out1 = oracle.paged_attention(scale=0.2, **inputs)
    np.testing.assert_allclose(out1[0, 1], mean, rtol=0, atol=1e-13)


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(3)
    inputs, q, Ks, Vs = random_paged_case(rng, [20], 1, 1, 4, 4, "bf16")
    kc = inputs["key_cache"]
    qv = torch.tensor([[[1.0, 0.0, 0.0, 0.0]]], dtype=torch.bfloat16)
    inputs["query_bits"] = bits16(qv)
    blk, off = inputs["block_tables"][0, 13 // 4], 13 % 4
    for t in range(20):
        b, o = inputs["block_tables"][0, t // 4], t % 4
        kc[b, o, 0] = bits16(torch.tensor([0.0, 1.0, 1.0, 1.0], dtype=torch.bfloat16))
    kc[blk, off, 0] = bits16(torch.tensor([64.0, 0.0, 0.0, 0.0], dtype=torch.bfloat16))
    out = oracle.paged_attention(scale=1.0, **inputs)
    # weight of the others is 19 e^-64 relative; the output equals v_13 to within that
    np.testing.assert_allclose(out[0, 0], Vs[0][13, 0].numpy(), rtol=0, atol=1e-25)


def test_block_permutation_is_bitwise_invariant():
    rng = np.random.default_rng(4)
    inputs, q, Ks, Vs = random_paged_case(rng, [50, 3, 16, 17], 4, 2, 16, 8, "bf16", extra_blocks=6)
    base = oracle.paged_attention(scale=0.25, **inputs)
    NB = inputs["key_cache"].shape[0]
    perm = np.random.default_rng(9).permutation(NB)          # old id -> new id
    kc = np.empty_like(inputs["key_cache"])
    vc = np.empty_like(inputs["value_cache"])
    kc[perm] = inputs["key_cache"]
    vc[perm] = inputs["value_cache"]
    moved = dict(inputs, key_cache=kc, value_cache=vc, block_tables=perm[inputs["block_tables"]].astype(np.int32))
    again = oracle.paged_attention(scale=0.25, **moved)
    assert np.array_equal(base, again)


def test_shared_prefix_blocks_equal_private_copies():
    """Sequences that share physical prefix blocks (reference count > 1, tutorial sec. 2.3) read the
    same data as sequences holding private copies of those blocks."""
    rng = np.random.default_rng(6)
    bs, Hkv, d, H = 8, 2, 16, 4
    prefix_blocks, suffix = 3, [5, 11, 5]
    NB = prefix_blocks * 4 + 8
    kc = rng.integers(0x3000, 0x4000, (NB, bs, Hkv, d)).astype(np.uint16)  # finite bf16 values
    vc = rng.integers(0x3000, 0x4000, (NB, bs, Hkv, d)).astype(np.uint16)
    shared = [0, 1, 2]
    tails = [[12], [13, 14], [15]]
    kc[15], vc[15] = kc[12], vc[12]   # sequence 2's suffix equals sequence 0's
    lens = [prefix_blocks * bs + x for x in suffix]
    tables = np.zeros((3, 5), np.int32)
    for s in range(3):
        row = shared + tails[s]
        tables[s, :len(row)] = row
    q = np.repeat(rng.integers(0x3000, 0x4000, (1, H, d)).astype(np.uint16), 3, axis=0)
    out_shared = oracle.paged_attention(q, "bf16", kc, vc, "bf16", tables, np.array(lens, np.int32), 0.1)
    # private copies of the prefix for every sequence
    private = tables.copy()
    for s in range(3):
        for j in range(prefix_blocks):
            dst = 3 + 3 * s + j
            kc[dst], vc[dst] = kc[shared[j]], vc[shared[j]]
            private[s, j] = dst
    out_private = oracle.paged_attention(q, "bf16", kc, vc, "bf16", private, np.array(lens, np.int32), 0.1)
    assert np.array_equal(out_shared, out_private)
    assert np.array_equal(out_shared[0], out_shared[2])      # same query, same logical tokens


def tutorial_per_block_loop(q, K, V, bs, scale):
    """The tutorial page's loop (sec. 2.2), restated: softmax inside each block, outputs summed."""
    out = torch.zeros_like(q)
    for start in range(0, K.shape[0], bs):
        scores = (q @ K[start:start + bs].T) * scale
        out += torch.softmax(scores, dim=-1) @ V[start:start + bs]
    return out


def test_tutorial_loop_is_a_negative_control():
    rng = np.random.default_rng(8)
    bs, d = 8, 16
    for L, should_match in [(5, True), (8, True), (9, False), (40, False)]:
        inputs, q, Ks, Vs = random_paged_case(rng, [L], 1, 1, d, bs, "bf16")
        out = oracle.paged_attention(scale=0.5, **inputs)[0, 0]
        loop = tutorial_per_block_loop(q[0], Ks[0][:, 0], Vs[0][:, 0], bs, 0.5)[0].numpy()
        if should_match:
            np.testing.assert_allclose(out, loop, rtol=0, atol=1e-12)
        else:
            assert np.max(np.abs(out - loop)) > 0.1


def test_zero_length_context_gives_zeros():
    rng = np.random.default_rng(10)
    inputs, *_ = random_paged_case(rng, [0, 3], 2, 2, 8, 4, "f16")
    out = oracle.paged_attention(scale=1.0, **inputs)
    assert np.all(out[0] == 0.0) and np.all(np.isfinite(out[1]))


def test_block_id_out_of_range_is_an_error():
    rng = np.random.default_rng(12)
    inputs, *_ = random_paged_case(rng, [10], 1, 1, 8, 4, "bf16")
    inputs["block_tables"][0, 1] = inputs["key_cache"].shape[0]
    with pytest.raises(oracle.OracleError):
        oracle.paged_attention(scale=1.0, **inputs)


def test_threads_do_not_change_the_result():
    rng = np.random.default_rng(13)
    inputs, *_ = random_paged_case(rng, [33, 70, 1, 9], 8, 2, 32, 16, "bf16")
    one = oracle.paged_attention(scale=0.2, num_threads=1, **inputs)
    many = oracle.paged_attention(scale=0.2, num_threads=5, **inputs)
    assert np.array_equal(one, many)
