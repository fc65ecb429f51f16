"""Pins for the oracle's per-block-scaled FP8 cache format (CPU only): each (block, kv head) has
its own scale; a value dequantises as code x scale[block][kv head].

* With every block of a head given the head's scale, the per-block format reproduces the per-head
  format bit for bit (attention outputs and written codes).
* Attention equals PyTorch's scaled_dot_product_attention in float64 on logical K/V that this test
  decodes itself (torch's float8 decode of each code times its block's scale).
* reshape_and_cache writes torch's round-to-nearest-even float8 cast of the float32 quotient
  x / scale[block][kv head].
* Planted mistakes (the per-block scale read per head, in attention or in the encoder) are caught.
"""
import os
import subprocess

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from helpers import bits16, logical_fp8, random_paged_case

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "pa_oracle.c")


def fp8_case(rng, lens, H, Hkv, d, bs):
    inputs, q, Ks, Vs = random_paged_case(rng, lens, H, Hkv, d, bs, "bf16")
    NB = inputs["key_cache"].shape[0]
    kb, vb = inputs["key_cache"], inputs["value_cache"]
    ks = rng.uniform(0.002, 0.02, (NB, Hkv)).astype(np.float32)
    vs = rng.uniform(0.002, 0.02, (NB, Hkv)).astype(np.float32)
    kc = oracle.quantize_e4m3_blocks(kb, "bf16", ks)
    vc = oracle.quantize_e4m3_blocks(vb, "bf16", vs)
    inputs = dict(inputs, key_cache=kc, value_cache=vc, kv_dtype="fp8_e4m3_block", k_scale=ks, v_scale=vs)
    return inputs, q


@pytest.mark.parametrize("H,Hkv,d,bs,lens", [(8, 2, 32, 8, [9, 40, 1]), (4, 4, 16, 16, [33, 16, 70])])
def test_matches_sdpa_on_self_decoded_kv(H, Hkv, d, bs, lens):
    rng = np.random.default_rng(H * 100 + bs)
    inputs, q = fp8_case(rng, lens, H, Hkv, d, bs)
    out = oracle.paged_attention(scale=0.3, **inputs)
    for s, L in enumerate(lens):
        K = logical_fp8(inputs["key_cache"], inputs["k_scale"], inputs["block_tables"], s, L, bs)
        V = logical_fp8(inputs["value_cache"], inputs["v_scale"], inputs["block_tables"], s, L, bs)
        ref = F.scaled_dot_product_attention(q[s].unsqueeze(1).unsqueeze(0), K.permute(1, 0, 2).unsqueeze(0),
                                             V.permute(1, 0, 2).unsqueeze(0), scale=0.3,
                                             enable_gqa=(H != Hkv))[0, :, 0, :].numpy()
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-12)


def test_uniform_block_scales_equal_the_per_head_format():
    rng = np.random.default_rng(7)
    inputs, q = fp8_case(rng, [30, 17], 4, 2, 16, 8)
    NB = inputs["key_cache"].shape[0]
    head_k = np.array([0.011, 0.004], np.float32)
    head_v = np.array([0.007, 0.013], np.float32)
    kb, vb = bits16(torch.randn(NB, 8, 2, 16).to(torch.bfloat16)), bits16(torch.randn(NB, 8, 2, 16).to(torch.bfloat16))
    kc_block = oracle.quantize_e4m3_blocks(kb, "bf16", np.tile(head_k, (NB, 1)))
    kc_head = oracle.quantize_e4m3(kb, "bf16", head_k)
    assert np.array_equal(kc_block, kc_head)
    vc = oracle.quantize_e4m3(vb, "bf16", head_v)
    per_block = oracle.paged_attention(**dict(inputs, key_cache=kc_head, value_cache=vc,
                                              k_scale=np.tile(head_k, (NB, 1)), v_scale=np.tile(head_v, (NB, 1))),
                                       scale=0.25)
    per_head = oracle.paged_attention(**dict(inputs, key_cache=kc_head, value_cache=vc, kv_dtype="fp8_e4m3",
                                             k_scale=head_k, v_scale=head_v), scale=0.25)
    assert np.array_equal(per_block, per_head)


def test_reshape_uses_the_slots_block_scale():
    rng = np.random.default_rng(8)
    NB, bs, Hkv, d, T = 6, 4, 2, 16, 15
    x = (torch.randn(T, Hkv, d) * 2).to(torch.bfloat16)
    ks = rng.uniform(0.003, 0.03, (NB, Hkv)).astype(np.float32)
    kc = np.full((NB, bs, Hkv, d), 0x7F, np.uint8)
    vc = np.full_like(kc, 0x7F)
    slots = rng.permutation(NB * bs)[:T].astype(np.int64)
    oracle.reshape_and_cache(bits16(x), bits16(x), "bf16", kc, vc, "fp8_e4m3_block", slots, ks, ks)
    for i, slot in enumerate(slots):
        blk = slot // bs
        y = x[i].float() / torch.from_numpy(ks[blk])[:, None]
        want = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        inside = y.abs().numpy() < 448
        assert np.array_equal(kc[blk, slot % bs][inside], want[inside])


MUTANTS = [
    ("attention_block_scale_read_per_head", "return (double)scale[(size_t)blk * num_kv_heads + kvh];",
     "return (double)scale[kvh];"),
    ("encoder_block_scale_read_per_head", "? (size_t)blk * num_kv_heads + h : (size_t)h;",
     "? (size_t)h : (size_t)h;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS)
def test_planted_mistakes_fail_the_pins(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, name
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-std=c11", "-O1", "-fPIC", "-shared", "-pthread", "-o", str(so), str(mutant), "-lm"],
                   check=True)
    failed = False
    with oracle.use_library(str(so)):
        for test in (test_matches_sdpa_on_self_decoded_kv, test_reshape_uses_the_slots_block_scale):
            try:
                if test is test_matches_sdpa_on_self_decoded_kv:
                    test(8, 2, 32, 8, [9, 40, 1])
                else:
                    test()
            except AssertionError:
                failed = True
    assert failed, f"mutant {name} passed every pin"
