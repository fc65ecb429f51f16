"""Pins for the oracle's reshape_and_cache, copy_blocks and swap_blocks (CPU only).

16-bit caches: written slots hold exactly the input bits, every other byte is untouched (checked
against a byte copy of the pool and this test's own slot arithmetic). FP8 caches: the stored code is
PyTorch's round-to-nearest-even float8 cast of the float32 quotient x / scale wherever that quotient is
inside the finite range, and the saturated code beyond it. copy_blocks: destinations equal sources
afterwards, nothing else changes.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import NAN_BITS, bits16


def make_pool(rng, NB, bs, Hkv, d, dtype):
    return rng.integers(0, 1 << 16, (NB, bs, Hkv, d), dtype=np.uint32).astype(np.uint16)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_reshape_and_cache_16bit_writes_exactly_the_slots(dtype):
    rng = np.random.default_rng(1)
    NB, bs, Hkv, d, T = 12, 8, 3, 16, 7
    kc, vc = make_pool(rng, NB, bs, Hkv, d, dtype), make_pool(rng, NB, bs, Hkv, d, dtype)
    kc0, vc0 = kc.copy(), vc.copy()
    key = rng.integers(0, 1 << 16, (T, Hkv, d), dtype=np.uint32).astype(np.uint16)
    value = rng.integers(0, 1 << 16, (T, Hkv, d), dtype=np.uint32).astype(np.uint16)
    slots = np.array([0, 95, 17, -1, 40, NB * bs, 63], np.int64)   # -1: padding; NB*bs: past the pool
    oracle.reshape_and_cache(key, value, dtype, kc, vc, dtype, slots)
    ek, ev = kc0.copy(), vc0.copy()
    for i, slot in enumerate(slots):
        if 0 <= slot < NB * bs:
            ek[slot // bs, slot % bs] = key[i]
            ev[slot // bs, slot % bs] = value[i]
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev)


def test_reshape_and_cache_fp8_matches_library_cast():
    rng = np.random.default_rng(2)
    NB, bs, Hkv, d, T = 6, 16, 4, 32, 40
    key = torch.randn(T, Hkv, d, dtype=torch.float64).to(torch.bfloat16)
    value = (torch.randn(T, Hkv, d, dtype=torch.float64) * 3).to(torch.bfloat16)
    ks = np.array([0.004, 0.01, 0.02, 0.008], np.float32)   # some |x|/scale exceed 448 -> saturate
    vs = np.array([0.03, 0.002, 0.05, 0.01], np.float32)
    kc = np.full((NB, bs, Hkv, d), 0x7F, np.uint8)
    vc = np.full((NB, bs, Hkv, d), 0x7F, np.uint8)
    slots = rng.permutation(NB * bs)[:T].astype(np.int64)
    oracle.reshape_and_cache(bits16(key), bits16(value), "bf16", kc, vc, "fp8_e4m3", slots, ks, vs)

    def expect(x, scale):
        y = x.float() / torch.from_numpy(scale)[:, None]        # float32 quotient, per kv head
        inside = y.abs() < 448
        codes = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        sat = np.where(y.numpy() < 0, 0xFE, 0x7E).astype(np.uint8)
        return np.where(inside.numpy(), codes, sat)

    ek, ev = expect(key, ks), expect(value, vs)
    assert (np.abs(key.float().numpy() / ks[:, None]) >= 448).any()   # the saturation path is exercised
    for i, slot in enumerate(slots):
        assert np.array_equal(kc[slot // bs, slot % bs], ek[i])
        assert np.array_equal(vc[slot // bs, slot % bs], ev[i])
    untouched = np.ones(NB * bs, bool)
    untouched[slots] = False
    assert np.all(kc.reshape(NB * bs, Hkv, d)[untouched] == 0x7F)


def test_quantize_helper_equals_reshape_path():
    rng = np.random.default_rng(3)
    vals = torch.randn(5, 4, 2, 8).to(torch.bfloat16)
    scale = np.array([0.01, 0.004], np.float32)
    q = oracle.quantize_e4m3(bits16(vals), "bf16", scale)
    y = vals.float() / torch.from_numpy(scale)[:, None]
    ref = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    inside = y.abs().numpy() < 448
    assert np.array_equal(q[inside], ref[inside])


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8_e4m3"])
def test_copy_blocks_copies_whole_blocks_only(kv_dtype):
    rng = np.random.default_rng(4)
    NB, bs, Hkv, d = 10, 16, 2, 8
    dt = np.uint8 if kv_dtype == "fp8_e4m3" else np.uint16
    kc = rng.integers(0, np.iinfo(dt).max, (NB, bs, Hkv, d)).astype(dt)
    vc = rng.integers(0, np.iinfo(dt).max, (NB, bs, Hkv, d)).astype(dt)
    kc0, vc0 = kc.copy(), vc.copy()
    pairs = np.array([[1, 7], [4, 2], [0, 9]], np.int64)
    oracle.copy_blocks(kc, vc, kv_dtype, pairs)
    ek, ev = kc0.copy(), vc0.copy()
    for s, t in pairs:
        ek[t], ev[t] = kc0[s], vc0[s]
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev)


def test_copy_blocks_rejects_out_of_range_ids():
    kc = np.zeros((4, 2, 1, 8), np.uint16)
    vc = np.zeros_like(kc)
    with pytest.raises(oracle.OracleError):
        oracle.copy_blocks(kc, vc, "bf16", np.array([[0, 4]], np.int64))


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8_e4m3"])
def test_swap_blocks_moves_whole_blocks_between_pools(kv_dtype):
    rng = np.random.default_rng(5)
    dt = np.uint8 if kv_dtype == "fp8_e4m3" else np.uint16
    dev_k = rng.integers(0, np.iinfo(dt).max, (12, 8, 2, 16)).astype(dt)
    dev_v = rng.integers(0, np.iinfo(dt).max, (12, 8, 2, 16)).astype(dt)
    host_k = np.zeros((5, 8, 2, 16), dt)
    host_v = np.zeros_like(host_k)
    out_pairs = np.array([[3, 0], [7, 4], [11, 2]], np.int64)          # swap-out: device -> host
    oracle.swap_blocks(host_k, host_v, dev_k, dev_v, kv_dtype, out_pairs)
    for s, d in out_pairs:
        assert np.array_equal(host_k[d], dev_k[s]) and np.array_equal(host_v[d], dev_v[s])
    assert np.all(host_k[[1, 3]] == 0) and np.all(host_v[[1, 3]] == 0)  # untouched host blocks
    back_k, back_v = np.zeros_like(dev_k), np.zeros_like(dev_v)
    oracle.swap_blocks(back_k, back_v, host_k, host_v, kv_dtype, out_pairs[:, ::-1].copy())  # swap-in
    for s, d in out_pairs:
        assert np.array_equal(back_k[s], dev_k[s]) and np.array_equal(back_v[s], dev_v[s])
    with pytest.raises(oracle.OracleError):
        oracle.swap_blocks(host_k, host_v, dev_k, dev_v, kv_dtype, np.array([[12, 0]], np.int64))
