"""GPU parity: the C-ABI library against the oracle on the same seeded inputs.

* Every config of the workload table at its full size, in the launch configuration the benchmark
  uses (automatic partition size): one decode step (copy_blocks of the copy-on-write pairs,
  reshape_and_cache of the new tokens, paged attention). Every attention output is compared element by element
  with the oracle (max-abs within the stated tolerance); the whole key and value pools after the step
  are compared byte for byte with the oracle's (reshape_and_cache and copy_blocks are bit-exact, and
  nothing else in the pool may change).
* Split-K partition sizes from one stage to the whole context agree with the oracle.
* Smaller ragged cases over every supported head size, block size, dtype and group size. Their
  contexts go down to one token, where outputs reach about 5 in magnitude; there each element is
  bounded by the stated tolerance plus half an ulp of the output dtype at that magnitude.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from helpers import bits16
from steps import TOLERANCE, elementwise_bound, gpu_step, initial_pools, oracle_step, pool_bits, to_device_pool

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    from pagedattention_paged_kv_attention_b200 import pagedattn
    return pagedattn


def max_abs_err(out_dev, ref):
    got = out_dev.double().cpu().numpy()
    assert np.all(np.isfinite(got)), "non-finite output (a poisoned element was read)"
    return float(np.max(np.abs(got - ref))) if ref.size else 0.0


@pytest.mark.parametrize("name", list(W.CONFIGS))
def test_config_step_matches_oracle(P, name):
    cfg = W.CONFIGS[name]
    w = W.make_workload(cfg)
    kc, vc = initial_pools(w)
    kc_dev, vc_dev = to_device_pool(kc, cfg), to_device_pool(vc, cfg)
    out, ws = gpu_step(P, w, kc_dev, vc_dev)
    torch.cuda.synchronize()
    ref = oracle_step(w, kc, vc)
    err = max_abs_err(out, ref)
    assert err <= TOLERANCE[cfg.kv_dtype], f"{name}: max-abs error {err}"
    assert P.get_device_error(ws) == 0
    # Pools: byte-exact against the oracle's pools after the same step.
    assert torch.equal(pool_bits(kc_dev), pool_bits(to_device_pool(kc, cfg))), "key pool differs"
    assert torch.equal(pool_bits(vc_dev), pool_bits(to_device_pool(vc, cfg))), "value pool differs"


@pytest.mark.parametrize("partition_size", [64, 128, 512, 2048, 4096])
def test_split_k_partition_sizes(P, partition_size):
    cfg = W.CONFIGS["70b_gqa"]
    w = W.make_workload(cfg, num_seqs=16, prefilled=True)
    kc, vc = initial_pools(w)
    ref = oracle_step(w, kc, vc, write_new=False)
    out, ws = gpu_step(P, w, to_device_pool(kc, cfg), to_device_pool(vc, cfg), write_new=False,
                       partition_size=partition_size)
    assert max_abs_err(out, ref) <= TOLERANCE["bf16"]
    assert P.get_device_error(ws) == 0


def small_case(kv_dtype, dtype, head_size, block_size, H, Hkv, lens, seed):
    cfg = W.Config(name="case", description="ragged parity case", num_seqs=len(lens), num_heads=H,
                   num_kv_heads=Hkv, head_size=head_size, block_size=block_size, dtype=dtype,
                   kv_dtype=kv_dtype, seed=seed, context_lens=tuple(lens))
    return cfg, W.make_workload(cfg)


CASES = []
for d in (64, 128):
    for bs in (8, 16, 32, 64):
        for (H, Hkv) in ((4, 4), (8, 4), (12, 3), (16, 4), (32, 4), (24, 1)):
            CASES.append(("bf16", "bf16", d, bs, H, Hkv))
for bs in (8, 16, 32):
    for (H, Hkv) in ((8, 8), (8, 2), (32, 4), (64, 8), (6, 1)):
        CASES.append(("fp8_e4m3", "bf16", 128, bs, H, Hkv))
        CASES.append(("fp8_e4m3", "f16", 128, bs, H, Hkv))
for bs in (8, 16, 32):
    for (H, Hkv) in ((8, 2), (32, 4), (64, 8), (12, 3), (8, 8), (6, 1)):
        CASES.append(("fp8_e4m3_block", "bf16", 128, bs, H, Hkv))
    CASES.append(("fp8_e4m3_block", "f16", 128, bs, 16, 2))
for (H, Hkv) in ((8, 8), (16, 2)):
    CASES.append(("f16", "f16", 64, 16, H, Hkv))
    CASES.append(("f16", "f16", 128, 32, H, Hkv))
LENS = [1, 2, 7, 8, 9, 63, 64, 65, 127, 200, 511, 513, 1000]


@pytest.mark.parametrize("kv_dtype,dtype,d,bs,H,Hkv", CASES)
def test_ragged_small_cases(P, kv_dtype, dtype, d, bs, H, Hkv):
    seed = zlib.crc32(repr((kv_dtype, dtype, d, bs, H, Hkv)).encode()) % 1000
    cfg, w = small_case(kv_dtype, dtype, d, bs, H, Hkv, LENS, seed=seed)
    kc, vc = initial_pools(w)
    kc_dev, vc_dev = to_device_pool(kc, cfg), to_device_pool(vc, cfg)
    for ps in (0, 64, 192):
        k2, v2 = kc_dev.clone(), vc_dev.clone()
        out, ws = gpu_step(P, w, k2, v2, partition_size=ps)
        kcc, vcc = kc.copy(), vc.copy()
        ref = oracle_step(w, kcc, vcc)
        got = out.double().cpu().numpy()
        assert np.all(np.isfinite(got))
        excess = np.abs(got - ref) - elementwise_bound(ref, kv_dtype, dtype)
        assert np.max(excess) <= 0, f"partition_size={ps}: worst excess {np.max(excess)}"
        assert P.get_device_error(ws) == 0
        assert torch.equal(pool_bits(k2), pool_bits(to_device_pool(kcc, cfg)))
        assert torch.equal(pool_bits(v2), pool_bits(to_device_pool(vcc, cfg)))


def test_fp8_encode_exhaustive_against_oracle(P):
    """Every bf16 and every f16 bit pattern through reshape_and_cache into an E4M3 cache, for several
    scales, bit-exact against the oracle's encoder (IEEE division, RNE, satfinite, NaN kept)."""
    for dtype, tdt in (("bf16", torch.bfloat16), ("f16", torch.float16)):
        bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
        Hkv, d = 4, 128
        T = 65536 // (Hkv * d)
        vals = bits.reshape(T, Hkv, d)
        scales = np.array([1.0, 0.0123, 3.7e-3, 250.0], np.float32)
        kc = np.zeros((T, 1, Hkv, d), np.uint8)
        vc = np.zeros_like(kc)
        slots = np.arange(T, dtype=np.int64)
        oracle.reshape_and_cache(vals, vals, dtype, kc, vc, "fp8_e4m3", slots, scales, scales)
        key = torch.from_numpy(vals.view(np.int16).copy()).view(tdt).cuda()
        kd = torch.zeros((T, 1, Hkv, d), dtype=torch.uint8, device="cuda")
        vd = torch.zeros_like(kd)
        sc = torch.from_numpy(scales).cuda()
        P.reshape_and_cache(key, key, kd, vd, torch.from_numpy(slots).cuda(), sc, sc)
        assert np.array_equal(kd.cpu().numpy(), kc), dtype
        assert np.array_equal(vd.cpu().numpy(), vc), dtype
