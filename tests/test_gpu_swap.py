"""swap_blocks on the GPU, bit-exact against the oracle: swap-out of blocks from a device pool to a
pinned host pool, swap-in back to other device blocks, round trip, untouched blocks unchanged, and
pageable host memory refused before any launch."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from steps import initial_pools, to_device_pool

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["7b", "shared_prefix_fp8"])
def test_swap_out_and_in_match_oracle(name):
    from pagedattention_paged_kv_attention_b200 import pagedattn as P
    import dataclasses
    cfg = dataclasses.replace(W.CONFIGS[name], num_blocks=None)   # pool sized to the batch
    w = W.make_workload(cfg, num_seqs=8)
    kc, vc = initial_pools(w)                                   # oracle-side pools
    dk, dv = to_device_pool(kc, cfg), to_device_pool(vc, cfg)
    n_host = 96
    host_k = torch.zeros((n_host,) + tuple(dk.shape[1:]), dtype=dk.dtype).pin_memory()
    host_v = torch.zeros_like(host_k).pin_memory()
    rng = np.random.default_rng(1)
    src = w.used_blocks.numpy()[rng.permutation(len(w.used_blocks))[:64]]
    dst = rng.permutation(n_host)[:64]
    out_map = np.stack([src, dst], 1).astype(np.int64)
    # swap-out: device -> pinned host (mapping in device memory)
    P.swap_blocks(host_k, host_v, dk, dv, torch.from_numpy(out_map).cuda())
    torch.cuda.synchronize()
    ok, ov = np.zeros((n_host,) + kc.shape[1:], kc.dtype), np.zeros((n_host,) + vc.shape[1:], vc.dtype)
    oracle.swap_blocks(ok, ov, kc, vc, cfg.kv_dtype, out_map)
    hk = host_k.view(torch.uint8 if host_k.dtype == torch.uint8 else torch.int16).numpy().view(kc.dtype)
    hv = host_v.view(torch.uint8 if host_v.dtype == torch.uint8 else torch.int16).numpy().view(vc.dtype)
    assert np.array_equal(hk, ok) and np.array_equal(hv, ov)
    # swap-in: pinned host -> other device blocks (mapping in pinned host memory)
    free = np.setdiff1d(np.arange(w.num_blocks), w.used_blocks.numpy())[:64]
    in_map = np.stack([dst, free], 1).astype(np.int64)
    dk2, dv2 = dk.clone(), dv.clone()
    P.swap_blocks(dk2, dv2, host_k, host_v, torch.from_numpy(in_map).pin_memory())
    torch.cuda.synchronize()
    ek, ev = kc.copy(), vc.copy()
    oracle.swap_blocks(ek, ev, ok, ov, cfg.kv_dtype, in_map)
    assert torch.equal(dk2.cpu().view(-1).view(torch.uint8), torch.from_numpy(ek.view(np.uint8).reshape(-1)))
    assert torch.equal(dv2.cpu().view(-1).view(torch.uint8), torch.from_numpy(ev.view(np.uint8).reshape(-1)))
    # round trip: the swapped-in blocks equal the originals
    assert np.array_equal(ek[free], kc[src]) and np.array_equal(ev[free], vc[src])


def test_pageable_host_memory_is_refused():
    from pagedattention_paged_kv_attention_b200 import pagedattn as P
    dk = torch.zeros((4, 16, 2, 64), dtype=torch.bfloat16, device="cuda")
    host = torch.zeros((4, 16, 2, 64), dtype=torch.bfloat16)          # pageable
    m = torch.tensor([[0, 1]], dtype=torch.int64, device="cuda")
    with pytest.raises(P.PagedAttnError) as e:
        P.swap_blocks(host, host, dk, dk, m)
    assert e.value.status == P.PA_ERR_INVALID_ARGUMENT
