"""The multi-layer cache ops on the GPU, bit-exact against the oracle applied layer by layer:
reshape_and_cache_layers writes every layer's new tokens into that layer's pools in one launch, and
copy_blocks_layers applies one copy-on-write mapping to every layer's pools in one launch. Each
layer has its own pool contents, inputs and (FP8) scales, so a layer index mix-up shows."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from helpers import bits16
from steps import initial_pools, pool_bits, to_device_pool

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,layers", [("tiny", 3), ("7b", 4), ("shared_prefix_fp8", 5)])
def test_layers_match_oracle_per_layer(name, layers):
    from pagedattention_paged_kv_attention_b200 import pagedattn as P
    cfg = dataclasses.replace(W.CONFIGS[name], num_blocks=None, cow_pairs=max(W.CONFIGS[name].cow_pairs, 8))
    base = W.make_workload(cfg, num_seqs=min(cfg.num_seqs, 16), placement_seed=99)
    lens = base.context_lens.tolist()
    # Other layers: same lengths and placement (so the same slots and cow pairs), other values.
    ws = [base] + [W.make_workload(cfg, seed=cfg.seed + 17 * l, context_lens=lens, placement_seed=99)
                   for l in range(1, layers)]
    for w in ws[1:]:
        assert torch.equal(w.slot_mapping, base.slot_mapping) and torch.equal(w.cow_mapping, base.cow_mapping)
    pools = [initial_pools(w) for w in ws]
    dk = [to_device_pool(k, cfg) for k, _ in pools]
    dv = [to_device_pool(v, cfg) for _, v in pools]
    fp8 = cfg.kv_dtype == "fp8_e4m3"
    ks = [w.k_scale.cuda() for w in ws] if fp8 else None
    vs = [w.v_scale.cuda() for w in ws] if fp8 else None
    slots = base.slot_mapping.cuda()
    keep2 = P.copy_blocks_layers(dk, dv, base.cow_mapping.cuda())     # copy-on-write, then the new tokens
    keep = P.reshape_and_cache_layers([w.new_key.cuda() for w in ws], [w.new_value.cuda() for w in ws], dk, dv,
                                      slots, ks, vs)
    torch.cuda.synchronize()
    del keep, keep2
    for l, w in enumerate(ws):
        kc, vc = pools[l]
        sk = None if not fp8 else w.k_scale.numpy()
        sv = None if not fp8 else w.v_scale.numpy()
        oracle.copy_blocks(kc, vc, cfg.kv_dtype, base.cow_mapping.numpy())
        oracle.reshape_and_cache(bits16(w.new_key), bits16(w.new_value), cfg.dtype, kc, vc, cfg.kv_dtype,
                                 base.slot_mapping.numpy(), sk, sv)
        assert torch.equal(pool_bits(dk[l]), pool_bits(to_device_pool(kc, cfg))), f"layer {l}: key pool"
        assert torch.equal(pool_bits(dv[l]), pool_bits(to_device_pool(vc, cfg))), f"layer {l}: value pool"


def test_layers_empty_and_invalid():
    from pagedattention_paged_kv_attention_b200 import pagedattn as P
    kc = [torch.zeros((4, 16, 2, 64), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    vc = [torch.zeros_like(k) for k in kc]
    P.copy_blocks_layers(kc, vc, torch.zeros((0, 2), dtype=torch.int64, device="cuda"))   # no pairs: no-op
    empty = torch.zeros((0, 2, 64), dtype=torch.bfloat16, device="cuda")
    P.reshape_and_cache_layers([empty, empty], [empty, empty], kc, vc,
                               torch.zeros((0,), dtype=torch.int64, device="cuda"))
    torch.cuda.synchronize()
    assert all(int(k.abs().sum()) == 0 for k in kc + vc)
    # FP8 caches without scale arrays are refused before any launch
    k8 = [torch.zeros((4, 16, 2, 128), dtype=torch.uint8, device="cuda")]
    x = torch.zeros((1, 2, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(P.PagedAttnError) as e:
        P.reshape_and_cache_layers([x], [x], k8, k8, torch.zeros((1,), dtype=torch.int64, device="cuda"))
    assert e.value.status == P.PA_ERR_INVALID_ARGUMENT
