"""Guard bytes around every buffer a kernel writes (GPU): each pool, output and host pool is the middle
of a larger allocation whose margins hold a fixed byte pattern. After reshape_and_cache (slots at the
pool's first and last positions, padding and past-the-pool slots), the multi-layer variants,
copy_blocks (first and last blocks), swap_blocks in both directions, decode attention and prefill
attention, every margin byte must be unchanged."""
import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu
PATTERN = 0xA5
MARGIN = 4096  # bytes on each side


def guarded(shape, dtype, device="cuda", pin=False):
    """(buffer, view): a view of `shape` in the middle of a byte buffer with PATTERN margins."""
    elem = torch.empty((), dtype=dtype).element_size()
    n = int(np.prod(shape)) * elem
    buf = torch.full((n + 2 * MARGIN,), PATTERN, dtype=torch.uint8)
    buf = buf.pin_memory() if pin else buf.to(device)
    view = buf[MARGIN:MARGIN + n].view(dtype).view(shape)
    return buf, view


def margins_intact(buf):
    b = buf.cpu()
    return bool((b[:MARGIN] == PATTERN).all()) and bool((b[-MARGIN:] == PATTERN).all())


def test_write_kernels_stay_inside_their_buffers():
    from pagedattention_paged_kv_attention_b200 import pagedattn as P
    NB, bs, Hkv, d, T = 16, 16, 4, 128, 6
    kbuf, kc = guarded((NB, bs, Hkv, d), torch.bfloat16)
    vbuf, vc = guarded((NB, bs, Hkv, d), torch.bfloat16)
    kc.normal_(); vc.normal_()
    x = torch.randn(T, Hkv, d, device="cuda").to(torch.bfloat16)
    slots = torch.tensor([0, NB * bs - 1, -1, NB * bs, 37, 100], dtype=torch.int64, device="cuda")
    P.reshape_and_cache(x, x, kc, vc, slots)
    P.copy_blocks(kc, vc, torch.tensor([[0, NB - 1], [5, 3]], dtype=torch.int64, device="cuda"))
    # FP8 pool with per-block scales.
    k8buf, k8 = guarded((NB, bs, Hkv, d), torch.uint8)
    v8buf, v8 = guarded((NB, bs, Hkv, d), torch.uint8)
    sc = torch.full((NB, Hkv), 0.02, device="cuda")
    P.reshape_and_cache(x, x, k8, v8, slots, sc, sc)
    # Two layers in one launch.
    lb = [guarded((NB, bs, Hkv, d), torch.bfloat16) for _ in range(4)]
    keep = P.reshape_and_cache_layers([x, x], [x, x], [lb[0][1], lb[1][1]], [lb[2][1], lb[3][1]], slots)
    keep2 = P.copy_blocks_layers([lb[0][1], lb[1][1]], [lb[2][1], lb[3][1]],
                                 torch.tensor([[0, NB - 1]], dtype=torch.int64, device="cuda"))
    # Swap out to a guarded pinned host pool and back.
    hkbuf, hk = guarded((4, bs, Hkv, d), torch.bfloat16, pin=True)
    hvbuf, hv = guarded((4, bs, Hkv, d), torch.bfloat16, pin=True)
    P.swap_blocks(hk, hv, kc, vc, torch.tensor([[0, 0], [NB - 1, 3]], dtype=torch.int64, device="cuda"))
    P.swap_blocks(kc, vc, hk, hv, torch.tensor([[3, 5], [0, NB - 1]], dtype=torch.int64, device="cuda"))
    torch.cuda.synchronize()
    del keep, keep2
    for name, buf in [("key", kbuf), ("value", vbuf), ("fp8 key", k8buf), ("fp8 value", v8buf),
                      ("host key", hkbuf), ("host value", hvbuf)] + [(f"layer pool {i}", b) for i, (b, _) in enumerate(lb)]:
        assert margins_intact(buf), f"{name}: a margin byte changed"


def test_attention_outputs_stay_inside_their_buffers():
    from pagedattention_paged_kv_attention_b200 import pagedattn as P
    cfg = W.CONFIGS["tiny"]
    w = W.make_workload(cfg, prefilled=True)
    dev = torch.device("cuda")
    kc, vc = w.key_values.to(dev), w.value_values.to(dev)
    S, H, d = w.query.shape
    obuf, out = guarded((S, H, d), w.query.dtype)
    mcl = int(w.context_lens.max())
    for ps in (0, 64):
        ws = P.make_workspace(S, H, cfg.num_kv_heads, d, mcl, ps)
        P.paged_attention(out, w.query.to(dev), kc, vc, w.block_tables.to(dev), w.context_lens.to(dev),
                          cfg.softmax_scale, mcl, ws, partition_size=ps)
    pcfg = W.PREFILL_CONFIGS["prefill_tiny"]
    pw = W.make_prefill_workload(pcfg)
    pk, pv = pw.key_values.to(dev), pw.value_values.to(dev)
    P.reshape_and_cache(pw.new_key.to(dev), pw.new_value.to(dev), pk, pv, pw.slot_mapping.to(dev))
    pobuf, pout = guarded(tuple(pw.query.shape), pw.query.dtype)
    pws = torch.zeros(64, dtype=torch.int32, device=dev)
    P.paged_prefill(pout, pw.query.to(dev), pk, pv, pw.block_tables.to(dev), pw.context_lens.to(dev),
                    pw.q_start.to(dev), pcfg.softmax_scale, pw.max_q_len, pws)
    torch.cuda.synchronize()
    assert margins_intact(obuf), "decode output margin changed"
    assert margins_intact(pobuf), "prefill output margin changed"
    assert torch.isfinite(out.float()).all() and torch.isfinite(pout.float()).all()
