"""One decode step (copy_blocks -> reshape_and_cache -> paged_attention) run two ways on the same
seeded inputs: through the oracle on the CPU, and through the C-ABI library on the GPU.

Test infrastructure: the GPU side gets its inputs from the generator (and, for FP8 caches, the
oracle's quantised pool); nothing flows from the GPU into the oracle.
"""
import numpy as np
import torch

import oracle
from helpers import bits16

TOLERANCE = {"f16": 2e-3, "bf16": 1e-2, "fp8_e4m3": 3e-2, "fp8_e4m3_block": 3e-2}   # max-abs, per cache format
MANTISSA_BITS = {"f16": 10, "bf16": 7}


def elementwise_bound(ref, cache_dtype, out_dtype):
    """Per-element bound for cases outside the workload table: the stated max-abs tolerance plus half
    an ulp of the output dtype at the reference's magnitude. Contexts of a few tokens give outputs up
    to about 5 in magnitude, where rounding to bf16 alone moves a value by up to 2^-6 = 0.0156."""
    mag = np.maximum(np.abs(ref), 2.0 ** -14)
    half_ulp = np.exp2(np.floor(np.log2(mag)) - MANTISSA_BITS[out_dtype] - 1)
    return TOLERANCE[cache_dtype] + half_ulp


def initial_pools(w):
    """The cache contents before the step, as oracle arrays (uint16 bits, or E4M3 codes)."""
    cfg = w.cfg
    kb = bits16(w.key_values)
    vb = bits16(w.value_values)
    if cfg.kv_dtype == "fp8_e4m3":
        kb = oracle.quantize_e4m3(kb, cfg.dtype, w.k_scale.numpy())
        vb = oracle.quantize_e4m3(vb, cfg.dtype, w.v_scale.numpy())
    elif cfg.kv_dtype == "fp8_e4m3_block":
        kb = oracle.quantize_e4m3_blocks(kb, cfg.dtype, w.k_scale.numpy())
        vb = oracle.quantize_e4m3_blocks(vb, cfg.dtype, w.v_scale.numpy())
    return kb, vb


def oracle_step(w, kc, vc, write_new=True, copy=True):
    """Mutates kc/vc (numpy) like the step does; returns the fp64 attention output."""
    cfg = w.cfg
    ks = None if w.k_scale is None else w.k_scale.numpy()
    vs = None if w.v_scale is None else w.v_scale.numpy()
    if copy and w.cow_mapping.shape[0]:
        oracle.copy_blocks(kc, vc, cfg.kv_dtype, w.cow_mapping.numpy())
    if write_new:
        oracle.reshape_and_cache(bits16(w.new_key), bits16(w.new_value), cfg.dtype, kc, vc, cfg.kv_dtype,
                                 w.slot_mapping.numpy(), ks, vs)
    return oracle.paged_attention(bits16(w.query), cfg.dtype, kc, vc, cfg.kv_dtype, w.block_tables.numpy(),
                                  w.context_lens.numpy(), cfg.softmax_scale, ks, vs)


def to_device_pool(arr, cfg):
    if cfg.kv_dtype.startswith("fp8"):
        return torch.from_numpy(arr).cuda()                       # uint8 codes
    t = torch.from_numpy(arr.view(np.int16)).cuda()
    return t.view(torch.bfloat16 if cfg.kv_dtype == "bf16" else torch.float16)


def pool_bits(t):
    """Device pool -> raw integer view for byte comparison."""
    return t if t.dtype == torch.uint8 else t.view(torch.int16)


def gpu_step(P, w, kc_dev, vc_dev, write_new=True, copy=True, partition_size=0, workspace=None,
             block_tables=None, context_lens=None, max_context_len=None):
    """Runs the step through the library on the GPU; mutates kc_dev/vc_dev; returns out (device)."""
    cfg = w.cfg
    dev = kc_dev.device
    ks = None if w.k_scale is None else w.k_scale.to(dev)
    vs = None if w.v_scale is None else w.v_scale.to(dev)
    if copy and w.cow_mapping.shape[0]:
        P.copy_blocks(kc_dev, vc_dev, w.cow_mapping.to(dev))
    if write_new:
        P.reshape_and_cache(w.new_key.to(dev), w.new_value.to(dev), kc_dev, vc_dev, w.slot_mapping.to(dev), ks, vs)
    bt = (w.block_tables if block_tables is None else block_tables).to(dev)
    cl = (w.context_lens if context_lens is None else context_lens).to(dev)
    mcl = int(cl.max().item()) if max_context_len is None and cl.numel() else (max_context_len or 0)
    q = w.query.to(dev)
    out = torch.empty_like(q)
    S, H, d = q.shape
    if workspace is None:
        workspace = P.make_workspace(S, H, cfg.num_kv_heads, d, mcl, partition_size, device=dev)
    P.paged_attention(out, q, kc_dev, vc_dev, bt, cl, cfg.softmax_scale, mcl, workspace, ks, vs,
                      partition_size=partition_size)
    return out, workspace
