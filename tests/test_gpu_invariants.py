"""GPU invariants and edge cases of the library (no oracle needed for the bitwise ones).

* moving physical blocks (a second placement of the same logical data) leaves the output bitwise
  identical, and so do repeated runs (determinism);
* a context of one token returns that token's value exactly; equal keys give the mean of V;
* sequences that share prefix blocks give bitwise the same output as private copies of the blocks;
* a block id outside the pool and a context longer than its table set the device error word and
  NaN the affected rows without faulting; every other row stays correct;
* block-table entries past ceil(L / block_size) may hold anything (decode and prefill);
* empty batches and zero-length contexts.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from helpers import bits16
from steps import TOLERANCE, gpu_step, initial_pools, oracle_step, to_device_pool

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    from pagedattention_paged_kv_attention_b200 import pagedattn
    return pagedattn


def run(P, w, **kw):
    kc, vc = initial_pools(w)
    out, ws = gpu_step(P, w, to_device_pool(kc, w.cfg), to_device_pool(vc, w.cfg), **kw)
    torch.cuda.synchronize()
    return out, ws


@pytest.mark.parametrize("name", ["7b", "70b_gqa", "shared_prefix_fp8"])
def test_block_placement_invariance_and_determinism(P, name):
    cfg = W.CONFIGS[name]
    a = W.make_workload(cfg, num_seqs=24, prefilled=True)
    b = W.make_workload(cfg, num_seqs=24, prefilled=True, placement_seed=1234)
    assert not torch.equal(a.block_tables, b.block_tables)
    oa, _ = run(P, a, write_new=False, copy=False)
    ob, _ = run(P, b, write_new=False, copy=False)
    oa2, _ = run(P, a, write_new=False, copy=False)
    assert torch.equal(oa.view(torch.int16), ob.view(torch.int16))
    assert torch.equal(oa.view(torch.int16), oa2.view(torch.int16))


def test_single_token_returns_its_value_exactly(P):
    cfg = W.CONFIGS["70b_gqa"]
    w = W.make_workload(cfg, context_lens=[1] * 8)
    out, ws = run(P, w)      # the step writes the one token, then attends to it
    G = cfg.num_heads // cfg.num_kv_heads
    expect = w.new_value.cuda().repeat_interleave(G, dim=1)
    assert torch.equal(out.view(torch.int16), expect.view(torch.int16))


def test_equal_keys_give_mean_of_values(P):
    cfg = W.CONFIGS["7b"]
    w = W.make_workload(cfg, num_seqs=4, prefilled=True)
    kc, vc = initial_pools(w)
    kc[...] = bits16(torch.tensor([0.5], dtype=torch.bfloat16))[0]
    out, _ = gpu_step(P, w, to_device_pool(kc, cfg), to_device_pool(vc, cfg), write_new=False)
    vals = w.value_values.double()
    for s in range(4):
        L = int(w.context_lens[s])
        rows = []
        for t in range(L):
            rows.append(vals[int(w.block_tables[s, t // cfg.block_size]), t % cfg.block_size])
        mean = torch.stack(rows).mean(0).numpy()          # [Hkv, d]
        got = out[s].double().cpu().numpy()
        assert np.max(np.abs(got - mean)) <= 2 ** -8


def test_shared_prefix_equals_private_copies(P):
    cfg = W.CONFIGS["shared_prefix_fp8"]
    w = W.make_workload(cfg, num_seqs=8, prefilled=True)
    kc, vc = initial_pools(w)
    k_dev, v_dev = to_device_pool(kc, cfg), to_device_pool(vc, cfg)
    shared, _ = gpu_step(P, w, k_dev, v_dev, write_new=False, copy=False)
    # give sequence 0 private copies of the prefix blocks (copy-on-write destinations)
    pairs = w.cow_mapping
    P.copy_blocks(k_dev, v_dev, pairs.cuda())
    tables = w.block_tables.clone()
    prefix = cfg.shared_prefix_tokens // cfg.block_size
    tables[0, :prefix] = pairs[:prefix, 1].to(torch.int32)
    private, _ = gpu_step(P, w, k_dev, v_dev, write_new=False, copy=False, block_tables=tables)
    assert torch.equal(shared.view(torch.int16), private.view(torch.int16))


def test_bad_block_id_and_bad_length_are_reported(P):
    cfg = W.CONFIGS["70b_gqa"]
    w = W.make_workload(cfg, num_seqs=6, prefilled=True)
    kc, vc = initial_pools(w)
    ref = oracle_step(w, kc.copy(), vc.copy(), write_new=False)
    tables = w.block_tables.clone()
    tables[1, 3] = w.num_blocks + 5           # outside the pool
    tables[2, 0] = -7
    lens = w.context_lens.clone()
    lens[4] = tables.shape[1] * cfg.block_size + 1   # longer than its table
    mcl = int(lens.max())
    out, ws = gpu_step(P, w, to_device_pool(kc, cfg), to_device_pool(vc, cfg), write_new=False,
                       block_tables=tables, context_lens=lens, max_context_len=mcl)
    err = P.get_device_error(ws)
    assert err & P.PA_DEVERR_BLOCK_ID and err & P.PA_DEVERR_CONTEXT_LEN
    o = out.double().cpu().numpy()
    for s in (1, 2, 4):
        assert np.all(np.isnan(o[s])), s
    for s in (0, 3, 5):
        assert np.max(np.abs(o[s] - ref[s])) <= TOLERANCE["bf16"]
    P.clear_device_error(ws)
    assert P.get_device_error(ws) == 0


def test_zero_length_contexts_and_empty_batch(P):
    cfg = W.CONFIGS["tiny"]
    w = W.make_workload(cfg, context_lens=[0, 5, 0, 17])
    kc, vc = initial_pools(w)
    out, ws = gpu_step(P, w, to_device_pool(kc, cfg), to_device_pool(vc, cfg))
    ref = oracle_step(w, kc, vc)
    o = out.double().cpu().numpy()
    assert np.all(o[0] == 0) and np.all(o[2] == 0)
    assert np.max(np.abs(o - ref)) <= TOLERANCE["f16"]
    # an empty batch is a no-op
    q = torch.empty((0, 8, 64), dtype=torch.float16, device="cuda")
    P.paged_attention(torch.empty_like(q), q, to_device_pool(kc, cfg), to_device_pool(vc, cfg),
                      torch.zeros((0, 4), dtype=torch.int32, device="cuda"),
                      torch.zeros((0,), dtype=torch.int32, device="cuda"), 0.125, 0, ws)
    torch.cuda.synchronize()


def test_copy_blocks_touches_only_destinations(P):
    cfg = W.CONFIGS["shared_prefix_fp8"]
    w = W.make_workload(cfg, num_seqs=32)
    kc, vc = initial_pools(w)
    k_dev, v_dev = to_device_pool(kc, cfg), to_device_pool(vc, cfg)
    P.copy_blocks(k_dev, v_dev, w.cow_mapping.cuda())
    oracle.copy_blocks(kc, vc, "fp8_e4m3", w.cow_mapping.numpy())
    assert np.array_equal(k_dev.cpu().numpy(), kc) and np.array_equal(v_dev.cpu().numpy(), vc)
    assert P.copy_blocks_check(w.cow_mapping, w.num_blocks)
    bad = w.cow_mapping.clone()
    bad[1, 1] = bad[0, 0]                      # a destination that is also a source
    assert not P.copy_blocks_check(bad, w.num_blocks)


def poisoned_past_context(tables, lens, block_size, num_blocks, extra=160):
    """The block tables widened by `extra` columns, with every entry past ceil(L / block_size) of each
    row replaced by ids outside the pool (negative, past the pool, INT32_MAX)."""
    S, mb = tables.shape
    wide = torch.empty((S, mb + extra), dtype=torch.int32)
    wide[:, :mb] = tables
    bad = torch.tensor([-1, num_blocks, 2 ** 31 - 1, -(2 ** 31)], dtype=torch.int32)
    for s in range(S):
        need = -(-int(lens[s]) // block_size)
        wide[s, need:] = bad.repeat((mb + extra - need) // 4 + 1)[:mb + extra - need]
    return wide


@pytest.mark.parametrize("name", ["7b", "70b_gqa", "long_splitk"])
def test_table_entries_past_the_context_are_not_used(P, name):
    """Only the first ceil(L / block_size) entries of a table row are read: poisoning the rest with
    ids outside the pool changes no output bit and sets no error bit."""
    cfg = W.CONFIGS[name]
    w = W.make_workload(cfg, num_seqs=min(10, cfg.num_seqs), prefilled=True)
    wide = poisoned_past_context(w.block_tables, w.context_lens, cfg.block_size, w.num_blocks)
    ref, ws_ref = run(P, w, write_new=False, copy=False, partition_size=cfg.partition_size)
    out, ws = run(P, w, write_new=False, copy=False, partition_size=cfg.partition_size, block_tables=wide)
    assert P.get_device_error(ws) == 0 and P.get_device_error(ws_ref) == 0
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_prefill_table_entries_past_the_context_are_not_used(P):
    cfg = W.PREFILL_CONFIGS["prefill_tiny"]
    w = W.make_prefill_workload(cfg)
    dev = torch.device("cuda")
    kc, vc = w.key_values.to(dev), w.value_values.to(dev)
    P.reshape_and_cache(w.new_key.to(dev), w.new_value.to(dev), kc, vc, w.slot_mapping.to(dev))
    q = w.query.to(dev)
    outs = []
    for tables in (w.block_tables, poisoned_past_context(w.block_tables, w.context_lens, cfg.block_size,
                                                         w.num_blocks)):
        out = torch.full_like(q, float("nan"))
        ws = torch.zeros(64, dtype=torch.int32, device=dev)
        P.paged_prefill(out, q, kc, vc, tables.to(dev), w.context_lens.to(dev), w.q_start.to(dev),
                        cfg.softmax_scale, w.max_q_len, ws)
        torch.cuda.synchronize()
        assert P.get_device_error(ws) == 0
        outs.append(out)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
