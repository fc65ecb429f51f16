"""The native block manager driving the device path through a serving session: prompts written
through add_sequence's slots, a prefix shared between requests, beam-style forks, copy-on-write,
a swap to pinned host memory and back, and a finished sequence released. Every decode step runs
copy_blocks -> reshape_and_cache -> paged_attention on the GPU with the manager's plan, and its
output is compared with the oracle's attention over each sequence's LOGICAL history, laid out in
an identity block table of its own (so the reference depends on none of the manager's decisions).
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import bits16
from steps import TOLERANCE

pytestmark = pytest.mark.gpu

H, HKV, D, BS, NB, NH = 8, 2, 128, 16, 48, 24


def logical_reference(query, hist_k, hist_v, seqs, scale):
    """Oracle attention over each sequence's history in a fresh identity layout."""
    lens = [len(hist_k[s]) for s in seqs]
    width = max(-(-L // BS) for L in lens)
    pool_k = np.zeros((len(seqs) * width, BS, HKV, D), np.uint16)
    pool_v = np.zeros_like(pool_k)
    tables = np.zeros((len(seqs), width), np.int32)
    for i, s in enumerate(seqs):
        k = bits16(torch.stack(hist_k[s]))
        v = bits16(torch.stack(hist_v[s]))
        for t in range(lens[i]):
            pool_k[i * width + t // BS, t % BS] = k[t]
            pool_v[i * width + t // BS, t % BS] = v[t]
        tables[i] = np.arange(i * width, (i + 1) * width)
    return oracle.paged_attention(bits16(query), "bf16", pool_k, pool_v, "bf16", tables,
                                  np.array(lens, np.int32), scale)


def test_session_driven_by_block_manager():
    from pagedattention_paged_kv_attention_b200 import pagedattn as P
    from pagedattention_paged_kv_attention_b200.block_manager import BlockManager
    g = torch.Generator().manual_seed(7)
    dev = torch.device("cuda")
    kc = torch.zeros((NB, BS, HKV, D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    host_k = torch.zeros((NH, BS, HKV, D), dtype=torch.bfloat16).pin_memory()
    host_v = torch.zeros_like(host_k).pin_memory()
    bm = BlockManager(NB, BS, NH)
    hist_k, hist_v = {}, {}
    scale = D ** -0.5

    def rows(n):
        return [torch.randn((HKV, D), generator=g).to(torch.bfloat16) for _ in range(n)]

    def write(seq, slots, ks, vs):
        if len(slots):
            P.reshape_and_cache(torch.stack(ks).to(dev), torch.stack(vs).to(dev), kc, vc,
                                torch.from_numpy(np.ascontiguousarray(slots)).to(dev))

    # Request 0: a 40-token prompt.
    hist_k[0], hist_v[0] = rows(40), rows(40)
    write(0, bm.add_sequence(0, 40), hist_k[0], hist_v[0])
    # Request 1 shares the first 37 prompt tokens of request 0; only the 2 full blocks are shared, so
    # tokens 32..49 are written (32..36 equal to request 0's).
    k1, v1 = rows(13), rows(13)
    hist_k[1], hist_v[1] = hist_k[0][:37] + k1, hist_v[0][:37] + v1
    slots = bm.add_sequence(1, 50, 0, 37)
    assert len(slots) == 50 - 32
    write(1, slots, hist_k[1][32:], hist_v[1][32:])
    assert bm.ref_count(int(bm.block_tables([0], 3)[0][0, 0])) == 2
    # A beam of request 0.
    bm.fork(0, 2)
    hist_k[2], hist_v[2] = list(hist_k[0]), list(hist_v[0])

    swapped, cow_seen, ws = set(), 0, None
    for step in range(24):
        if step == 4:
            bm.fork(1, 3)
            hist_k[3], hist_v[3] = list(hist_k[1]), list(hist_v[1])
        if step == 8:                                             # preempt beam 2
            m = bm.swap_out(2)
            P.swap_blocks(host_k, host_v, kc, vc, torch.from_numpy(m).to(dev))
            swapped.add(2)
        if step == 13:
            m = bm.swap_in(2)
            P.swap_blocks(kc, vc, host_k, host_v, torch.from_numpy(m).pin_memory())
            swapped.discard(2)
        if step == 17:                                            # request 0 finishes
            bm.free_sequence(0)
            del hist_k[0], hist_v[0]
        seqs = sorted(s for s in hist_k if s not in swapped)
        slots, cow, tables, lens = bm.plan_decode(seqs, max_blocks=8, pad=0)
        cow_seen += len(cow)
        nk, nv = rows(len(seqs)), rows(len(seqs))
        for s, a, b in zip(seqs, nk, nv):
            hist_k[s].append(a)
            hist_v[s].append(b)
        if len(cow):
            P.copy_blocks(kc, vc, torch.from_numpy(np.ascontiguousarray(cow)).to(dev))
        write(None, slots, nk, nv)
        q = torch.randn((len(seqs), H, D), generator=g).to(torch.bfloat16)
        out = torch.empty((len(seqs), H, D), dtype=torch.bfloat16, device=dev)
        mcl = int(lens.max())
        ws = P.make_workspace(len(seqs), H, HKV, D, mcl)
        P.paged_attention(out, q.to(dev), kc, vc, torch.from_numpy(tables).to(dev),
                          torch.from_numpy(lens).to(dev), scale, mcl, ws)
        torch.cuda.synchronize()
        assert P.get_device_error(ws) == 0
        ref = logical_reference(q, hist_k, hist_v, seqs, scale)
        err = float(np.max(np.abs(out.double().cpu().numpy() - ref)))
        assert err <= TOLERANCE["bf16"], f"step {step}: max-abs error {err}"
        assert lens.tolist() == [len(hist_k[s]) for s in seqs]
    assert cow_seen >= 2                                          # the forks forced copies
    assert bm.num_free_blocks()[1] == NH                          # host pool back to empty
