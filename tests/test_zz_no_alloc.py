"""The no-allocation entry point, pa_paged_attention_static, against pa_paged_attention.

Some callers cannot allocate device memory: plugins hosted by an engine that owns all device memory,
and serving loops that must not allocate once they run. pa_paged_attention_static serves them with a
fixed scratch array inside the library. Here it is called through the C ABI twice in a row, on two
different batches whose split-K partials need that scratch. Both entry points run the same kernels
with the same plan, so each output must equal the allocating entry point's (caller workspace) bit for
bit, and the oracle's within the bf16 tolerance the other tests use. The device error word must be
handed out and then cleared, and a warm call must take no device memory.
This file is collected last so that a run stopping at the first failure has run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from helpers import bits16

pytestmark = pytest.mark.gpu

TOLERANCE_BF16 = 1e-2
PARTITION = 512


def static_call(P, out, w, cfg, lens, mcl, err):
    P.paged_attention_static(out, w.query, w.key_values, w.value_values, w.block_tables, lens,
                             cfg.softmax_scale, mcl, partition_size=PARTITION, device_error_out=err)


def test_static_scratch_matches_caller_workspace_on_two_calls_in_a_row():
    from pagedattention_paged_kv_attention_b200 import pagedattn as P

    cfg = W.CONFIGS["long_splitk"]
    for seed in (11, 12):
        w = W.make_workload(cfg, seed=seed, num_seqs=3, device="cuda", prefilled=True)
        S, H, d = w.query.shape
        mcl = int(w.context_lens.max())
        assert P.workspace_size(S, H, cfg.num_kv_heads, d, mcl, PARTITION) > P.WORKSPACE_HEADER_BYTES
        ws = P.make_workspace(S, H, cfg.num_kv_heads, d, mcl, PARTITION)
        ref = torch.empty_like(w.query)
        P.paged_attention(ref, w.query, w.key_values, w.value_values, w.block_tables, w.context_lens,
                          cfg.softmax_scale, mcl, ws, partition_size=PARTITION)
        out = torch.full_like(w.query, float("nan"))
        err = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
        static_call(P, out, w, cfg, w.context_lens, mcl, err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), "static and caller workspace differ"
        expect = oracle.paged_attention(bits16(w.query), cfg.dtype, bits16(w.key_values), bits16(w.value_values),
                                        cfg.kv_dtype, w.block_tables.cpu().numpy(), w.context_lens.cpu().numpy(),
                                        cfg.softmax_scale)
        assert np.max(np.abs(out.double().cpu().numpy() - expect)) <= TOLERANCE_BF16


def test_static_error_word_is_handed_out_then_cleared_and_nothing_is_allocated():
    from pagedattention_paged_kv_attention_b200 import pagedattn as P

    cfg = W.CONFIGS["long_splitk"]
    w = W.make_workload(cfg, seed=13, num_seqs=3, device="cuda", prefilled=True)
    mcl = int(w.context_lens.max())
    bad_lens = w.context_lens.clone()
    bad_lens[1] = w.block_tables.shape[1] * cfg.block_size + 1   # past its table: NaN row + error bit
    out = torch.empty_like(w.query)
    err = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
    static_call(P, out, w, cfg, bad_lens, max(mcl, int(bad_lens.max())), err)
    torch.cuda.synchronize()
    assert int(err.item()) & P.PA_DEVERR_CONTEXT_LEN
    assert torch.isnan(out[1].float()).all() and torch.isfinite(out[0].float()).all()
    # The next clean call starts from a cleared word; a warm call takes no device memory.
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    static_call(P, out, w, cfg, w.context_lens, mcl, err)
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    assert int(err.item()) == 0
    assert torch.isfinite(out.float()).all()
    assert free_after == free_before, (free_before, free_after)


def test_static_scratch_rejects_requests_beyond_its_size():
    from pagedattention_paged_kv_attention_b200 import pagedattn as P

    S, H, Hkv, d, mcl = 2048, 64, 8, 128, 32768
    assert P.workspace_size(S, H, Hkv, d, mcl, 64) > (32 << 20)
    status = P.lib.pa_paged_attention_static(16, 16, P.PA_BF16, 16, 16, P.PA_BF16, None, None, 16, 512, 16, S, H,
                                             Hkv, d, 16, 100, mcl, 0.1, 64, None, None)
    assert status == P.PA_ERR_WORKSPACE_TOO_SMALL
