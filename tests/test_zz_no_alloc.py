"""The no-allocation entry point, pa_paged_attention_static, against pa_paged_attention.

Some callers cannot allocate device memory: plugins hosted by an engine that owns all device memory,
and serving loops that must not allocate once they run. pa_paged_attention_static serves them with a
fixed scratch array inside the library. Here it is called through the C ABI twice in a row, on two
different batches whose split-K partials need that scratch, and each output is checked against the
allocating entry point (caller workspace) within the bf16 tolerance the other tests use.
This file is collected last so that a run stopping at the first failure has run every other test.
"""
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

TOLERANCE_BF16 = 1e-2
PARTITION = 512


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
        P.paged_attention_static(out, w.query, w.key_values, w.value_values, w.block_tables, w.context_lens,
                                 cfg.softmax_scale, mcl, partition_size=PARTITION, device_error_out=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert torch.isfinite(out).all()
        assert (out.float() - ref.float()).abs().max().item() <= TOLERANCE_BF16


def test_static_scratch_rejects_requests_beyond_its_size():
    from pagedattention_paged_kv_attention_b200 import pagedattn as P

    S, H, Hkv, d, mcl = 2048, 64, 8, 128, 32768
    assert P.workspace_size(S, H, Hkv, d, mcl, 64) > (32 << 20)
    status = P.lib.pa_paged_attention_static(16, 16, P.PA_BF16, 16, 16, P.PA_BF16, None, None, 16, 512, 16, S, H,
                                             Hkv, d, 16, 100, mcl, 0.1, 64, None, None)
    assert status == P.PA_ERR_WORKSPACE_TOO_SMALL
