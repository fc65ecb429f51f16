"""The read-bandwidth probes (include/pa_probe.h) that the benchmark uses as same-run ceilings.

They read and fold data and write their sink only when the fold hits one fixed word: on zeroed buffers
the fold is known, so the sink must stay 0. The paged probe skips block ids outside the pool and
contexts longer than the table, like the attention kernel, without faulting.
"""
import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    from pagedattention_paged_kv_attention_b200 import pagedattn
    return pagedattn


def test_stream_read_runs_and_leaves_sink(P):
    buf = torch.zeros(1 << 22, dtype=torch.uint8, device="cuda")  # 4 MB: every fold is 0
    for repeat in (1, 2, 7):
        sink = P.probe_stream_read(buf, repeat=repeat)
        torch.cuda.synchronize()
        assert int(sink.item()) == 0


def test_paged_read_skips_invalid_ids_and_lengths(P):
    cfg = W.CONFIGS["tiny"]
    w = W.make_workload(cfg, seed=cfg.seed, device="cuda")
    kc = torch.zeros_like(w.key_values)
    vc = torch.zeros_like(w.value_values)
    tables = w.block_tables.clone()
    lens = w.context_lens.clone()
    NB, bs = kc.shape[0], kc.shape[1]
    tables[0, 0] = -5                       # outside the pool: skipped
    tables[1, 0] = NB + 3                   # past the pool: skipped
    lens[2] = tables.shape[1] * bs + 1      # longer than its table: the sequence is skipped
    sink = P.probe_paged_read(kc, vc, tables, lens)
    torch.cuda.synchronize()
    assert int(sink.item()) == 0
    # the unmodified batch as well
    sink = P.probe_paged_read(kc, vc, w.block_tables, w.context_lens)
    torch.cuda.synchronize()
    assert int(sink.item()) == 0
