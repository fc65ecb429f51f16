"""Failure detection on the GPU without a fault: a bounded wait that nothing satisfies gives up after a
short limit, reports PA_DEVERR_TIMEOUT through the error word, and the context stays usable (a normal
attention call right after still matches the oracle)."""
import time

import numpy as np
import pytest
import torch

import workloads as W
from steps import TOLERANCE, gpu_step, initial_pools, oracle_step, to_device_pool

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    from pagedattention_paged_kv_attention_b200 import pagedattn as P
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    P.selftest_wait_timeout(word, 50_000_000)  # 50 ms
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(word.item()) & P.PA_DEVERR_TIMEOUT
    assert 0.04 <= elapsed < 5.0
    cfg = W.CONFIGS["tiny"]
    w = W.make_workload(cfg)
    kc, vc = initial_pools(w)
    out, ws = gpu_step(P, w, to_device_pool(kc, cfg), to_device_pool(vc, cfg))
    ref = oracle_step(w, kc, vc)
    assert np.max(np.abs(out.double().cpu().numpy() - ref)) <= TOLERANCE["f16"]
    assert P.get_device_error(ws) == 0


def test_selftest_rejects_bad_arguments():
    from pagedattention_paged_kv_attention_b200 import pagedattn as P
    assert P.lib.pa_selftest_wait_timeout(None, 1000, None) == P.PA_ERR_INVALID_ARGUMENT
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert P.lib.pa_selftest_wait_timeout(word.data_ptr(), 0, None) == P.PA_ERR_INVALID_ARGUMENT
    assert P.lib.pa_selftest_wait_timeout(word.data_ptr(), 20_000_000_000, None) == P.PA_ERR_INVALID_ARGUMENT
