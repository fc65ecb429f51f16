"""The C ABI without a GPU: the library builds, loads, exports every symbol the header declares, plans
launches as documented, and rejects bad arguments with a status code before any CUDA call (every
call below would fault or fail if it reached the device, and none needs one)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in sorted(os.listdir(os.path.join(ROOT, "include")))
           if h.endswith(".h")]


@pytest.fixture(scope="module")
def P():
    from pagedattention_paged_kv_attention_b200 import build
    build.build()
    from pagedattention_paged_kv_attention_b200 import pagedattn
    return pagedattn


def declared_functions():
    text = "".join(open(h).read() for h in HEADERS)
    return sorted(set(re.findall(r"PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports(P):
    assert declared_functions() == sorted(P.EXPORTS)


def test_every_declared_symbol_is_exported(P):
    lib = ctypes.CDLL(P.LIBRARY_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(P):
    for code in range(7):
        assert P.lib.pa_status_string(code) and b"unknown" not in P.lib.pa_status_string(code)
    assert P.lib.pa_status_string(99) == b"unknown pa_status"


def test_partition_planning(P):
    assert P.partition_size(8, 32, 8, 32768, 512) == 512
    assert P.partition_size(8, 32, 8, 32768, 100) == -1           # not a multiple of 64
    assert P.partition_size(8, 32, 8, 32768, -64) == -1
    assert P.partition_size(4, 8, 8, 100) >= 100                  # tiny: one partition
    # About five items per CTA (148 SMs) at max_context_len, at most 32 partitions, a multiple of 64.
    assert P.partition_size(64, 32, 32, 1996) == 704                # 7B shape: 256 units
    assert P.partition_size(128, 64, 8, 4092) == 768                # 70B shape: 128 units
    assert P.partition_size(256, 32, 8, 1535) == 576
    assert P.partition_size(8, 32, 8, 32768) == 1024                # long contexts: capped at 32 partitions
    assert P.partition_size(4096, 32, 32, 2048) == 2048             # many sequences: no split
    for args in [(1, 8, 8, 1), (65535, 64, 8, 2 ** 31 - 1), (3, 24, 1, 500000)]:
        ps = P.partition_size(*args)
        assert ps % 64 == 0 and ps >= 256


def test_workspace_size(P):
    S, H, Hkv, d = 8, 32, 8, 128
    ws = P.workspace_size(S, H, Hkv, d, 32768, 512)
    parts = 32768 // 512
    assert ws >= 256 + S * H * parts * (d + 2) * 4
    assert P.workspace_size(4, 8, 8, 64, 100, 0) == 256           # one partition: header only
    assert P.workspace_size(4, 8, 3, 64, 100, 0) == 0             # H % Hkv != 0


def call_attention(P, **over):
    args = dict(out=16, query=16, q_dtype=P.PA_BF16, key_cache=16, value_cache=16, kv_dtype=P.PA_BF16, k_scale=None,
                v_scale=None, block_tables=16, max_blocks_per_seq=4, context_lens=16, num_seqs=2, num_heads=8,
                num_kv_heads=2, head_size=128, block_size=16, num_blocks=10, max_context_len=64, scale=0.1,
                partition_size=0, workspace=16, workspace_bytes=1 << 20, stream=None)
    args.update(over)
    return P.lib.pa_paged_attention(*args.values())


@pytest.mark.parametrize("over,status", [
    (dict(out=None), 1), (dict(query=None), 1), (dict(workspace=None), 1), (dict(block_tables=None), 1),
    (dict(out=8), 1), (dict(key_cache=24), 1), (dict(num_heads=6, num_kv_heads=4), 1),
    (dict(num_kv_heads=0), 1), (dict(num_seqs=-1), 1), (dict(max_context_len=-1), 1),
    (dict(scale=float("nan")), 1), (dict(partition_size=100), 1), (dict(q_dtype=2), 1), (dict(q_dtype=7), 1),
    (dict(kv_dtype=2), 1),                                                   # FP8 without scales
    (dict(head_size=96), 2), (dict(block_size=4), 2), (dict(block_size=128), 2),
    (dict(kv_dtype=0), 2),                                                   # f16 cache with bf16 query
    (dict(kv_dtype=2, k_scale=16, v_scale=16, head_size=64), 2),
    (dict(kv_dtype=3), 1),                                                   # per-block FP8 without scales
    (dict(kv_dtype=3, k_scale=16, v_scale=16, head_size=64), 2),            # per-block FP8: head size 128 only
    (dict(kv_dtype=4, k_scale=16, v_scale=16), 1),                          # no such cache format
    (dict(workspace_bytes=255), 3), (dict(max_context_len=4096, partition_size=64, workspace_bytes=1024), 3),
    (dict(num_seqs=0), 0),                                                   # empty batch: nothing to do
])
def test_attention_rejects_bad_arguments_without_cuda(P, over, status):
    assert call_attention(P, **over) == status


def call_static(P, **over):
    args = dict(out=16, query=16, q_dtype=P.PA_BF16, key_cache=16, value_cache=16, kv_dtype=P.PA_BF16, k_scale=None,
                v_scale=None, block_tables=16, max_blocks_per_seq=4, context_lens=16, num_seqs=2, num_heads=8,
                num_kv_heads=2, head_size=128, block_size=16, num_blocks=10, max_context_len=64, scale=0.1,
                partition_size=0, device_error_out=None, stream=None)
    args.update(over)
    return P.lib.pa_paged_attention_static(*args.values())


@pytest.mark.parametrize("over,status", [
    (dict(out=None), 1), (dict(out=8), 1), (dict(num_heads=6, num_kv_heads=4), 1), (dict(q_dtype=7), 1),
    (dict(kv_dtype=2), 1), (dict(head_size=96), 2), (dict(block_size=4), 2), (dict(kv_dtype=0), 2),
    (dict(device_error_out=18), 1), (dict(num_seqs=0), 0),
])
def test_static_entry_checks_arguments_like_the_workspace_entry(P, over, status):
    assert call_static(P, **over) == status


@pytest.mark.parametrize("bad", [dict(q_dtype=7), dict(kv_dtype=2), dict(head_size=96), dict(out=None)])
def test_static_entry_reports_a_bad_argument_before_an_oversize_request(P, bad):
    """A request too large for the fixed array that is also invalid for another reason reports the
    other reason: the argument checks come before the size comparison."""
    big = dict(num_seqs=2048, num_heads=64, num_kv_heads=8, max_blocks_per_seq=2048, max_context_len=32768,
               partition_size=64)
    assert call_static(P, **big) == P.PA_ERR_WORKSPACE_TOO_SMALL
    assert call_static(P, **big, **bad) == call_attention(P, **{k: v for k, v in big.items()}, **bad)
    assert call_static(P, **big, **bad) in (P.PA_ERR_INVALID_ARGUMENT, P.PA_ERR_UNSUPPORTED)


def test_reshape_and_copy_reject_bad_arguments(P):
    L = P.lib
    ok = dict(key=16, value=16, in_dtype=P.PA_BF16, key_cache=16, value_cache=16, kv_dtype=P.PA_BF16,
              k_scale=None, v_scale=None, slot_mapping=16, num_tokens=3, num_kv_heads=2, head_size=64,
              block_size=16, num_blocks=4, stream=None)

    def rc(**over):
        a = dict(ok)
        a.update(over)
        return L.pa_reshape_and_cache(*a.values())

    assert rc(key=None) == 1 and rc(slot_mapping=4) == 1 and rc(num_tokens=-1) == 1
    assert rc(kv_dtype=P.PA_FP8_E4M3) == 1                 # no scales
    assert rc(kv_dtype=P.PA_F16) == 2 and rc(head_size=60) == 2
    assert rc(num_tokens=0) == 0
    assert L.pa_copy_blocks(16, 16, P.PA_BF16, None, 3, 2, 64, 16, 4, None) == 1
    assert L.pa_copy_blocks(16, 16, P.PA_BF16, 16, -1, 2, 64, 16, 4, None) == 1
    assert L.pa_copy_blocks(16, 16, P.PA_BF16, 16, 0, 2, 64, 16, 4, None) == 0


def test_copy_blocks_check_on_host_mappings(P):
    import torch
    assert P.copy_blocks_check(torch.tensor([[0, 5], [1, 6]]), 8)
    assert not P.copy_blocks_check(torch.tensor([[0, 5], [1, 5]]), 8)      # duplicate destination
    assert not P.copy_blocks_check(torch.tensor([[0, 5], [5, 6]]), 8)      # destination is a source
    assert not P.copy_blocks_check(torch.tensor([[0, 8]]), 8)              # outside the pool
    assert P.copy_blocks_check(torch.zeros((0, 2), dtype=torch.int64), 8)


def test_layer_ops_reject_bad_arguments(P):
    L = P.lib
    ok = dict(keys=16, values=16, in_dtype=P.PA_BF16, key_caches=16, value_caches=16, kv_dtype=P.PA_BF16,
              k_scales=None, v_scales=None, slot_mapping=16, num_tokens=3, num_layers=4, num_kv_heads=2,
              head_size=64, block_size=16, num_blocks=4, stream=None)

    def rc(**over):
        a = dict(ok)
        a.update(over)
        return L.pa_reshape_and_cache_layers(*a.values())

    assert rc(keys=None) == 1 and rc(key_caches=12) == 1 and rc(num_layers=-1) == 1
    assert rc(kv_dtype=P.PA_FP8_E4M3) == 1                 # no scale arrays
    assert rc(kv_dtype=P.PA_F16) == 2 and rc(head_size=60) == 2 and rc(num_layers=70000) == 2
    assert rc(num_tokens=0) == 0 and rc(num_layers=0) == 0
    cb = L.pa_copy_blocks_layers
    assert cb(None, 16, 4, P.PA_BF16, 16, 3, 2, 64, 16, 4, None) == 1
    assert cb(16, 16, 4, P.PA_BF16, None, 3, 2, 64, 16, 4, None) == 1
    assert cb(16, 16, 4, P.PA_BF16, 16, 3, 1, 4, 1, 4, None) == 2          # an 8-byte block: not 16-byte vectors
    assert cb(16, 16, 4, P.PA_BF16, 16, 0, 2, 64, 16, 4, None) == 0        # no pairs


def test_binding_rejects_tensors_the_library_would_misread(P):
    """The binding checks what a pointer cannot carry (layout, element type, rank, device) and raises
    before any library call."""
    import torch
    bt = torch.zeros((4, 8), dtype=torch.int32)
    assert P._arg(bt, "block_tables", P._I32, 2, cuda=False) is not None
    assert P._arg(None, "k_scale") is None
    with pytest.raises(ValueError, match="contiguous"):
        P._arg(bt.t(), "block_tables", P._I32, 2, cuda=False)
    with pytest.raises(ValueError, match="dtype"):
        P._arg(bt.to(torch.int64), "block_tables", P._I32, 2, cuda=False)
    with pytest.raises(ValueError, match="dimensions"):
        P._arg(bt.view(-1), "block_tables", P._I32, 2, cuda=False)
    with pytest.raises(ValueError, match="CUDA tensor"):
        P._arg(bt, "block_tables", P._I32, 2)
    with pytest.raises(TypeError):
        P._arg(bt.numpy(), "block_tables", P._I32, 2, cuda=False)
    q = torch.zeros((2, 8, 64), dtype=torch.bfloat16)
    kc = torch.zeros((4, 16, 2, 64), dtype=torch.bfloat16)
    cl = torch.zeros(2, dtype=torch.int32)
    ws = torch.zeros(1024, dtype=torch.uint8)
    with pytest.raises(ValueError, match="out/query"):
        P.paged_attention(torch.zeros((2, 8, 32), dtype=torch.bfloat16), q, kc, kc, bt[:2], cl, 0.1, 64, ws)
    with pytest.raises(ValueError, match="key_cache/value_cache"):
        P.paged_attention(q.clone(), q, kc, kc.half(), bt[:2], cl, 0.1, 64, ws)
    with pytest.raises(ValueError, match="CUDA tensor"):       # host tensors never reach a kernel
        P.paged_attention(q.clone(), q, kc, kc, bt[:2], cl, 0.1, 64, ws)
    x = torch.zeros((3, 2, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="key/value"):
        P.reshape_and_cache(x, x[:2], kc, kc, torch.zeros(3, dtype=torch.int64))
    with pytest.raises(ValueError, match="CUDA tensor"):
        P.reshape_and_cache(x, x, kc, kc, torch.zeros(3, dtype=torch.int64))
    with pytest.raises(ValueError, match="contiguous"):   # swap pools may be host memory, but dense
        P.swap_blocks(kc.transpose(1, 2), kc, kc, kc, torch.zeros((1, 2), dtype=torch.int64))
    with pytest.raises(ValueError, match="dtype"):
        P.swap_blocks(kc, kc, kc, kc, torch.zeros((1, 2), dtype=torch.int32))


def test_sizes_near_int_max_do_not_wrap(P):
    """Partition counts are computed without int overflow: the workspace for a maximum context length
    of 2^31 - 1 is the layout's size for ceil((2^31 - 1) / ps) partitions."""
    r256 = lambda x: -(-x // 256) * 256
    for L, ps in ((2**31 - 1, 64), (2**31 - 64, 64), (2**31 - 1, 4096), (1025, 64)):
        rows = 8 * -(-L // ps)
        assert P.workspace_size(1, 8, 8, 128, L, ps) == 256 + 2 * r256(rows * 4) + r256(rows * 128 * 4), (L, ps)


def test_cache_writes_reject_rows_beyond_int_indexing(P):
    """Every call here is refused during validation, before any CUDA call (the pointers are dummies)."""
    L = P.lib
    args = lambda hkv, d: (16, 16, P.PA_BF16, 16, 16, P.PA_BF16, None, None, 16, 3, hkv, d, 16, 4, None)
    assert L.pa_reshape_and_cache(*args((1 << 16) + 1, 256)) == P.PA_ERR_UNSUPPORTED  # 2^24 + 256 elements
    assert L.pa_reshape_and_cache(*args(1 << 24, 1 << 10)) == P.PA_ERR_UNSUPPORTED  # product overflows int
    assert L.pa_reshape_and_cache_layers(16, 16, P.PA_BF16, 16, 16, P.PA_BF16, None, None, 16, 3, 2, 1 << 24,
                                         1 << 10, 16, 4, None) == P.PA_ERR_UNSUPPORTED


def test_probes_reject_bad_arguments(P):
    L = P.lib
    assert L.pa_probe_stream_read(None, 1024, 1, 16, None) == P.PA_ERR_INVALID_ARGUMENT
    assert L.pa_probe_stream_read(16, 1000, 1, 16, None) == P.PA_ERR_INVALID_ARGUMENT      # not a multiple of 16
    assert L.pa_probe_stream_read(24, 1024, 1, 16, None) == P.PA_ERR_INVALID_ARGUMENT      # misaligned
    assert L.pa_probe_stream_read(16, 1024, 0, 16, None) == P.PA_ERR_INVALID_ARGUMENT      # repeat < 1
    assert L.pa_probe_stream_read(16, 1024, 1, None, None) == P.PA_ERR_INVALID_ARGUMENT    # no sink
    ok = dict(kc=16, vc=16, dt=P.PA_BF16, bt=16, mb=4, cl=16, S=2, Hkv=8, d=128, bs=16, NB=10, sink=16)

    def paged(**over):
        a = dict(ok, **over)
        return L.pa_probe_paged_read(a["kc"], a["vc"], a["dt"], a["bt"], a["mb"], a["cl"], a["S"], a["Hkv"], a["d"],
                                     a["bs"], a["NB"], a["sink"], None)
    assert paged(S=0) == P.PA_OK
    assert paged(kc=None) == P.PA_ERR_INVALID_ARGUMENT
    assert paged(bt=18) == P.PA_ERR_INVALID_ARGUMENT
    assert paged(dt=9) == P.PA_ERR_INVALID_ARGUMENT
    assert paged(Hkv=1, d=4) == P.PA_ERR_UNSUPPORTED            # token row of 8 bytes: not 16-byte vectors


def call_prefill(P, **over):
    args = dict(out=16, query=16, q_dtype=P.PA_BF16, key_cache=16, value_cache=16, kv_dtype=P.PA_BF16, k_scale=None,
                v_scale=None, block_tables=16, max_blocks_per_seq=4, context_lens=16, q_start=16, num_seqs=2,
                num_q_tokens=64, num_heads=8, num_kv_heads=2, head_size=128, block_size=16, num_blocks=10, max_q_len=32,
                scale=0.1, workspace=16, workspace_bytes=256, stream=None)
    args.update(over)
    return P.lib.pa_paged_prefill(*args.values())


@pytest.mark.parametrize("over,status", [
    (dict(out=None), 1), (dict(q_start=None), 1), (dict(workspace=None), 1), (dict(key_cache=24), 1),
    (dict(scale=0.0), 1), (dict(scale=float("inf")), 1), (dict(num_heads=6, num_kv_heads=4), 1),
    (dict(kv_dtype=2), 1),                                                   # FP8 without scales
    (dict(kv_dtype=3, k_scale=16), 1),                                       # per-block FP8, one scale missing
    (dict(kv_dtype=2, k_scale=16, v_scale=16, head_size=64), 2),             # FP8: head size 128 only
    (dict(kv_dtype=0), 2),                                                   # f16 cache with a bf16 query
    (dict(head_size=96), 2), (dict(block_size=4), 2), (dict(num_heads=24, num_kv_heads=1), 2),
    (dict(workspace_bytes=128), 3),
    (dict(num_seqs=0), 0), (dict(max_q_len=0), 0),                           # nothing to compute
])
def test_prefill_rejects_bad_arguments_without_cuda(P, over, status):
    assert call_prefill(P, **over) == status
