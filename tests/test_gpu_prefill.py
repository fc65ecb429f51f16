"""GPU parity of the causal paged prefill (tcgen05 path) against the oracle.

Each case runs the prefill step the way a serving engine does: reshape_and_cache writes the chunk's
keys and values into their slots, then paged prefill attention runs over the paged cache. The oracle
takes the same two steps on the same seeded inputs.

* Small and ragged cases over every supported head size, block size, dtype and group size, contexts
  within one KV tile and across several, whole prompts and chunks (including one-token and empty
  chunks): every output element is compared. Rows with short prefixes reach |out| of a few units, so
  each element is bounded by the stated tolerance plus half an ulp of the output dtype there.
* The full-size workloads in the benchmark's launch configuration: the step runs whole; every row of
  whole sequences (the shortest prompt; for the chunked workload two adjacent sequences) is compared
  with the oracle, and sampled rows of the rest are recomputed one by one (a row at position p equals
  a one-token chunk of the context truncated to p + 1).
* Contract violations (a chunk longer than its context, a block id outside the pool) set the device
  error word without faulting.
* FP8-E4M3 caches with per-kv-head and per-block scales: ragged cases compared element by element,
  and the full-size FP8 chunked workloads on whole sequences and sampled rows; the pools after the
  step's FP8 reshape_and_cache match the oracle's byte for byte.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from helpers import bits16
from steps import TOLERANCE, elementwise_bound, pool_bits, to_device_pool

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    from pagedattention_paged_kv_attention_b200 import pagedattn
    return pagedattn


def oracle_pools(w):
    """The oracle's pools after writing the chunks (uint16 bits)."""
    kc, vc = bits16(w.key_values), bits16(w.value_values)
    oracle.reshape_and_cache(bits16(w.new_key), bits16(w.new_value), w.cfg.dtype, kc, vc, w.cfg.dtype,
                             w.slot_mapping.numpy())
    return kc, vc


def gpu_prefill_step(P, w, kc_dev=None, vc_dev=None):
    cfg = w.cfg
    dev = torch.device("cuda")
    if kc_dev is None:
        kc_dev, vc_dev = w.key_values.to(dev), w.value_values.to(dev)
    P.reshape_and_cache(w.new_key.to(dev), w.new_value.to(dev), kc_dev, vc_dev, w.slot_mapping.to(dev))
    q = w.query.to(dev)
    out = torch.full_like(q, float("nan"))
    ws = torch.zeros(64, dtype=torch.int32, device=dev)
    P.paged_prefill(out, q, kc_dev, vc_dev, w.block_tables.to(dev), w.context_lens.to(dev), w.q_start.to(dev),
                    cfg.softmax_scale, w.max_q_len, ws)
    return out, ws, kc_dev, vc_dev


def check_all_rows(out, ref, cfg):
    got = out.double().cpu().numpy()
    assert np.all(np.isfinite(got)), "non-finite output"
    bound = elementwise_bound(ref, cfg.dtype, cfg.dtype)
    worst = np.max(np.abs(got - ref) - bound) if ref.size else -1
    assert worst <= 0, f"max excess over the bound {worst}"


def test_prefill_tiny_all_rows(P):
    cfg = W.PREFILL_CONFIGS["prefill_tiny"]
    w = W.make_prefill_workload(cfg)
    out, ws, kc_dev, _ = gpu_prefill_step(P, w)
    torch.cuda.synchronize()
    assert P.get_device_error(ws) == 0
    kc, vc = oracle_pools(w)
    assert torch.equal(pool_bits(kc_dev).cpu(), torch.from_numpy(kc.view(np.int16)))
    ref = oracle.paged_prefill(bits16(w.query), cfg.dtype, kc, vc, cfg.dtype, w.block_tables.numpy(),
                               w.context_lens.numpy(), w.q_start.numpy(), cfg.softmax_scale)
    check_all_rows(out, ref, cfg)
    assert np.max(np.abs(out.double().cpu().numpy() - ref)) <= TOLERANCE["bf16"] + 2 ** -7


RAGGED = [
    # (H, Hkv, d, bs, dtype, lens, chunks)
    (8, 8, 128, 16, "bf16", [1, 17, 128, 129, 300], None),            # G = 1, whole prompts
    (8, 2, 128, 16, "bf16", [200, 64, 513], [200, 1, 130]),            # G = 4, chunks
    (16, 2, 128, 8, "f16", [255, 256, 257], [100, 256, 0]),            # G = 8, an empty chunk
    (32, 2, 64, 32, "bf16", [40, 380], [40, 260]),                     # G = 16, d = 64
    (4, 2, 64, 64, "f16", [5, 190, 400], None),                        # G = 2, block 64
    (8, 4, 128, 128, "bf16", [129, 1000], [129, 333]),                 # block 128
    (12, 12, 64, 16, "f16", [77, 3], [12, 3]),                         # G = 1, d = 64
]


@pytest.mark.parametrize("case", RAGGED, ids=lambda c: f"H{c[0]}_Hkv{c[1]}_d{c[2]}_bs{c[3]}_{c[4]}")
def test_prefill_ragged(P, case):
    H, Hkv, d, bs, dtype, lens, chunks = case
    cfg = W.PrefillConfig(name="ragged", description="", num_seqs=len(lens), num_heads=H, num_kv_heads=Hkv,
                          head_size=d, block_size=bs, dtype=dtype, seed=zlib.crc32(repr(case).encode()),
                          context_lens=tuple(lens))
    w = W.make_prefill_workload(cfg, chunk_lens=chunks)
    out, ws, _, _ = gpu_prefill_step(P, w)
    torch.cuda.synchronize()
    assert P.get_device_error(ws) == 0
    kc, vc = oracle_pools(w)
    ref = oracle.paged_prefill(bits16(w.query), dtype, kc, vc, dtype, w.block_tables.numpy(),
                               w.context_lens.numpy(), w.q_start.numpy(), cfg.softmax_scale)
    check_all_rows(out, ref, cfg)


def sampled_rows_reference(w, kc, vc, rows):
    """Oracle output of the given query rows, each as a one-token chunk over its truncated context."""
    q_start = w.q_start.numpy()
    lens = w.context_lens.numpy()
    seq = np.searchsorted(q_start, rows, side="right") - 1
    n = q_start[seq + 1] - q_start[seq]
    pos = lens[seq] - n + (rows - q_start[seq])
    qbits = bits16(w.query)[rows]
    return oracle.paged_prefill(qbits, w.cfg.dtype, kc, vc, w.cfg.dtype, w.block_tables.numpy()[seq],
                                (pos + 1).astype(np.int32), np.arange(len(rows) + 1, dtype=np.int32),
                                w.cfg.softmax_scale)


@pytest.mark.parametrize("name", ["prefill_7b", "prefill_70b_gqa", "chunked_prefill"])
def test_prefill_full_size_sampled_rows(P, name):
    cfg = W.PREFILL_CONFIGS[name]
    w = W.make_prefill_workload(cfg)
    out, ws, _, _ = gpu_prefill_step(P, w)
    torch.cuda.synchronize()
    assert P.get_device_error(ws) == 0
    got = out.double().cpu().numpy()
    assert np.all(np.isfinite(got))
    kc, vc = oracle_pools(w)
    T = w.query.shape[0]
    rng = np.random.default_rng(zlib.crc32(name.encode()))
    q_start = w.q_start.numpy()
    # Every sequence's first and last rows, plus random rows.
    rows = np.unique(np.concatenate([q_start[:-1], q_start[1:] - 1, rng.integers(0, T, 48)]))
    ref = sampled_rows_reference(w, kc, vc, rows)
    err = np.max(np.abs(got[rows] - ref))
    assert err <= TOLERANCE[cfg.dtype], f"{name}: max-abs error {err} on {len(rows)} sampled rows"


def whole_sequences(name, lens, q_start):
    """Sequences whose every row is checked at full size: for the chunked workload the two adjacent
    sequences with the smallest total context (so a sequence boundary in the query rows lies between
    them), for the prompt workloads the shortest prompt. The oracle is fp64 and slow; these keep the
    test to tens of seconds while covering every query tile and every diagonal tile of each sequence."""
    if name == "chunked_prefill":
        pair = int(np.argmin(lens[:-1] + lens[1:]))
        return [pair, pair + 1]
    return [int(np.argmin(lens))]


@pytest.mark.parametrize("name", ["prefill_7b", "prefill_70b_gqa", "chunked_prefill"])
def test_prefill_full_size_every_row_of_whole_sequences(P, name):
    cfg = W.PREFILL_CONFIGS[name]
    w = W.make_prefill_workload(cfg)
    out, ws, _, _ = gpu_prefill_step(P, w)
    torch.cuda.synchronize()
    assert P.get_device_error(ws) == 0
    got = out.double().cpu().numpy()
    kc, vc = oracle_pools(w)
    lens, q_start = w.context_lens.numpy(), w.q_start.numpy()
    seqs = whole_sequences(name, lens, q_start)
    rows = np.concatenate([np.arange(q_start[s], q_start[s + 1]) for s in seqs])
    sub_start = np.concatenate([[0], np.cumsum([q_start[s + 1] - q_start[s] for s in seqs])]).astype(np.int32)
    ref = oracle.paged_prefill(bits16(w.query)[rows], cfg.dtype, kc, vc, cfg.dtype, w.block_tables.numpy()[seqs],
                               lens[seqs], sub_start, cfg.softmax_scale)
    err = np.max(np.abs(got[rows] - ref))
    assert err <= TOLERANCE[cfg.dtype], f"{name}: max-abs error {err} over every row of sequences {seqs}"


def test_contract_violations_are_flagged(P):
    cfg = W.PREFILL_CONFIGS["prefill_tiny"]
    w = W.make_prefill_workload(cfg)
    dev = torch.device("cuda")
    kc, vc = w.key_values.to(dev), w.value_values.to(dev)
    P.reshape_and_cache(w.new_key.to(dev), w.new_value.to(dev), kc, vc, w.slot_mapping.to(dev))
    q = w.query.to(dev)
    out = torch.zeros_like(q)
    # Chunk longer than its context: sequence 1 claims 128 rows over a context of 100.
    lens = w.context_lens.clone()
    lens[1] = 100
    ws = torch.zeros(64, dtype=torch.int32, device=dev)
    P.paged_prefill(out, q, kc, vc, w.block_tables.to(dev), lens.to(dev), w.q_start.to(dev), cfg.softmax_scale,
                    w.max_q_len, ws)
    torch.cuda.synchronize()
    assert P.get_device_error(ws) & P.PA_DEVERR_CONTEXT_LEN
    rows = slice(int(w.q_start[1]), int(w.q_start[2]))
    assert torch.isnan(out[rows].float()).all() and torch.isfinite(out[:int(w.q_start[1])].float()).all()
    # A block id outside the pool.
    tables = w.block_tables.clone()
    tables[2, 3] = w.num_blocks + 5
    ws.zero_()
    P.paged_prefill(out, q, kc, vc, tables.to(dev), w.context_lens.to(dev), w.q_start.to(dev), cfg.softmax_scale,
                    w.max_q_len, ws)
    torch.cuda.synchronize()
    assert P.get_device_error(ws) & P.PA_DEVERR_BLOCK_ID


# ---------------------------------------------------------------------------------------------------
# FP8-E4M3 caches (one scale per kv head, or per (block, kv head)): the pool is quantised by the oracle's
# encoder, the step's reshape_and_cache writes the chunk in FP8 (bit-exact against the oracle's), and
# the prefill reads the codes.
# ---------------------------------------------------------------------------------------------------
def fp8_pools(w):
    """The oracle's E4M3 pools before the step and after it writes the chunk, and the scales."""
    cfg = w.cfg
    kd = cfg.cache_dtype
    ks, vs = w.k_scale.numpy(), w.v_scale.numpy()
    quant = oracle.quantize_e4m3 if kd == "fp8_e4m3" else oracle.quantize_e4m3_blocks
    kc0, vc0 = quant(bits16(w.key_values), cfg.dtype, ks), quant(bits16(w.value_values), cfg.dtype, vs)
    kc, vc = kc0.copy(), vc0.copy()
    oracle.reshape_and_cache(bits16(w.new_key), bits16(w.new_value), cfg.dtype, kc, vc, kd, w.slot_mapping.numpy(),
                             ks, vs)
    return kc0, vc0, kc, vc, ks, vs


def fp8_prefill_step(P, w):
    kc0, vc0, kc, vc, ks, vs = fp8_pools(w)
    dev = torch.device("cuda")
    kd, vd = torch.from_numpy(kc0).to(dev), torch.from_numpy(vc0).to(dev)
    ks_d, vs_d = torch.from_numpy(ks).to(dev), torch.from_numpy(vs).to(dev)
    P.reshape_and_cache(w.new_key.to(dev), w.new_value.to(dev), kd, vd, w.slot_mapping.to(dev), ks_d, vs_d)
    q = w.query.to(dev)
    out = torch.full_like(q, float("nan"))
    ws = torch.zeros(64, dtype=torch.int32, device=dev)
    P.paged_prefill(out, q, kd, vd, w.block_tables.to(dev), w.context_lens.to(dev), w.q_start.to(dev),
                    w.cfg.softmax_scale, w.max_q_len, ws, k_scale=ks_d, v_scale=vs_d)
    torch.cuda.synchronize()
    assert P.get_device_error(ws) == 0
    assert np.array_equal(kd.cpu().numpy(), kc) and np.array_equal(vd.cpu().numpy(), vc), "FP8 pools differ"
    return out, kc, vc, ks, vs


FP8_CASES = [
    # (H, Hkv, bs, dtype, kv_dtype, lens, chunks)
    (8, 8, 16, "bf16", "fp8_e4m3", [1, 17, 128, 129, 300], None),
    (8, 2, 16, "bf16", "fp8_e4m3_block", [200, 64, 513], [200, 1, 130]),
    (16, 2, 8, "f16", "fp8_e4m3", [255, 256, 257], [100, 256, 0]),
    (16, 2, 32, "f16", "fp8_e4m3_block", [40, 380], [40, 260]),
    (8, 4, 128, "bf16", "fp8_e4m3_block", [129, 1000], [129, 333]),
]


@pytest.mark.parametrize("case", FP8_CASES, ids=lambda c: f"H{c[0]}_Hkv{c[1]}_bs{c[2]}_{c[3]}_{c[4]}")
def test_prefill_fp8_ragged(P, case):
    H, Hkv, bs, dtype, kvd, lens, chunks = case
    cfg = W.PrefillConfig(name="fp8", description="", num_seqs=len(lens), num_heads=H, num_kv_heads=Hkv, head_size=128,
                          block_size=bs, dtype=dtype, seed=zlib.crc32(repr(case).encode()), context_lens=tuple(lens),
                          kv_dtype=kvd)
    w = W.make_prefill_workload(cfg, chunk_lens=chunks)
    out, kc, vc, ks, vs = fp8_prefill_step(P, w)
    ref = oracle.paged_prefill(bits16(w.query), dtype, kc, vc, kvd, w.block_tables.numpy(), w.context_lens.numpy(),
                               w.q_start.numpy(), cfg.softmax_scale, ks, vs)
    got = out.double().cpu().numpy()
    assert np.all(np.isfinite(got)), "non-finite output"
    worst = np.max(np.abs(got - ref) - elementwise_bound(ref, kvd, dtype)) if ref.size else -1
    assert worst <= 0, f"max excess over the bound {worst}"


@pytest.mark.parametrize("name", ["chunked_prefill_fp8", "chunked_prefill_fp8_block"])
def test_prefill_fp8_full_size(P, name):
    """Full-size FP8 chunked prefill: every row of two adjacent whole sequences and sampled rows of the
    rest against the oracle, within the FP8 tolerance."""
    cfg = W.PREFILL_CONFIGS[name]
    w = W.make_prefill_workload(cfg)
    out, kc, vc, ks, vs = fp8_prefill_step(P, w)
    got = out.double().cpu().numpy()
    assert np.all(np.isfinite(got))
    lens, q_start = w.context_lens.numpy(), w.q_start.numpy()
    seqs = whole_sequences("chunked_prefill", lens, q_start)
    rows = np.concatenate([np.arange(q_start[s], q_start[s + 1]) for s in seqs])
    sub_start = np.concatenate([[0], np.cumsum([q_start[s + 1] - q_start[s] for s in seqs])]).astype(np.int32)
    ref = oracle.paged_prefill(bits16(w.query)[rows], cfg.dtype, kc, vc, cfg.cache_dtype, w.block_tables.numpy()[seqs],
                               lens[seqs], sub_start, cfg.softmax_scale, ks, vs)
    err = np.max(np.abs(got[rows] - ref))
    assert err <= TOLERANCE[cfg.cache_dtype], f"{name}: max-abs error {err} over whole sequences {seqs}"
    rng = np.random.default_rng(zlib.crc32(name.encode()))
    T = w.query.shape[0]
    sample = np.unique(np.concatenate([q_start[:-1], q_start[1:] - 1, rng.integers(0, T, 48)]))
    seq = np.searchsorted(q_start, sample, side="right") - 1
    n = q_start[seq + 1] - q_start[seq]
    pos = lens[seq] - n + (sample - q_start[seq])
    ref_s = oracle.paged_prefill(bits16(w.query)[sample], cfg.dtype, kc, vc, cfg.cache_dtype,
                                 w.block_tables.numpy()[seq], (pos + 1).astype(np.int32),
                                 np.arange(len(sample) + 1, dtype=np.int32), cfg.softmax_scale, ks, vs)
    err_s = np.max(np.abs(got[sample] - ref_s))
    assert err_s <= TOLERANCE[cfg.cache_dtype], f"{name}: max-abs error {err_s} on sampled rows"
