"""Seeded synthetic inputs for paged decode attention.

Shared by the tests (GPU path and oracle alike), the benchmark and the smoke check. This module holds
none of the method's arithmetic: it draws context lengths, physical block placements, block tables,
N(0,1) query/key/value values and new tokens, and lays values out block by block in the cache layout
``[num_blocks, block_size, num_kv_heads, head_size]``. It never computes attention, never quantises
and never writes a token into a slot: FP8 caches are returned as their unquantised 16-bit values plus
the per-kv-head scale, and each consumer quantises them with its own code.

Recipe (the same for every config; sizes in ``CONFIGS``):
  * context lengths: an explicit list, or uniform integers in [lo, hi] (numpy PCG64, sub-seed "lens");
    the shared-prefix config uses prefix + uniform suffix;
  * each sequence holds ceil(L / block_size) logical blocks; the shared-prefix config's first blocks are
    the same physical blocks in every table (reference count = number of sequences);
  * physical ids: a seeded permutation of the pool (sub-seed "perm"); used blocks take the first ids,
    copy-on-write destinations the next ones, the poison block the next one; the pool is either a
    fixed size or ceil(1.2 x the blocks needed);
  * values: N(0,1) float32 from a seeded torch generator, cast (round to nearest even) to the query /
    cache dtype, drawn in logical order (sequence, then logical block), so the logical data do not
    depend on the placement;
  * poison: every element not holding a valid token (unused blocks, the tail of each last block, and
    the slot of the new token before it is written) is NaN; unused block-table entries point at a
    NaN-filled poison block;
  * the decode token of sequence s sits at logical position L_s - 1; its key/value are returned as
    ``new_key``/``new_value`` with ``slot_mapping[s] = table[s][(L_s-1) // bs] * bs + (L_s-1) % bs``;
  * FP8 scale per kv head: max |x| over that head's drawn values / 448, in float32.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np
import torch

FP8_MAX = 448.0  # largest finite OCP E4M3 magnitude (used only to size the calibration scale)

_TORCH_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}
_NAN_BITS = {"f16": 0x7E00, "bf16": 0x7FC0}


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    description: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_size: int
    block_size: int
    dtype: str                      # query / output / new-token dtype: "f16" or "bf16"
    kv_dtype: str                   # "f16", "bf16", "fp8_e4m3" (per-kv-head scales) or "fp8_e4m3_block"
    seed: int
    context_lens: Optional[Sequence[int]] = None   # explicit lengths
    len_range: Optional[tuple] = None              # uniform [lo, hi]
    shared_prefix_tokens: int = 0                  # shared prefix (multiple of block_size)
    num_blocks: Optional[int] = None               # fixed pool size; else ceil(1.2 x needed)
    cow_pairs: int = 0                             # copy-on-write pairs per step
    partition_size: int = 0                        # 0 = library's choice
    scale: Optional[float] = None                  # None = 1/sqrt(head_size)

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.head_size)


CONFIGS = {
    "tiny": Config(
        name="tiny",
        description="tiny paged decode: 4 seqs, context_lens {1,17,33,100}, 8 heads (MHA), head_size 64, "
                    "block_size 16, 64 physical blocks, fp16, scale 1/8, reshape_and_cache of 4 new tokens",
        num_seqs=4, num_heads=8, num_kv_heads=8, head_size=64, block_size=16, dtype="f16",
        kv_dtype="f16", seed=1, context_lens=(1, 17, 33, 100), num_blocks=64, scale=1.0 / 8.0),
    "7b": Config(
        name="7b",
        description="7B-shape decode: 64 seqs, context_lens U[512,2048], 32 q / 32 kv heads, head_size 128, "
                    "block_size 16, bf16, blocks shuffled across a 16384-block pool",
        num_seqs=64, num_heads=32, num_kv_heads=32, head_size=128, block_size=16, dtype="bf16",
        kv_dtype="bf16", seed=2, len_range=(512, 2048), num_blocks=16384),
    "70b_gqa": Config(
        name="70b_gqa",
        description="70B-shape GQA decode: 128 seqs, context_lens U[1024,4096], 64 q / 8 kv heads, "
                    "head_size 128, block_size 8, bf16, pool 1.2x the used blocks",
        num_seqs=128, num_heads=64, num_kv_heads=8, head_size=128, block_size=8, dtype="bf16",
        kv_dtype="bf16", seed=3, len_range=(1024, 4096)),
    "long_splitk": Config(
        name="long_splitk",
        description="long-context split-K decode: 8 seqs x 32768 tokens, 32 q / 8 kv heads, head_size 128, "
                    "block_size 32, bf16, pool 1.2x the used blocks, partition 512 tokens + reduce",
        num_seqs=8, num_heads=32, num_kv_heads=8, head_size=128, block_size=32, dtype="bf16",
        kv_dtype="bf16", seed=4, context_lens=(32768,) * 8, partition_size=512),
    "shared_prefix_fp8": Config(
        name="shared_prefix_fp8",
        description="shared-prefix serving batch: 256 seqs sharing a 1024-token prefix (64 blocks) plus "
                    "private suffixes U[1,512], 32 q / 8 kv heads, head_size 128, block_size 16, FP8-E4M3 KV "
                    "with per-kv-head fp32 scale, reshape_and_cache of 256 tokens + copy_blocks of 64 pairs",
        num_seqs=256, num_heads=32, num_kv_heads=8, head_size=128, block_size=16, dtype="bf16",
        kv_dtype="fp8_e4m3", seed=5, len_range=(1, 512), shared_prefix_tokens=1024, cow_pairs=64),
    "shared_prefix_fp8_block": Config(
        name="shared_prefix_fp8_block",
        description="the shared-prefix serving batch with an FP8-E4M3 cache scaled per (block, kv head): 256 "
                    "seqs, 1024-token shared prefix + suffixes U[1,512], 32 q / 8 kv heads, head_size 128, "
                    "block_size 16, reshape_and_cache of 256 tokens + copy_blocks of 64 pairs",
        num_seqs=256, num_heads=32, num_kv_heads=8, head_size=128, block_size=16, dtype="bf16",
        kv_dtype="fp8_e4m3_block", seed=6, len_range=(1, 512), shared_prefix_tokens=1024, cow_pairs=64),
}


def sub_seeds(seed: int, n: int = 8):
    """Independent 63-bit seeds derived from one base seed (numpy SeedSequence)."""
    ss = np.random.SeedSequence(seed)
    return [int(x) & ((1 << 63) - 1) for x in ss.generate_state(n, dtype=np.uint64)]


@dataclasses.dataclass
class Workload:
    cfg: Config
    seed: int
    context_lens: torch.Tensor      # int32 [S]
    block_tables: torch.Tensor      # int32 [S, max_blocks]
    num_blocks: int
    poison_block: int
    used_blocks: torch.Tensor       # int64 physical ids holding data (logical order, shared ones once)
    query: torch.Tensor             # [S, H, d] in cfg.dtype
    key_values: torch.Tensor        # [NB, bs, Hkv, d] in cfg.dtype (or the cache dtype if 16-bit)
    value_values: torch.Tensor
    new_key: torch.Tensor           # [S, Hkv, d] in cfg.dtype
    new_value: torch.Tensor
    slot_mapping: torch.Tensor      # int64 [S]
    cow_mapping: torch.Tensor       # int64 [N, 2]
    k_scale: Optional[torch.Tensor]  # float32 [Hkv], or [num_blocks, Hkv] for per-block scales (FP8 only)
    v_scale: Optional[torch.Tensor]

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max().item()) if self.context_lens.numel() else 0

    def kv_tokens(self) -> int:
        return int(self.context_lens.to(torch.int64).sum().item())


def _lengths(cfg: Config, rng: np.random.Generator, num_seqs: int) -> np.ndarray:
    if cfg.context_lens is not None:
        lens = np.array(cfg.context_lens, dtype=np.int64)
        assert len(lens) == num_seqs
    else:
        lo, hi = cfg.len_range
        lens = rng.integers(lo, hi + 1, size=num_seqs, dtype=np.int64)
    return lens + cfg.shared_prefix_tokens


def make_workload(cfg: Config, seed: Optional[int] = None, device="cpu", num_seqs: Optional[int] = None,
                  placement_seed: Optional[int] = None, prefilled: bool = False,
                  context_lens: Optional[Sequence[int]] = None) -> Workload:
    """Build one batch of synthetic decode inputs.

    seed            base seed (default cfg.seed); values and lengths follow it.
    placement_seed  seed of the physical permutation only (default: derived from seed). Two workloads
                    that differ only in placement_seed hold the same logical data in other blocks.
    num_seqs        a smaller batch of the same config (the first num_seqs lengths; values redrawn).
    prefilled       also store the new token at position L-1 (otherwise that slot is poisoned and the
                    new token is only in new_key/new_value).
    context_lens    override the lengths (tests of edge cases).
    """
    seed = cfg.seed if seed is None else seed
    S_full = cfg.num_seqs
    S = S_full if num_seqs is None else num_seqs
    s_lens, s_perm, s_q, s_k, s_v, s_new, s_cow, _ = sub_seeds(seed)
    if placement_seed is not None:
        s_perm = sub_seeds(placement_seed)[1]
    bs, Hkv, H, d = cfg.block_size, cfg.num_kv_heads, cfg.num_heads, cfg.head_size

    if context_lens is not None:
        lens = np.array(context_lens, dtype=np.int64)
        S = len(lens)
    else:
        lens = _lengths(cfg, np.random.default_rng(s_lens), S_full)[:S]
    nblocks = (lens + bs - 1) // bs
    prefix_blocks = cfg.shared_prefix_tokens // bs
    assert cfg.shared_prefix_tokens % bs == 0
    private = np.maximum(nblocks - prefix_blocks, 0)
    needed = prefix_blocks + int(private.sum())
    extra = cfg.cow_pairs + 1  # copy-on-write destinations + one poison block
    if cfg.num_blocks is not None:
        NB = cfg.num_blocks
    else:
        NB = int(math.ceil(1.2 * (needed + cfg.cow_pairs)))
        NB = max(NB, needed + extra)
    assert needed + extra <= NB, "pool too small"

    perm = np.random.default_rng(s_perm).permutation(NB)
    used = perm[:needed]
    cow_dst = perm[needed:needed + cfg.cow_pairs]
    poison = int(perm[needed + cfg.cow_pairs])

    max_blocks = int(max(1, nblocks.max() if S else 1))
    tables = np.full((S, max_blocks), poison, dtype=np.int64)
    cursor = prefix_blocks
    for s in range(S):
        tables[s, :min(prefix_blocks, nblocks[s])] = used[:min(prefix_blocks, nblocks[s])]
        n_priv = int(private[s])
        tables[s, prefix_blocks:prefix_blocks + n_priv] = used[cursor:cursor + n_priv]
        cursor += n_priv

    tdtype = _TORCH_DTYPES[cfg.dtype]
    fp8 = cfg.kv_dtype.startswith("fp8")
    store_dtype = tdtype if fp8 else _TORCH_DTYPES[cfg.kv_dtype]
    store_key = cfg.dtype if fp8 else cfg.kv_dtype
    dev = torch.device(device)

    def gen(s):
        g = torch.Generator(device=dev)
        g.manual_seed(s)
        return g

    gq = gen(s_q)
    query = torch.randn((S, H, d), generator=gq, device=dev, dtype=torch.float32).to(tdtype)

    # Key/value blocks in logical order (shared prefix blocks once), then placed at their ids.
    used_t = torch.from_numpy(used.astype(np.int64)).to(dev)
    nan_bits = _NAN_BITS[store_key]
    kv = []
    for s_vals in (s_k, s_v):
        pool = torch.empty((NB, bs, Hkv, d), dtype=store_dtype, device=dev)
        pool.view(torch.int16).fill_(nan_bits)
        vals = torch.randn((needed, bs, Hkv, d), generator=gen(s_vals), device=dev,
                           dtype=torch.float32).to(store_dtype)
        pool[used_t] = vals
        del vals
        kv.append(pool)
    key_pool, value_pool = kv

    # The decode token is logical position L-1 of each sequence.
    tables_t = torch.from_numpy(tables).to(dev)
    lens_t = torch.from_numpy(lens).to(dev)
    seq_idx = torch.arange(S, device=dev)
    last = (lens_t - 1).clamp(min=0)
    blk_of_last = tables_t[seq_idx, last // bs]
    slot = blk_of_last * bs + last % bs
    slot = torch.where(lens_t > 0, slot, torch.full_like(slot, -1))
    safe_blk = torch.where(lens_t > 0, blk_of_last, torch.zeros_like(blk_of_last))
    off = (last % bs)
    new_key = key_pool[safe_blk, off].clone().to(tdtype)
    new_value = value_pool[safe_blk, off].clone().to(tdtype)

    # FP8 calibration scale from the drawn values (before poisoning).
    k_scale = v_scale = None
    if cfg.kv_dtype == "fp8_e4m3":
        k_amax = key_pool[used_t].float().abs().amax(dim=(0, 1, 3))
        v_amax = value_pool[used_t].float().abs().amax(dim=(0, 1, 3))
        k_scale = (k_amax / FP8_MAX).to(torch.float32)
        v_scale = (v_amax / FP8_MAX).to(torch.float32)
    elif cfg.kv_dtype == "fp8_e4m3_block":
        # One scale per (block, kv head): max |x| over the block's drawn values of that head / 448;
        # blocks without data get 1; copy-on-write destinations carry their source block's scales.
        scales = []
        for pool in (key_pool, value_pool):
            sc = torch.ones((NB, Hkv), dtype=torch.float32, device=dev)
            amax = pool[used_t].float().abs().amax(dim=(1, 3))
            sc[used_t] = torch.where(amax > 0, amax / FP8_MAX, torch.ones_like(amax))
            if cfg.cow_pairs:
                src = torch.from_numpy(used[:cfg.cow_pairs].astype(np.int64)).to(dev)
                sc[torch.from_numpy(cow_dst.astype(np.int64)).to(dev)] = sc[src]
            scales.append(sc)
        k_scale, v_scale = scales

    # Poison the tail of each sequence's last block (from L-1, or from L when prefilled).
    for s in range(S):
        L = int(lens[s])
        if L == 0:
            continue
        first_bad = L if prefilled else L - 1
        blk_last = int(tables[s, (L - 1) // bs])
        start = first_bad - ((L - 1) // bs) * bs
        if start < bs:
            key_pool[blk_last, start:].view(torch.int16).fill_(nan_bits)
            value_pool[blk_last, start:].view(torch.int16).fill_(nan_bits)

    cow = np.stack([used[:cfg.cow_pairs], cow_dst], axis=1) if cfg.cow_pairs else np.zeros((0, 2), np.int64)
    return Workload(
        cfg=cfg, seed=seed,
        context_lens=torch.from_numpy(lens.astype(np.int32)).to(dev),
        block_tables=torch.from_numpy(tables.astype(np.int32)).to(dev),
        num_blocks=NB, poison_block=poison, used_blocks=used_t,
        query=query, key_values=key_pool, value_values=value_pool,
        new_key=new_key, new_value=new_value,
        slot_mapping=slot.to(torch.int64),
        cow_mapping=torch.from_numpy(cow.astype(np.int64)).to(dev),
        k_scale=k_scale, v_scale=v_scale)


def ideal_bytes(context_lens, num_kv_heads: int, head_size: int, kv_elem_bytes: int, block_size: int,
                num_heads: int, q_elem_bytes: int) -> dict:
    """Algorithmic bytes of one paged-attention call: each valid token's K and V row once, the block
    ids covering each context, the query and the output."""
    lens = np.asarray(context_lens, dtype=np.int64)
    kv = int(lens.sum()) * num_kv_heads * head_size * kv_elem_bytes * 2
    ids = int(((lens + block_size - 1) // block_size).sum()) * 4
    q = len(lens) * num_heads * head_size * q_elem_bytes
    return {"kv": kv, "block_ids": ids, "query": q, "out": q, "total": kv + ids + 2 * q}


# ------------------------------------------------------------------------------------------------
# Prefill (a chunk of new query tokens per sequence, causal over its prefix).
#
# Recipe: context lengths as above (explicit or uniform); each sequence's chunk is its last
# n_s = min(chunk, L_s) tokens (chunk None: the whole prompt, n_s = L_s); the pool holds every context
# token except the chunk's, whose slots are NaN until the step writes them (the chunk's keys and values
# are returned as new_key/new_value with their slot_mapping, in row order); the query rows are the
# chunks back to back (q_start the prefix sums of n_s); N(0,1) values drawn in logical order; random
# block placement over a pool of ceil(1.2 x needed) blocks plus a NaN poison block for padding.
# ------------------------------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class PrefillConfig:
    name: str
    description: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_size: int
    block_size: int
    dtype: str
    seed: int
    context_lens: Optional[Sequence[int]] = None
    len_range: Optional[tuple] = None
    chunk: Optional[int] = None                    # None: the whole prompt is the chunk
    scale: Optional[float] = None
    kv_dtype: Optional[str] = None                 # None: the query dtype; or "fp8_e4m3" / "fp8_e4m3_block"

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.head_size)

    @property
    def cache_dtype(self) -> str:
        return self.kv_dtype or self.dtype


PREFILL_CONFIGS = {
    "prefill_tiny": PrefillConfig(
        name="prefill_tiny",
        description="small prefill: 3 prompts of 37, 128 and 200 tokens, 8 q / 2 kv heads, head_size 128, "
                    "block_size 16, bf16",
        num_seqs=3, num_heads=8, num_kv_heads=2, head_size=128, block_size=16, dtype="bf16", seed=11,
        context_lens=(37, 128, 200)),
    "prefill_7b": PrefillConfig(
        name="prefill_7b",
        description="7B-shape prompt prefill: 16 prompts U[1024,4096] tokens, 32 q / 32 kv heads, head_size 128, "
                    "block_size 16, bf16, causal",
        num_seqs=16, num_heads=32, num_kv_heads=32, head_size=128, block_size=16, dtype="bf16", seed=12,
        len_range=(1024, 4096)),
    "prefill_70b_gqa": PrefillConfig(
        name="prefill_70b_gqa",
        description="70B-shape GQA prompt prefill: 16 prompts U[1024,4096] tokens, 64 q / 8 kv heads, "
                    "head_size 128, block_size 16, bf16, causal",
        num_seqs=16, num_heads=64, num_kv_heads=8, head_size=128, block_size=16, dtype="bf16", seed=13,
        len_range=(1024, 4096)),
    "chunked_prefill": PrefillConfig(
        name="chunked_prefill",
        description="chunked prefill: 32 sequences with contexts U[2048,8192], the last 512 tokens of each as "
                    "the chunk, 32 q / 8 kv heads, head_size 128, block_size 16, bf16",
        num_seqs=32, num_heads=32, num_kv_heads=8, head_size=128, block_size=16, dtype="bf16", seed=14,
        len_range=(2048, 8192), chunk=512),
    "chunked_prefill_fp8": PrefillConfig(
        name="chunked_prefill_fp8",
        description="chunked prefill over an FP8-E4M3 cache with one scale per kv head: 32 sequences with "
                    "contexts U[2048,8192], the last 512 tokens of each as the chunk, 32 q / 8 kv heads, "
                    "head_size 128, block_size 16, bf16 queries",
        num_seqs=32, num_heads=32, num_kv_heads=8, head_size=128, block_size=16, dtype="bf16", seed=15,
        len_range=(2048, 8192), chunk=512, kv_dtype="fp8_e4m3"),
    "chunked_prefill_fp8_block": PrefillConfig(
        name="chunked_prefill_fp8_block",
        description="chunked prefill over an FP8-E4M3 cache with one scale per (block, kv head): 32 sequences "
                    "with contexts U[2048,8192], the last 512 tokens of each as the chunk, 32 q / 8 kv heads, "
                    "head_size 128, block_size 16, bf16 queries",
        num_seqs=32, num_heads=32, num_kv_heads=8, head_size=128, block_size=16, dtype="bf16", seed=16,
        len_range=(2048, 8192), chunk=512, kv_dtype="fp8_e4m3_block"),
}


@dataclasses.dataclass
class PrefillWorkload:
    cfg: PrefillConfig
    context_lens: torch.Tensor      # int32 [S]
    q_start: torch.Tensor           # int32 [S + 1]
    block_tables: torch.Tensor      # int32 [S, max_blocks]
    num_blocks: int
    query: torch.Tensor             # [T, H, d]
    key_values: torch.Tensor        # [NB, bs, Hkv, d]; the chunks' slots are NaN
    value_values: torch.Tensor
    new_key: torch.Tensor           # [T, Hkv, d]: the chunks' keys, row order
    new_value: torch.Tensor
    slot_mapping: torch.Tensor      # int64 [T]
    k_scale: Optional[torch.Tensor] = None   # FP8 caches: float32 [Hkv], or [num_blocks, Hkv] per block
    v_scale: Optional[torch.Tensor] = None

    @property
    def max_q_len(self) -> int:
        q = self.q_start
        return int((q[1:] - q[:-1]).max().item()) if q.numel() > 1 else 0

    def causal_pairs(self) -> int:
        """(query row, visible key) pairs per head: sum over sequences of n(L-n) + n(n+1)/2."""
        L = self.context_lens.to(torch.int64)
        n = (self.q_start[1:] - self.q_start[:-1]).to(torch.int64)
        return int((n * (L - n) + n * (n + 1) // 2).sum().item())


def make_prefill_workload(cfg: PrefillConfig, seed: Optional[int] = None, device="cpu",
                          num_seqs: Optional[int] = None,
                          context_lens: Optional[Sequence[int]] = None,
                          chunk_lens: Optional[Sequence[int]] = None) -> PrefillWorkload:
    seed = cfg.seed if seed is None else seed
    s_lens, s_perm, s_q, s_k, s_v, _, _, _ = sub_seeds(seed)
    bs, Hkv, H, d = cfg.block_size, cfg.num_kv_heads, cfg.num_heads, cfg.head_size
    if context_lens is not None:
        lens = np.array(context_lens, dtype=np.int64)
    elif cfg.context_lens is not None:
        lens = np.array(cfg.context_lens, dtype=np.int64)
    else:
        lo, hi = cfg.len_range
        lens = np.random.default_rng(s_lens).integers(lo, hi + 1, size=cfg.num_seqs, dtype=np.int64)
    if num_seqs is not None:
        lens = lens[:num_seqs]
    S = len(lens)
    if chunk_lens is not None:
        n = np.array(chunk_lens, dtype=np.int64)
    else:
        n = lens.copy() if cfg.chunk is None else np.minimum(lens, cfg.chunk)
    assert np.all(n <= lens) and np.all(n >= 0)
    nblocks = (lens + bs - 1) // bs
    needed = int(nblocks.sum())
    NB = max(int(math.ceil(1.2 * needed)), needed + 1)
    perm = np.random.default_rng(s_perm).permutation(NB)
    used, poison = perm[:needed], int(perm[needed])
    max_blocks = int(max(1, nblocks.max() if S else 1))
    tables = np.full((S, max_blocks), poison, dtype=np.int64)
    cursor = 0
    for s in range(S):
        tables[s, :nblocks[s]] = used[cursor:cursor + nblocks[s]]
        cursor += int(nblocks[s])

    tdtype = _TORCH_DTYPES[cfg.dtype]
    nan_bits = _NAN_BITS[cfg.dtype]
    dev = torch.device(device)

    def gen(sd):
        g = torch.Generator(device=dev)
        g.manual_seed(sd)
        return g

    q_start = np.concatenate([[0], np.cumsum(n)]).astype(np.int64)
    T = int(q_start[-1])
    query = torch.randn((T, H, d), generator=gen(s_q), device=dev, dtype=torch.float32).to(tdtype)
    used_t = torch.from_numpy(used.astype(np.int64)).to(dev)
    pools = []
    for s_vals in (s_k, s_v):
        pool = torch.empty((NB, bs, Hkv, d), dtype=tdtype, device=dev)
        pool.view(torch.int16).fill_(nan_bits)
        pool[used_t] = torch.randn((needed, bs, Hkv, d), generator=gen(s_vals), device=dev,
                                   dtype=torch.float32).to(tdtype)
        pools.append(pool)
    key_pool, value_pool = pools

    # FP8 calibration scales from the drawn values (the chunk's included), as for decode: max |x| / 448
    # per kv head, or per (block, kv head) with 1 for blocks without data.
    k_scale = v_scale = None
    if cfg.cache_dtype == "fp8_e4m3":
        k_scale, v_scale = [(pool[used_t].float().abs().amax(dim=(0, 1, 3)) / FP8_MAX).to(torch.float32)
                            for pool in pools]
    elif cfg.cache_dtype == "fp8_e4m3_block":
        scales = []
        for pool in pools:
            sc = torch.ones((NB, Hkv), dtype=torch.float32, device=dev)
            amax = pool[used_t].float().abs().amax(dim=(1, 3))
            sc[used_t] = torch.where(amax > 0, amax / FP8_MAX, torch.ones_like(amax))
            scales.append(sc)
        k_scale, v_scale = scales

    # The chunk rows: slots of positions L-n .. L-1, their values taken out of the pool and poisoned there.
    tables_t = torch.from_numpy(tables).to(dev)
    seq_of_row = torch.from_numpy(np.repeat(np.arange(S), n)).to(dev)
    pos = torch.from_numpy(np.concatenate([np.arange(L - k, L) for L, k in zip(lens, n)]) if T else
                           np.zeros(0, np.int64)).to(dev)
    blk = tables_t[seq_of_row, pos // bs]
    off = pos % bs
    new_key = key_pool[blk, off].clone()
    new_value = value_pool[blk, off].clone()
    key_pool[blk, off] = torch.full_like(new_key.view(torch.int16), nan_bits).view(tdtype)
    value_pool[blk, off] = torch.full_like(new_value.view(torch.int16), nan_bits).view(tdtype)
    # Tails of last blocks past each context stay NaN from the fill (they were drawn, so re-poison).
    for s in range(S):
        L = int(lens[s])
        if L % bs:
            b_last = int(tables[s, (L - 1) // bs])
            key_pool[b_last, L % bs:].view(torch.int16).fill_(nan_bits)
            value_pool[b_last, L % bs:].view(torch.int16).fill_(nan_bits)
    return PrefillWorkload(
        cfg=cfg, context_lens=torch.from_numpy(lens.astype(np.int32)).to(dev),
        q_start=torch.from_numpy(q_start.astype(np.int32)).to(dev),
        block_tables=torch.from_numpy(tables.astype(np.int32)).to(dev), num_blocks=NB,
        query=query, key_values=key_pool, value_values=value_pool, new_key=new_key, new_value=new_value,
        slot_mapping=(blk * bs + off).to(torch.int64), k_scale=k_scale, v_scale=v_scale)
