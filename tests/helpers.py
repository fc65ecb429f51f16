"""Small test-side helpers: dtype marshalling between torch tensors and the oracle's raw bits.

No attention arithmetic lives here.
"""
import math

import numpy as np
import torch

TORCH_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}
NAN_BITS = {"f16": 0x7E00, "bf16": 0x7FC0}


def bits16(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bits of a CPU fp16/bf16 tensor."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits16(bits: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).view(TORCH_DTYPES[dtype])


def parse_scale(text):
    table = {"ln3": math.log(3.0), "ln2": math.log(2.0), "ln3/2": math.log(3.0) / 2, "1": 1.0}
    return table[text] if isinstance(text, str) else float(text)


def golden_case_arrays(case):
    """Inputs of a hand-derived golden case as oracle-ready arrays."""
    H, Hkv, d = case["num_heads"], case["num_kv_heads"], case["head_size"]
    bs, NB = case["block_size"], case["num_blocks"]
    qd, kvd = case["q_dtype"], case["kv_dtype"]
    q = torch.tensor(case["query"], dtype=torch.float64).to(TORCH_DTYPES[qd])
    if kvd == "fp8_e4m3":
        kc = np.full((NB, bs, Hkv, d), 0x7F, np.uint8)
        vc = np.full((NB, bs, Hkv, d), 0x7F, np.uint8)
        for p in case["placed_codes"]:
            kc[p["block"], p["offset"], p["head"]] = [int(c, 16) for c in p["k"]]
            vc[p["block"], p["offset"], p["head"]] = [int(c, 16) for c in p["v"]]
    else:
        kc = np.full((NB, bs, Hkv, d), NAN_BITS[kvd], np.uint16)
        vc = np.full((NB, bs, Hkv, d), NAN_BITS[kvd], np.uint16)
        for p in case["placed"]:
            kc[p["block"], p["offset"], p["head"]] = bits16(torch.tensor(p["k"]).to(TORCH_DTYPES[kvd]))
            vc[p["block"], p["offset"], p["head"]] = bits16(torch.tensor(p["v"]).to(TORCH_DTYPES[kvd]))
    ks = np.array(case.get("k_scale", [1.0] * Hkv), np.float32)
    vs = np.array(case.get("v_scale", [1.0] * Hkv), np.float32)
    return dict(query_bits=bits16(q), q_dtype=qd, key_cache=kc, value_cache=vc, kv_dtype=kvd,
                block_tables=np.array(case["block_tables"], np.int32),
                context_lens=np.array(case["context_lens"], np.int32),
                scale=parse_scale(case["scale"]),
                k_scale=ks if kvd == "fp8_e4m3" else None, v_scale=vs if kvd == "fp8_e4m3" else None)


def random_paged_case(rng: np.random.Generator, lens, num_heads, num_kv_heads, head_size, block_size,
                      dtype="bf16", extra_blocks=3, logical=False):
    """A random paged cache built the other way round from the oracle: logical contiguous K/V first,
    then each token written into block table[t // bs] at offset t % bs by this test-side code.
    Returns (inputs for the oracle, logical q/K/V as float64 torch tensors)."""
    td = TORCH_DTYPES[dtype]
    S = len(lens)
    nblk = [(L + block_size - 1) // block_size for L in lens]
    NB = sum(nblk) + extra_blocks
    perm = rng.permutation(NB)
    max_blocks = max(1, max(nblk))
    tables = np.full((S, max_blocks), perm[-1], np.int32)   # unused entries -> a poisoned block
    kc = np.full((NB, block_size, num_kv_heads, head_size), NAN_BITS[dtype], np.uint16)
    vc = np.full_like(kc, NAN_BITS[dtype])
    q = torch.from_numpy(rng.standard_normal((S, num_heads, head_size))).to(td)
    Ks, Vs = [], []
    cursor = 0
    for s, L in enumerate(lens):
        tables[s, :nblk[s]] = perm[cursor:cursor + nblk[s]]
        cursor += nblk[s]
        K = torch.from_numpy(rng.standard_normal((L, num_kv_heads, head_size))).to(td)
        V = torch.from_numpy(rng.standard_normal((L, num_kv_heads, head_size))).to(td)
        kb, vb = bits16(K), bits16(V)
        for t in range(L):
            blk = tables[s, t // block_size]
            kc[blk, t % block_size] = kb[t]
            vc[blk, t % block_size] = vb[t]
        Ks.append(K.to(torch.float64))
        Vs.append(V.to(torch.float64))
    inputs = dict(query_bits=bits16(q), q_dtype=dtype, key_cache=kc, value_cache=vc, kv_dtype=dtype,
                  block_tables=tables, context_lens=np.array(lens, np.int32))
    return inputs, q.to(torch.float64), Ks, Vs


def logical_fp8(codes, scales, tables, s, L, bs):
    """This test-side gather and decode of an FP8 cache: [L, Hkv, d] float64 for sequence s, each code
    decoded by torch's float8_e4m3fn and multiplied by its scale -- scales [Hkv] (per kv head) or
    [num_blocks, Hkv] (per physical block and kv head)."""
    rows = []
    for t in range(L):
        blk = tables[s, t // bs]
        c = torch.from_numpy(codes[blk, t % bs].copy()).view(torch.float8_e4m3fn).to(torch.float64)
        sc = scales[blk] if scales.ndim == 2 else scales
        rows.append(c * torch.from_numpy(sc.astype(np.float64))[:, None])
    return torch.stack(rows)
