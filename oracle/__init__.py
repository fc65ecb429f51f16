"""CPU oracle for paged decode attention (TEST INFRASTRUCTURE ONLY).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import this
package. It wraps the plain C reference in ``pa_oracle.c`` (fp64, definition-level) with numpy
marshalling. Arrays of 16-bit floats are passed as their raw bits (``uint16``), FP8-E4M3 as ``uint8``
codes.

What it computes and which page passage each function follows is stated in ``pa_oracle.c``:
  * ``paged_attention``   -- softmax(q K^T * scale) V over the whole context, K/V reached through the
                             block table (tutorial page "企业官网建设流程全解析", sec. 2.1 and 2.2);
  * ``reshape_and_cache`` -- new tokens written into their physical slots (page
                             "vLLM的诞生背景...", section "PagedAttention的破局思路");
  * ``copy_blocks``       -- copy-on-write of whole blocks (same page, "PagedAttention的局限性");
  * E4M3 / f16 / bf16 scalar codecs from their format definitions.
"""
import ctypes
import os

import numpy as np

from . import build as _build

F16, BF16, E4M3, E4M3_BLOCK = 0, 1, 2, 3   # E4M3_BLOCK: E4M3 codes, one scale per (block, kv head)
_DTYPE_CODES = {"f16": F16, "fp16": F16, "float16": F16, "bf16": BF16, "bfloat16": BF16,
                "fp8_e4m3": E4M3, "e4m3": E4M3, "fp8_e4m3_block": E4M3_BLOCK}

_default = None


def dtype_code(name):
    if isinstance(name, int):
        return name
    return _DTYPE_CODES[name]


def _bind(path):
    L = ctypes.CDLL(path)
    p = ctypes.c_void_p
    i = ctypes.c_int
    i64 = ctypes.c_int64
    sz = ctypes.c_size_t
    L.or_f16_to_double.restype = ctypes.c_double
    L.or_f16_to_double.argtypes = [ctypes.c_uint16]
    L.or_bf16_to_double.restype = ctypes.c_double
    L.or_bf16_to_double.argtypes = [ctypes.c_uint16]
    L.or_e4m3_to_double.restype = ctypes.c_double
    L.or_e4m3_to_double.argtypes = [ctypes.c_uint8]
    L.or_e4m3_from_float.restype = ctypes.c_uint8
    L.or_e4m3_from_float.argtypes = [ctypes.c_float]
    for name in ("or_e4m3_to_double_n", "or_e4m3_from_float_n", "or_f16_to_double_n",
                 "or_bf16_to_double_n"):
        getattr(L, name).restype = None
        getattr(L, name).argtypes = [p, p, sz]
    L.or_paged_attention.restype = i
    L.or_paged_attention.argtypes = [p, p, i, p, p, i, p, p, p, i, p, i, i, i, i, i, i,
                                     ctypes.c_double, i]
    L.or_paged_prefill.restype = i
    L.or_paged_prefill.argtypes = [p, p, i, p, p, i, p, p, p, i, p, p, i, i, i, i, i, i, ctypes.c_double, i]
    L.or_reshape_and_cache.restype = i
    L.or_reshape_and_cache.argtypes = [p, p, i, p, p, i, p, p, p, i64, i, i, i, i64]
    L.or_copy_blocks.restype = i
    L.or_copy_blocks.argtypes = [p, p, i, p, i64, i, i, i, i64]
    L.or_swap_blocks.restype = i
    L.or_swap_blocks.argtypes = [p, p, p, p, i, p, i64, i, i, i, i64, i64]
    return L


_lib_override = None


def lib():
    """The loaded C library (built on first use). ``use_library`` swaps in another build."""
    global _default
    if _lib_override is not None:
        return _lib_override
    if _default is None:
        _default = _bind(_build.build())
    return _default


class use_library:
    """Context manager: route every call of this module to the library at ``path`` (used by the
    tests that plant a mistake in a copy of the oracle and check that the pins catch it)."""

    def __init__(self, path):
        self.lib = _bind(path)

    def __enter__(self):
        global _lib_override
        self.prev = _lib_override
        _lib_override = self.lib
        return self.lib

    def __exit__(self, *exc):
        global _lib_override
        _lib_override = self.prev
        return False


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def default_threads():
    return max(1, os.cpu_count() or 1)


# ----------------------------------------------------------------------------------------------
# Scalar codecs (vectorised over numpy arrays).
# ----------------------------------------------------------------------------------------------
def e4m3_to_double(codes):
    c = _c(codes, np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().or_e4m3_to_double_n(_ptr(c), _ptr(out), c.size)
    return out


def e4m3_from_float(x):
    f = _c(x, np.float32)
    out = np.empty(f.shape, np.uint8)
    lib().or_e4m3_from_float_n(_ptr(f), _ptr(out), f.size)
    return out


def f16_to_double(bits):
    b = _c(bits, np.uint16)
    out = np.empty(b.shape, np.float64)
    lib().or_f16_to_double_n(_ptr(b), _ptr(out), b.size)
    return out


def bf16_to_double(bits):
    b = _c(bits, np.uint16)
    out = np.empty(b.shape, np.float64)
    lib().or_bf16_to_double_n(_ptr(b), _ptr(out), b.size)
    return out


def to_double(bits, dtype):
    code = dtype_code(dtype)
    if code == F16:
        return f16_to_double(bits)
    if code == BF16:
        return bf16_to_double(bits)
    return e4m3_to_double(bits)


# ----------------------------------------------------------------------------------------------
# The path's three operations.
# ----------------------------------------------------------------------------------------------
class OracleError(RuntimeError):
    pass


def paged_attention(query_bits, q_dtype, key_cache, value_cache, kv_dtype, block_tables,
                    context_lens, scale, k_scale=None, v_scale=None, num_threads=None):
    """fp64 output [S, H, d] of paged decode attention (definition in pa_oracle.c).

    query_bits: uint16 [S, H, d]; key_cache/value_cache: uint16 or uint8 [NB, bs, Hkv, d];
    block_tables: int32 [S, max_blocks]; context_lens: int32 [S]; k_scale/v_scale: float32 [Hkv].
    """
    q = _c(query_bits, np.uint16)
    kc = key_cache if key_cache.flags.c_contiguous else np.ascontiguousarray(key_cache)
    vc = value_cache if value_cache.flags.c_contiguous else np.ascontiguousarray(value_cache)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    S, H, d = q.shape
    NB, bs, Hkv, d2 = kc.shape
    assert d2 == d and vc.shape == kc.shape and bt.shape[0] == S and cl.shape == (S,)
    ks = None if k_scale is None else _c(k_scale, np.float32)
    vs = None if v_scale is None else _c(v_scale, np.float32)
    out = np.zeros((S, H, d), np.float64)
    st = lib().or_paged_attention(_ptr(out), _ptr(q), dtype_code(q_dtype), _ptr(kc), _ptr(vc),
                                  dtype_code(kv_dtype), _ptr(ks), _ptr(vs), _ptr(bt), bt.shape[1],
                                  _ptr(cl), S, H, Hkv, d, bs, NB, float(scale),
                                  num_threads or default_threads())
    if st != 0:
        raise OracleError(f"or_paged_attention failed with status {st}")
    return out


def paged_prefill(query_bits, q_dtype, key_cache, value_cache, kv_dtype, block_tables, context_lens,
                  q_start, scale, k_scale=None, v_scale=None, num_threads=None):
    """fp64 output [T, H, d] of causal paged prefill attention (definition in pa_oracle.c).

    query_bits: uint16 [T, H, d], the query chunks of all sequences back to back; q_start: int32
    [S + 1] row offsets (q_start[0] = 0, q_start[S] = T); context_lens: int32 [S], each including
    its chunk; other arguments as in paged_attention.
    """
    q = _c(query_bits, np.uint16)
    kc = key_cache if key_cache.flags.c_contiguous else np.ascontiguousarray(key_cache)
    vc = value_cache if value_cache.flags.c_contiguous else np.ascontiguousarray(value_cache)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    qs = _c(q_start, np.int32)
    T, H, d = q.shape
    NB, bs, Hkv, d2 = kc.shape
    S = cl.shape[0]
    assert d2 == d and vc.shape == kc.shape and bt.shape[0] == S and qs.shape == (S + 1,) and qs[-1] == T
    ks = None if k_scale is None else _c(k_scale, np.float32)
    vs = None if v_scale is None else _c(v_scale, np.float32)
    out = np.zeros((T, H, d), np.float64)
    st = lib().or_paged_prefill(_ptr(out), _ptr(q), dtype_code(q_dtype), _ptr(kc), _ptr(vc), dtype_code(kv_dtype),
                                _ptr(ks), _ptr(vs), _ptr(bt), bt.shape[1], _ptr(cl), _ptr(qs), S, H, Hkv, d, bs,
                                NB, float(scale), num_threads or default_threads())
    if st != 0:
        raise OracleError(f"or_paged_prefill failed with status {st}")
    return out


def reshape_and_cache(key_bits, value_bits, in_dtype, key_cache, value_cache, kv_dtype,
                      slot_mapping, k_scale=None, v_scale=None):
    """Write new tokens [T, Hkv, d] into the caches in place (slot < 0 or past the pool: skipped)."""
    k = _c(key_bits, np.uint16)
    v = _c(value_bits, np.uint16)
    assert key_cache.flags.c_contiguous and value_cache.flags.c_contiguous
    sm = _c(slot_mapping, np.int64)
    NB, bs, Hkv, d = key_cache.shape
    T = sm.shape[0]
    assert k.shape == (T, Hkv, d) and v.shape == (T, Hkv, d)
    ks = None if k_scale is None else _c(k_scale, np.float32)
    vs = None if v_scale is None else _c(v_scale, np.float32)
    st = lib().or_reshape_and_cache(_ptr(k), _ptr(v), dtype_code(in_dtype), _ptr(key_cache),
                                    _ptr(value_cache), dtype_code(kv_dtype), _ptr(ks), _ptr(vs),
                                    _ptr(sm), T, Hkv, d, bs, NB)
    if st != 0:
        raise OracleError(f"or_reshape_and_cache failed with status {st}")


def copy_blocks(key_cache, value_cache, kv_dtype, block_mapping):
    """Copy whole key and value blocks for each (src, dst) pair, in place."""
    assert key_cache.flags.c_contiguous and value_cache.flags.c_contiguous
    bm = _c(block_mapping, np.int64).reshape(-1, 2)
    NB, bs, Hkv, d = key_cache.shape
    st = lib().or_copy_blocks(_ptr(key_cache), _ptr(value_cache), dtype_code(kv_dtype), _ptr(bm),
                              bm.shape[0], Hkv, d, bs, NB)
    if st != 0:
        raise OracleError(f"or_copy_blocks failed with status {st}")


def swap_blocks(dst_key_cache, dst_value_cache, src_key_cache, src_value_cache, kv_dtype, block_mapping):
    """Copy whole blocks src_pool[src] -> dst_pool[dst] for each (src, dst) pair, in place on dst."""
    for a in (dst_key_cache, dst_value_cache, src_key_cache, src_value_cache):
        assert a.flags.c_contiguous
    bm = _c(block_mapping, np.int64).reshape(-1, 2)
    NBs, bs, Hkv, d = src_key_cache.shape
    NBd = dst_key_cache.shape[0]
    assert dst_key_cache.shape[1:] == src_key_cache.shape[1:]
    st = lib().or_swap_blocks(_ptr(dst_key_cache), _ptr(dst_value_cache), _ptr(src_key_cache),
                              _ptr(src_value_cache), dtype_code(kv_dtype), _ptr(bm), bm.shape[0], Hkv, d, bs,
                              NBs, NBd)
    if st != 0:
        raise OracleError(f"or_swap_blocks failed with status {st}")


def quantize_e4m3(values_bits, in_dtype, scale_per_head):
    """E4M3 codes of a [..., Hkv, d] array of 16-bit values with per-kv-head scales: the same
    arithmetic as writing every row through reshape_and_cache into an E4M3 cache."""
    from concurrent.futures import ThreadPoolExecutor

    vb = _c(values_bits, np.uint16)
    *lead, Hkv, d = vb.shape
    T = int(np.prod(lead)) if lead else 1
    flat = vb.reshape(T, Hkv, d)
    out = np.zeros((T, 1, Hkv, d), np.uint8)
    sc = _c(scale_per_head, np.float32)
    L = lib()

    def run(lo_hi):
        lo, hi = lo_hi
        n = hi - lo
        if n <= 0:
            return 0
        part_in = flat[lo:hi]
        part_out = out[lo:hi]
        scratch = np.zeros_like(part_out)
        sm = np.arange(n, dtype=np.int64)
        return L.or_reshape_and_cache(_ptr(part_in), _ptr(part_in), dtype_code(in_dtype), _ptr(part_out),
                                      _ptr(scratch), E4M3, _ptr(sc), _ptr(sc), _ptr(sm), n, Hkv, d, 1, n)

    workers = default_threads()
    step = (T + workers - 1) // workers
    with ThreadPoolExecutor(workers) as ex:
        statuses = list(ex.map(run, [(i, min(T, i + step)) for i in range(0, T, step)]))
    if any(statuses):
        raise OracleError(f"quantize_e4m3 failed with statuses {statuses}")
    return out.reshape(vb.shape)


def quantize_e4m3_blocks(pool_bits, in_dtype, scale_per_block):
    """E4M3 codes of a whole pool [NB, bs, Hkv, d] of 16-bit values with one scale per (block, kv
    head) ([NB, Hkv]): the same arithmetic as writing every slot through reshape_and_cache into a
    per-block-scaled E4M3 cache."""
    vb = _c(pool_bits, np.uint16)
    NB, bs, Hkv, d = vb.shape
    sc = _c(np.repeat(_c(scale_per_block, np.float32), bs, axis=0), np.float32)   # one row per slot
    rows = vb.reshape(NB * bs, Hkv, d)
    out = np.zeros((NB * bs, 1, Hkv, d), np.uint8)
    scratch = np.zeros_like(out)
    sm = np.arange(NB * bs, dtype=np.int64)
    st = lib().or_reshape_and_cache(_ptr(rows), _ptr(rows), dtype_code(in_dtype), _ptr(out), _ptr(scratch),
                                    E4M3_BLOCK, _ptr(sc), _ptr(sc), _ptr(sm), NB * bs, Hkv, d, 1, NB * bs)
    if st:
        raise OracleError(f"quantize_e4m3_blocks failed with status {st}")
    return out.reshape(NB, bs, Hkv, d)
