"""Thin ctypes binding of libpagedattn.so (the C ABI in include/pagedattn.h).

Argument marshalling only: tensors become device pointers and the current CUDA stream becomes a
cudaStream_t; every step of the computation runs in the library's CUDA kernels. PyTorch is used for
device memory and streams. Importing this module fails loudly if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# PA_LIBRARY_PATH selects another in-tree build of the same library (e.g. the timing-trace variant).
LIBRARY_PATH = os.environ.get("PA_LIBRARY_PATH") or os.path.join(_HERE, "libpagedattn.so")

(PA_OK, PA_ERR_INVALID_ARGUMENT, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE_TOO_SMALL, PA_ERR_CUDA, PA_ERR_OUT_OF_BLOCKS,
 PA_ERR_HOST_MEMORY) = range(7)
PA_F16, PA_BF16, PA_FP8_E4M3, PA_FP8_E4M3_BLOCK = 0, 1, 2, 3
PA_DEVERR_BLOCK_ID, PA_DEVERR_CONTEXT_LEN, PA_DEVERR_TIMEOUT = 0x1, 0x2, 0x4
WORKSPACE_HEADER_BYTES = 256

# Every symbol the public header declares (checked by the CPU test suite).
EXPORTS = (
    "pa_paged_attention_partition_size", "pa_paged_attention_workspace_size", "pa_paged_attention",
    "pa_reshape_and_cache", "pa_copy_blocks", "pa_copy_blocks_check", "pa_get_device_error",
    "pa_clear_device_error", "pa_status_string", "pa_paged_attention_static", "pa_selftest_wait_timeout",
    "pa_swap_blocks", "pa_reshape_and_cache_layers", "pa_copy_blocks_layers", "pa_paged_prefill",
    # include/pa_block_manager.h
    "pa_bm_create", "pa_bm_destroy", "pa_bm_add_sequence", "pa_bm_fork", "pa_bm_append_slots",
    "pa_bm_block_tables", "pa_bm_plan_decode", "pa_bm_free_sequence", "pa_bm_swap_out", "pa_bm_swap_in",
    "pa_bm_num_free_blocks", "pa_bm_sequence_info", "pa_bm_ref_count",
    # include/pa_probe.h
    "pa_probe_stream_read", "pa_probe_paged_read",
)

if not os.path.exists(LIBRARY_PATH):
    raise ImportError(f"{LIBRARY_PATH} is missing: build it with "
                      "`python -m pagedattention_paged_kv_attention_b200.build` (no CPU fallback exists)")

lib = ctypes.CDLL(LIBRARY_PATH)
_p, _i, _sz, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
lib.pa_status_string.restype = ctypes.c_char_p
lib.pa_status_string.argtypes = [_i]
lib.pa_paged_attention_partition_size.restype = _i
lib.pa_paged_attention_partition_size.argtypes = [_i, _i, _i, _i, _i]
lib.pa_paged_attention_workspace_size.restype = _sz
lib.pa_paged_attention_workspace_size.argtypes = [_i, _i, _i, _i, _i, _i]
lib.pa_paged_attention.restype = _i
lib.pa_paged_attention.argtypes = [_p, _p, _i, _p, _p, _i, _p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _i, _i, _f,
                                   _i, _p, _sz, _p]
lib.pa_paged_attention_static.restype = _i
lib.pa_paged_attention_static.argtypes = [_p, _p, _i, _p, _p, _i, _p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _i, _i,
                                          _f, _i, _p, _p]
lib.pa_probe_stream_read.restype = _i
lib.pa_probe_stream_read.argtypes = [_p, _sz, _i, _p, _p]
lib.pa_probe_paged_read.restype = _i
lib.pa_probe_paged_read.argtypes = [_p, _p, _i, _p, _i, _p, _i, _i, _i, _i, _i, _p, _p]
lib.pa_paged_prefill.restype = _i
lib.pa_paged_prefill.argtypes = [_p, _p, _i, _p, _p, _i, _p, _p, _p, _i, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _f,
                                 _p, _sz, _p]
lib.pa_reshape_and_cache.restype = _i
lib.pa_reshape_and_cache.argtypes = [_p, _p, _i, _p, _p, _i, _p, _p, _p, _i, _i, _i, _i, _i, _p]
lib.pa_copy_blocks.restype = _i
lib.pa_copy_blocks.argtypes = [_p, _p, _i, _p, _i, _i, _i, _i, _i, _p]
lib.pa_reshape_and_cache_layers.restype = _i
lib.pa_reshape_and_cache_layers.argtypes = [_p, _p, _i, _p, _p, _i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p]
lib.pa_copy_blocks_layers.restype = _i
lib.pa_copy_blocks_layers.argtypes = [_p, _p, _i, _i, _p, _i, _i, _i, _i, _i, _p]
_i64 = ctypes.c_int64
_ip = ctypes.POINTER(ctypes.c_int)
_i64p = ctypes.POINTER(ctypes.c_int64)
lib.pa_bm_create.restype = _i
lib.pa_bm_create.argtypes = [_i, _i, _i, ctypes.POINTER(_p)]
lib.pa_bm_destroy.restype = None
lib.pa_bm_destroy.argtypes = [_p]
lib.pa_bm_add_sequence.restype = _i
lib.pa_bm_add_sequence.argtypes = [_p, _i64, _i64, _i64, _i64, _p, _i64, _i64p]
lib.pa_bm_fork.restype = _i
lib.pa_bm_fork.argtypes = [_p, _i64, _i64]
lib.pa_bm_append_slots.restype = _i
lib.pa_bm_append_slots.argtypes = [_p, _p, _i, _p, _p, _ip]
lib.pa_bm_block_tables.restype = _i
lib.pa_bm_block_tables.argtypes = [_p, _p, _i, _p, _i, ctypes.c_int32, _p]
lib.pa_bm_plan_decode.restype = _i
lib.pa_bm_plan_decode.argtypes = [_p, _p, _i, _p, _p, _ip, _p, _i, ctypes.c_int32, _p]
lib.pa_bm_free_sequence.restype = _i
lib.pa_bm_free_sequence.argtypes = [_p, _i64]
lib.pa_bm_swap_out.restype = _i
lib.pa_bm_swap_out.argtypes = [_p, _i64, _p, _i, _ip]
lib.pa_bm_swap_in.restype = _i
lib.pa_bm_swap_in.argtypes = [_p, _i64, _p, _i, _ip]
lib.pa_bm_num_free_blocks.restype = _i
lib.pa_bm_num_free_blocks.argtypes = [_p, _ip, _ip]
lib.pa_bm_sequence_info.restype = _i
lib.pa_bm_sequence_info.argtypes = [_p, _i64, _i64p, _ip, _ip]
lib.pa_bm_ref_count.restype = _i
lib.pa_bm_ref_count.argtypes = [_p, _i, _ip]
lib.pa_swap_blocks.restype = _i
lib.pa_swap_blocks.argtypes = [_p, _p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _i, _p]
lib.pa_copy_blocks_check.restype = _i
lib.pa_copy_blocks_check.argtypes = [_p, _i, _i]
lib.pa_get_device_error.restype = _i
lib.pa_get_device_error.argtypes = [_p, ctypes.POINTER(ctypes.c_uint), _p]
lib.pa_clear_device_error.restype = _i
lib.pa_clear_device_error.argtypes = [_p, _p]
lib.pa_selftest_wait_timeout.restype = _i
lib.pa_selftest_wait_timeout.argtypes = [_p, ctypes.c_ulonglong, _p]


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.pa_status_string(status).decode()}")


def _check(status: int, where: str):
    if status != PA_OK:
        raise PagedAttnError(status, where)


def dtype_code(t: torch.dtype) -> int:
    if t == torch.float16:
        return PA_F16
    if t == torch.bfloat16:
        return PA_BF16
    if t in (torch.uint8, torch.float8_e4m3fn):
        return PA_FP8_E4M3
    raise ValueError(f"unsupported dtype {t}")


def cache_code(cache: torch.Tensor, k_scale=None) -> int:
    """The cache format: 16-bit, or E4M3 with per-kv-head scales ([Hkv]) or per-(block, kv head)
    scales ([num_blocks, Hkv])."""
    code = dtype_code(cache.dtype)
    if code == PA_FP8_E4M3 and k_scale is not None and k_scale.dim() == 2:
        return PA_FP8_E4M3_BLOCK
    return code


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_I32, _I64, _F32 = (torch.int32,), (torch.int64,), (torch.float32,)


def _arg(t, name, dtypes=None, dim=None, cuda=True):
    """The pointer of a tensor argument, after the checks the C ABI cannot make from a pointer: a dense
    row-major layout, the element type the call reads, the rank, and (for kernel operands) residence
    on a CUDA device. None passes through as a null pointer."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if dim is not None and t.dim() not in ((dim,) if isinstance(dim, int) else dim):
        raise ValueError(f"{name}: expected {dim} dimensions, got shape {tuple(t.shape)}")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name}: expected dtype {' or '.join(map(str, dtypes))}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous (the library reads a dense row-major layout)")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _same(a, b, what):
    if a.shape != b.shape or a.dtype != b.dtype:
        raise ValueError(f"{what}: shapes/dtypes differ ({tuple(a.shape)} {a.dtype} vs {tuple(b.shape)} {b.dtype})")


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def partition_size(num_seqs, num_heads, num_kv_heads, max_context_len, partition_size=0) -> int:
    return lib.pa_paged_attention_partition_size(num_seqs, num_heads, num_kv_heads, max_context_len, partition_size)


def workspace_size(num_seqs, num_heads, num_kv_heads, head_size, max_context_len, partition_size=0) -> int:
    return lib.pa_paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads, head_size, max_context_len,
                                                 partition_size)


def make_workspace(num_seqs, num_heads, num_kv_heads, head_size, max_context_len, partition_size=0,
                   device="cuda") -> torch.Tensor:
    """A zeroed workspace (error word cleared) sized for these arguments."""
    n = workspace_size(num_seqs, num_heads, num_kv_heads, head_size, max_context_len, partition_size)
    if n == 0:
        raise ValueError("invalid sizes for a workspace")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def paged_attention(out, query, key_cache, value_cache, block_tables, context_lens, scale, max_context_len,
                    workspace, k_scale=None, v_scale=None, partition_size=0, stream=None):
    """out[S,H,d] = paged decode attention of query[S,H,d] over key/value_cache[NB,bs,Hkv,d]."""
    S, H, d = query.shape
    NB, bs, Hkv, d2 = key_cache.shape
    _same(out, query, "out/query")
    _same(key_cache, value_cache, "key_cache/value_cache")
    st = lib.pa_paged_attention(
        _arg(out, "out"), _arg(query, "query"), dtype_code(query.dtype), _arg(key_cache, "key_cache"),
        _arg(value_cache, "value_cache"), cache_code(key_cache, k_scale), _arg(k_scale, "k_scale", _F32, (1, 2)),
        _arg(v_scale, "v_scale", _F32, (1, 2)), _arg(block_tables, "block_tables", _I32, 2), block_tables.shape[1],
        _arg(context_lens, "context_lens", _I32, 1), S, H, Hkv, d, bs, NB, int(max_context_len), float(scale),
        int(partition_size), _arg(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(st, "pa_paged_attention")
    return out


def paged_prefill(out, query, key_cache, value_cache, block_tables, context_lens, q_start, scale, max_q_len,
                  workspace, k_scale=None, v_scale=None, stream=None):
    """Causal prefill: out[T,H,d] for query chunks query[T,H,d] (rows q_start[s]..q_start[s+1]-1 of
    sequence s, the last rows of its context_lens[s] cached tokens) over key/value_cache[NB,bs,Hkv,d].
    FP8 (uint8 E4M3) caches take k_scale/v_scale: [Hkv] per kv head, or [NB, Hkv] per block."""
    T, H, d = query.shape
    NB, bs, Hkv, _ = key_cache.shape
    _same(out, query, "out/query")
    _same(key_cache, value_cache, "key_cache/value_cache")
    st = lib.pa_paged_prefill(_arg(out, "out"), _arg(query, "query"), dtype_code(query.dtype),
                              _arg(key_cache, "key_cache"), _arg(value_cache, "value_cache"),
                              cache_code(key_cache, k_scale), _arg(k_scale, "k_scale", _F32, (1, 2)),
                              _arg(v_scale, "v_scale", _F32, (1, 2)), _arg(block_tables, "block_tables", _I32, 2),
                              block_tables.shape[1], _arg(context_lens, "context_lens", _I32, 1),
                              _arg(q_start, "q_start", _I32, 1), context_lens.shape[0], T, H, Hkv, d, bs, NB,
                              int(max_q_len), float(scale), _arg(workspace, "workspace"),
                              workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "pa_paged_prefill")


def paged_attention_static(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                           max_context_len, k_scale=None, v_scale=None, partition_size=0, device_error_out=None,
                           stream=None):
    """paged_attention with the library's fixed scratch array instead of a caller workspace (for
    callers that cannot allocate device memory). device_error_out: optional int32/uint32 device
    tensor of one element that receives the device error word."""
    S, H, d = query.shape
    NB, bs, Hkv, d2 = key_cache.shape
    _same(out, query, "out/query")
    _same(key_cache, value_cache, "key_cache/value_cache")
    st = lib.pa_paged_attention_static(
        _arg(out, "out"), _arg(query, "query"), dtype_code(query.dtype), _arg(key_cache, "key_cache"),
        _arg(value_cache, "value_cache"), cache_code(key_cache, k_scale), _arg(k_scale, "k_scale", _F32, (1, 2)),
        _arg(v_scale, "v_scale", _F32, (1, 2)), _arg(block_tables, "block_tables", _I32, 2), block_tables.shape[1],
        _arg(context_lens, "context_lens", _I32, 1), S, H, Hkv, d, bs, NB, int(max_context_len), float(scale),
        int(partition_size), _arg(device_error_out, "device_error_out", (torch.int32, torch.uint32)),
        _stream(stream))
    _check(st, "pa_paged_attention_static")
    return out


def reshape_and_cache(key, value, key_cache, value_cache, slot_mapping, k_scale=None, v_scale=None, stream=None):
    """Write key/value[T,Hkv,d] into the caches at slot_mapping[T] (int64)."""
    T, Hkv, d = key.shape
    NB, bs = key_cache.shape[0], key_cache.shape[1]
    _same(key, value, "key/value")
    _same(key_cache, value_cache, "key_cache/value_cache")
    st = lib.pa_reshape_and_cache(_arg(key, "key"), _arg(value, "value"), dtype_code(key.dtype),
                                  _arg(key_cache, "key_cache"), _arg(value_cache, "value_cache"),
                                  cache_code(key_cache, k_scale), _arg(k_scale, "k_scale", _F32, (1, 2)),
                                  _arg(v_scale, "v_scale", _F32, (1, 2)),
                                  _arg(slot_mapping, "slot_mapping", _I64, 1), T, Hkv, d, bs, NB, _stream(stream))
    _check(st, "pa_reshape_and_cache")


def copy_blocks(key_cache, value_cache, block_mapping, stream=None):
    """Copy whole blocks block_mapping[N,2] (src, dst) (int64, device) in both caches."""
    NB, bs, Hkv, d = key_cache.shape
    _same(key_cache, value_cache, "key_cache/value_cache")
    st = lib.pa_copy_blocks(_arg(key_cache, "key_cache"), _arg(value_cache, "value_cache"),
                            dtype_code(key_cache.dtype), _arg(block_mapping, "block_mapping", _I64, 2),
                            block_mapping.shape[0], Hkv, d, bs, NB, _stream(stream))
    _check(st, "pa_copy_blocks")


def pointer_array(tensors, device="cuda"):
    """A device int64 array holding the data pointers of `tensors` (for the *_layers calls); each tensor
    must be a contiguous CUDA tensor."""
    for i, t in enumerate(tensors):
        _arg(t, f"layer {i} tensor")
    return torch.tensor([t.data_ptr() for t in tensors], dtype=torch.int64, device=device)


def reshape_and_cache_layers(keys, values, key_caches, value_caches, slot_mapping, k_scales=None, v_scales=None,
                             stream=None):
    """reshape_and_cache over all layers in one launch; arguments are per-layer lists of tensors."""
    L = len(key_caches)
    T, Hkv, d = keys[0].shape
    NB, bs = key_caches[0].shape[0], key_caches[0].shape[1]
    arrays = [pointer_array(x) for x in (keys, values, key_caches, value_caches)]
    ks = pointer_array(k_scales) if k_scales is not None else None
    vs = pointer_array(v_scales) if v_scales is not None else None
    st = lib.pa_reshape_and_cache_layers(*[_ptr(a) for a in arrays[:2]], dtype_code(keys[0].dtype),
                                         *[_ptr(a) for a in arrays[2:]],
                                         cache_code(key_caches[0], k_scales[0] if k_scales is not None else None), _ptr(ks),
                                         _ptr(vs), _arg(slot_mapping, "slot_mapping", _I64, 1), T, L, Hkv, d, bs, NB,
                                         _stream(stream))
    _check(st, "pa_reshape_and_cache_layers")
    return arrays  # keep the pointer arrays alive until the stream has used them


def copy_blocks_layers(key_caches, value_caches, block_mapping, stream=None):
    """copy_blocks over all layers in one launch (per-layer lists of cache tensors)."""
    NB, bs, Hkv, d = key_caches[0].shape
    kp, vp = pointer_array(key_caches), pointer_array(value_caches)
    st = lib.pa_copy_blocks_layers(_ptr(kp), _ptr(vp), len(key_caches), dtype_code(key_caches[0].dtype),
                                   _arg(block_mapping, "block_mapping", _I64, 2), block_mapping.shape[0], Hkv, d, bs,
                                   NB, _stream(stream))
    _check(st, "pa_copy_blocks_layers")
    return kp, vp


def swap_blocks(dst_key_cache, dst_value_cache, src_key_cache, src_value_cache, block_mapping, stream=None):
    """Copy whole blocks src_pool[m[i,0]] -> dst_pool[m[i,1]]; pools on the device or in pinned host memory."""
    NBs, bs, Hkv, d = src_key_cache.shape
    NBd = dst_key_cache.shape[0]
    # Pools and mapping may be device or pinned host memory; the library refuses pageable memory.
    st = lib.pa_swap_blocks(_arg(dst_key_cache, "dst_key_cache", cuda=False),
                            _arg(dst_value_cache, "dst_value_cache", cuda=False),
                            _arg(src_key_cache, "src_key_cache", cuda=False),
                            _arg(src_value_cache, "src_value_cache", cuda=False), dtype_code(src_key_cache.dtype),
                            _arg(block_mapping, "block_mapping", _I64, 2, cuda=False), block_mapping.shape[0], Hkv,
                            d, bs, NBs, NBd, _stream(stream))
    _check(st, "pa_swap_blocks")


def copy_blocks_check(block_mapping_host: torch.Tensor, num_blocks: int) -> bool:
    m = block_mapping_host.to(torch.int64).contiguous().cpu()
    return lib.pa_copy_blocks_check(_ptr(m), m.shape[0], num_blocks) == PA_OK


def get_device_error(workspace, stream=None) -> int:
    v = ctypes.c_uint(0)
    _check(lib.pa_get_device_error(_ptr(workspace), ctypes.byref(v), _stream(stream)), "pa_get_device_error")
    return v.value


def selftest_wait_timeout(device_error_word, limit_ns, stream=None):
    """Run the bounded-wait self-test: a wait that nothing satisfies gives up after limit_ns and ORs
    PA_DEVERR_TIMEOUT into device_error_word (a one-element int32 device tensor)."""
    _check(lib.pa_selftest_wait_timeout(_ptr(device_error_word), int(limit_ns), _stream(stream)),
           "pa_selftest_wait_timeout")


def clear_device_error(workspace, stream=None):
    _check(lib.pa_clear_device_error(_ptr(workspace), _stream(stream)), "pa_clear_device_error")


def probe_stream_read(buf, repeat=1, sink=None, stream=None):
    """Read-bandwidth probe (include/pa_probe.h): reads every byte of the device tensor `buf`,
    `repeat` times over, with 16-byte loads and no compute. `sink`: optional one-element int64 device
    tensor the probe may write."""
    if sink is None:
        sink = torch.zeros(1, dtype=torch.int64, device=buf.device)
    nbytes = buf.numel() * buf.element_size()
    _check(lib.pa_probe_stream_read(_arg(buf, "buf"), nbytes, int(repeat), _arg(sink, "sink", _I64),
                                    _stream(stream)), "pa_probe_stream_read")
    return sink


def probe_paged_read(key_cache, value_cache, block_tables, context_lens, sink=None, stream=None):
    """Reads exactly the K/V rows of the batch's valid tokens through the block table, with plain loads
    and no compute (include/pa_probe.h)."""
    if sink is None:
        sink = torch.zeros(1, dtype=torch.int64, device=key_cache.device)
    NB, bs, Hkv, d = key_cache.shape
    _same(key_cache, value_cache, "key_cache/value_cache")
    S, max_blocks = block_tables.shape
    _check(lib.pa_probe_paged_read(_arg(key_cache, "key_cache", dim=4), _arg(value_cache, "value_cache", dim=4),
                                   dtype_code(key_cache.dtype), _arg(block_tables, "block_tables", _I32, 2),
                                   max_blocks, _arg(context_lens, "context_lens", _I32, 1), S, Hkv, d, bs, NB,
                                   _arg(sink, "sink", _I64), _stream(stream)), "pa_probe_paged_read")
    return sink
