"""Thin binding of the native block manager (include/pa_block_manager.h).

Argument marshalling only: every decision (which block, which copy-on-write pair, which host block)
is taken by the C++ manager inside libpagedattn.so. Outputs are numpy arrays, or caller-supplied
pinned torch tensors for the per-step plan so that it can go to the device with one copy each.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from .pagedattn import PA_ERR_OUT_OF_BLOCKS, PagedAttnError, _check, lib

NO_SEQUENCE = -1


class OutOfBlocks(PagedAttnError):
    pass


def _call(status, where):
    if status == PA_ERR_OUT_OF_BLOCKS:
        raise OutOfBlocks(status, where)
    _check(status, where)


_TORCH_DTYPE = {np.int64: torch.int64, np.int32: torch.int32}


def _host_out(a, dtype, count, name):
    """Address of a caller-supplied output buffer, which the manager writes through a raw host
    pointer: it must be a numpy array or a CPU (e.g. pinned) torch tensor of `dtype`, dense, with room
    for `count` elements."""
    if isinstance(a, torch.Tensor):
        if a.dtype == _TORCH_DTYPE[dtype] and a.is_cpu and a.is_contiguous() and a.numel() >= count:
            return a.data_ptr()
    elif isinstance(a, np.ndarray):
        if a.dtype == dtype and a.flags.c_contiguous and a.size >= count:
            return a.ctypes.data
    raise ValueError(f"plan_decode: `{name}` must be a dense host array of {np.dtype(dtype)} with at least "
                     f"{count} elements")


class BlockManager:
    """Owns one native manager: num_blocks device blocks of block_size tokens, num_host_blocks host
    blocks for swapping."""

    def __init__(self, num_blocks: int, block_size: int, num_host_blocks: int = 0):
        self._h = None                    # set before the call, so a failed create still closes cleanly
        h = ctypes.c_void_p()
        _call(lib.pa_bm_create(num_blocks, block_size, num_host_blocks, ctypes.byref(h)), "pa_bm_create")
        self._h = h
        self.num_blocks, self.block_size, self.num_host_blocks = num_blocks, block_size, num_host_blocks

    def close(self):
        if self._h:
            lib.pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    def add_sequence(self, seq_id: int, num_tokens: int, prefix_seq: int = NO_SEQUENCE, prefix_tokens: int = 0):
        """Returns the slots (int64) of the prompt tokens still to be written."""
        slots = np.empty(max(num_tokens, 1), np.int64)
        n = ctypes.c_int64()
        _call(lib.pa_bm_add_sequence(self._h, seq_id, num_tokens, prefix_seq, prefix_tokens, slots.ctypes.data,
                                     num_tokens, ctypes.byref(n)), "pa_bm_add_sequence")
        return slots[:n.value]

    def fork(self, parent: int, child: int):
        _call(lib.pa_bm_fork(self._h, parent, child), "pa_bm_fork")

    def append_slots(self, seq_ids):
        """Returns (slot_mapping [n] int64, copy-on-write pairs [k, 2] int64)."""
        ids = np.ascontiguousarray(seq_ids, np.int64)
        n = len(ids)
        slots = np.empty(max(n, 1), np.int64)
        pairs = np.empty((max(n, 1), 2), np.int64)
        k = ctypes.c_int()
        _call(lib.pa_bm_append_slots(self._h, ids.ctypes.data, n, slots.ctypes.data, pairs.ctypes.data,
                                     ctypes.byref(k)), "pa_bm_append_slots")
        return slots[:n], pairs[:k.value]

    def block_tables(self, seq_ids, max_blocks: int, pad: int = 0):
        """Returns (tables [n, max_blocks] int32, context_lens [n] int32)."""
        ids = np.ascontiguousarray(seq_ids, np.int64)
        n = len(ids)
        tables = np.empty((n, max(max_blocks, 1)), np.int32)
        lens = np.empty(max(n, 1), np.int32)
        _call(lib.pa_bm_block_tables(self._h, ids.ctypes.data, n, tables.ctypes.data, max_blocks, pad,
                                     lens.ctypes.data), "pa_bm_block_tables")
        return tables[:, :max_blocks], lens[:n]

    def plan_decode(self, seq_ids, max_blocks: int, pad: int = 0, out=None):
        """One decode step's plan. `out` may hold preallocated (e.g. pinned) tensors or arrays
        (slot_mapping [n] int64, cow [n, 2] int64, tables [n, max_blocks] int32, lens [n] int32);
        returns (slot_mapping, cow_pairs[:k], tables, lens)."""
        ids = np.ascontiguousarray(seq_ids, np.int64)
        n = len(ids)
        if out is None:
            out = (np.empty(n, np.int64), np.empty((n, 2), np.int64), np.empty((n, max_blocks), np.int32),
                   np.empty(n, np.int32))
        slots, cow, tables, lens = out
        k = ctypes.c_int()
        _call(lib.pa_bm_plan_decode(self._h, ids.ctypes.data, n, _host_out(slots, np.int64, n, "slot_mapping"),
                                    _host_out(cow, np.int64, 2 * n, "cow"), ctypes.byref(k),
                                    _host_out(tables, np.int32, n * max_blocks, "tables"), max_blocks, pad,
                                    _host_out(lens, np.int32, n, "lens")), "pa_bm_plan_decode")
        return slots, cow[:k.value], tables, lens

    def free_sequence(self, seq_id: int):
        _call(lib.pa_bm_free_sequence(self._h, seq_id), "pa_bm_free_sequence")

    def _swap(self, fn, name, seq_id):
        _, nblocks, _ = self.sequence_info(seq_id)
        m = np.empty((max(nblocks, 1), 2), np.int64)
        k = ctypes.c_int()
        _call(fn(self._h, seq_id, m.ctypes.data, nblocks, ctypes.byref(k)), name)
        return m[:k.value]

    def swap_out(self, seq_id: int):
        """(device block, host block) pairs for swap_blocks."""
        return self._swap(lib.pa_bm_swap_out, "pa_bm_swap_out", seq_id)

    def swap_in(self, seq_id: int):
        """(host block, device block) pairs for swap_blocks."""
        return self._swap(lib.pa_bm_swap_in, "pa_bm_swap_in", seq_id)

    def num_free_blocks(self):
        d, h = ctypes.c_int(), ctypes.c_int()
        _call(lib.pa_bm_num_free_blocks(self._h, ctypes.byref(d), ctypes.byref(h)), "pa_bm_num_free_blocks")
        return d.value, h.value

    def sequence_info(self, seq_id: int):
        """(tokens, blocks, swapped)."""
        t, b, s = ctypes.c_int64(), ctypes.c_int(), ctypes.c_int()
        _call(lib.pa_bm_sequence_info(self._h, seq_id, ctypes.byref(t), ctypes.byref(b), ctypes.byref(s)),
              "pa_bm_sequence_info")
        return t.value, b.value, bool(s.value)

    def ref_count(self, block: int) -> int:
        c = ctypes.c_int()
        _call(lib.pa_bm_ref_count(self._h, block, ctypes.byref(c)), "pa_bm_ref_count")
        return c.value
