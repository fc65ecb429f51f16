"""The native block manager under host allocation failure (CPU).

The manager's C++ source is rebuilt together with a replacement of the global operator new that
throws std::bad_alloc at the k-th allocation after it is armed. A fixed session (create, add with and
without a shared prefix, fork, appends with copy-on-write, decode plans, swap out and in, frees) runs
once for every k up to the session's allocation count, beside the manager's oracle. Each call must
either succeed with the oracle's result or return PA_ERR_HOST_MEMORY, and after every call all
observables (free counts, reference counts, sequence info, block tables) must equal the oracle's,
which skips a failed call. Later calls may then fail for ordinary reasons (a prefix that was never
added); they must fail exactly as the oracle does. So an allocation failure anywhere leaves the
manager as it was, and nothing is thrown across the C ABI.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

from oracle.block_manager import BlockManagerOracle, OracleBlockError, OutOfBlocks as OracleOut

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

INJECTOR = r"""
#include <cstdlib>
#include <new>

static long countdown = -1;  // allocations left before the failing one; -1: never fail
static long allocations = 0;

extern "C" void oom_fail_after(long n) { countdown = n; }
extern "C" long oom_allocations() { return allocations; }

static void* allocate(std::size_t n) {
  ++allocations;
  if (countdown == 0) {
    countdown = -1;
    throw std::bad_alloc();
  }
  if (countdown > 0) --countdown;
  void* p = std::malloc(n ? n : 1);
  if (!p) throw std::bad_alloc();
  return p;
}

void* operator new(std::size_t n) { return allocate(n); }
void* operator new[](std::size_t n) { return allocate(n); }
void* operator new(std::size_t n, const std::nothrow_t&) noexcept {
  try { return allocate(n); } catch (...) { return nullptr; }
}
void operator delete(void* p) noexcept { std::free(p); }
void operator delete[](void* p) noexcept { std::free(p); }
void operator delete(void* p, std::size_t) noexcept { std::free(p); }
void operator delete[](void* p, std::size_t) noexcept { std::free(p); }
"""


@pytest.fixture(scope="module")
def injected(tmp_path_factory):
    from pagedattention_paged_kv_attention_b200 import block_manager, pagedattn as P
    d = tmp_path_factory.mktemp("oom")
    src = d / "inject.cpp"
    src.write_text(INJECTOR)
    so = d / "libbm_oom.so"
    # -Bsymbolic: the manager's own calls bind to this library's operator new.
    subprocess.run(["g++", "-std=c++17", "-O1", "-shared", "-fPIC", "-Wl,-Bsymbolic", "-I",
                    os.path.join(ROOT, "include"), "-o", str(so),
                    os.path.join(ROOT, "pagedattention_paged_kv_attention_b200", "csrc", "pa_block_manager.cpp"),
                    str(src)], check=True)
    lib = ctypes.CDLL(str(so))
    for name in P.EXPORTS:
        if name.startswith("pa_bm_"):
            fn, real = getattr(lib, name), getattr(P.lib, name)
            fn.argtypes, fn.restype = real.argtypes, real.restype
    lib.oom_fail_after.argtypes = [ctypes.c_long]
    lib.oom_allocations.restype = ctypes.c_long
    saved = block_manager.lib
    block_manager.lib = lib           # the wrapper looks its library up at call time
    yield lib, block_manager, P
    block_manager.lib = saved


NB, BS, NH = 12, 4, 6
IDS = [0, 1, 2, 3]


def steps(bm, ref):
    """(native call, oracle call) pairs; each native result is compared with the oracle's."""
    tbl = lambda r: (r[2].tolist(), r[3].tolist())
    return [
        (lambda: bm.add_sequence(0, 10).tolist(), lambda: ref.add_sequence(0, 10)),
        (lambda: bm.add_sequence(1, 9, 0, 8).tolist(), lambda: ref.add_sequence(1, 9, 0, 8)),
        (lambda: bm.fork(1, 2), lambda: ref.fork(1, 2)),
        (lambda: bm.append_slots([0, 1, 2])[0].tolist(), lambda: ref.append_slots([0, 1, 2])[0]),
        (lambda: tbl(bm.plan_decode([0, 1, 2], 8, -1)),
         lambda: (ref.append_slots([0, 1, 2]), ref.block_tables([0, 1, 2], 8, -1))[1]),
        (lambda: [tuple(p) for p in bm.swap_out(2).tolist()], lambda: ref.swap_out(2)),
        (lambda: bm.append_slots([0, 1])[0].tolist(), lambda: ref.append_slots([0, 1])[0]),
        (lambda: [tuple(p) for p in bm.swap_in(2).tolist()], lambda: ref.swap_in(2)),
        (lambda: bm.free_sequence(1), lambda: ref.free_sequence(1)),
        (lambda: bm.add_sequence(3, 5, 2, 5).tolist(), lambda: ref.add_sequence(3, 5, 2, 5)),
        (lambda: tbl(bm.plan_decode([0, 2, 3], 8, -1)),
         lambda: (ref.append_slots([0, 2, 3]), ref.block_tables([0, 2, 3], 8, -1))[1]),
        (lambda: bm.free_sequence(0), lambda: ref.free_sequence(0)),
        (lambda: bm.free_sequence(2), lambda: ref.free_sequence(2)),
        (lambda: bm.free_sequence(3), lambda: ref.free_sequence(3)),
    ]


def snapshot(bm, ref):
    assert bm.num_free_blocks() == (ref.num_free_blocks(), ref.num_free_host_blocks())
    for b in range(NB):
        assert bm.ref_count(b) == ref.ref[b]
    for s in IDS:
        if s in ref.tables or s in ref.swapped:
            tokens, blocks, swapped = bm.sequence_info(s)
            assert (tokens, blocks, swapped) == (ref.lens[s], len(ref.tables.get(s, ref.swapped.get(s))),
                                                 s in ref.swapped)
    resident = sorted(ref.tables)
    if resident:
        t, l = bm.block_tables(resident, 8, pad=-1)
        assert (t.tolist(), l.tolist()) == ref.block_tables(resident, 8, pad=-1)


def run_session(lib, BM, P, fail_at):
    """Runs the session with the fail_at-th allocation failing (-1: none); returns the number of
    calls that reported PA_ERR_HOST_MEMORY."""
    lib.oom_fail_after(fail_at)
    try:
        bm = BM.BlockManager(NB, BS, NH)
    except P.PagedAttnError as e:
        assert e.status == P.PA_ERR_HOST_MEMORY
        lib.oom_fail_after(-1)
        bm = BM.BlockManager(NB, BS, NH)
        failed = 1
    else:
        failed = 0
    ref = BlockManagerOracle(NB, BS, NH)
    for native, oracle_call in steps(bm, ref):
        got, status = None, P.PA_OK
        try:
            got = native()
        except P.PagedAttnError as e:
            status = e.status
        if status == P.PA_ERR_HOST_MEMORY:
            failed += 1                   # the oracle skips the failed call
        else:
            want, expected = None, P.PA_OK
            try:
                want = oracle_call()
            except OracleOut:
                expected = P.PA_ERR_OUT_OF_BLOCKS
            except OracleBlockError:
                expected = P.PA_ERR_INVALID_ARGUMENT
            assert status == expected and got == want
        snapshot(bm, ref)
    bm.close()
    lib.oom_fail_after(-1)
    return failed


def test_every_allocation_failure_leaves_the_manager_unchanged(injected):
    lib, BM, P = injected
    before = lib.oom_allocations()
    assert run_session(lib, BM, P, -1) == 0
    total = lib.oom_allocations() - before
    assert total > 30                 # the session does allocate (the injector is in effect)
    failures = [run_session(lib, BM, P, k) for k in range(total)]
    assert all(f == 1 for f in failures), failures   # each armed failure surfaced exactly once
