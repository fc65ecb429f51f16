"""The native block manager (C++, through the C ABI) against its oracle, on the CPU: the same
seeded sessions of add / prefix-share / fork / append / free / swap calls give the same slots,
copy-on-write pairs, swap mappings, block tables, reference counts and free counts, decision by
decision (the allocation policy is fixed, so the results are unique). Failures (pool exhausted,
bad ids) must happen on the same calls and change nothing. The oracle itself is pinned in
test_oracle_block_manager.py."""
import numpy as np
import pytest

from oracle.block_manager import BlockManagerOracle, OracleBlockError, OutOfBlocks as OracleOut


@pytest.fixture(scope="module")
def BM():
    from pagedattention_paged_kv_attention_b200 import build
    build.build()
    from pagedattention_paged_kv_attention_b200 import block_manager
    return block_manager


def snapshot(bm, ref, ids):
    """Compare every observable of the two managers."""
    assert bm.num_free_blocks() == (ref.num_free_blocks(), ref.num_free_host_blocks())
    for b in range(ref.num_blocks):
        assert bm.ref_count(b) == ref.ref[b]
    resident = sorted(ref.tables)
    for s in ids:
        if s in ref.tables or s in ref.swapped:
            tokens, blocks, swapped = bm.sequence_info(s)
            assert tokens == ref.lens[s] and swapped == (s in ref.swapped)
            assert blocks == len(ref.tables[s] if s in ref.tables else ref.swapped[s])
    if resident:
        width = max(len(ref.tables[s]) for s in resident)
        t, l = bm.block_tables(resident, width, pad=-1)
        rt, rl = ref.block_tables(resident, width, pad=-1)
        assert t.tolist() == rt and l.tolist() == rl


def run_both(bm, ref, fn_native, fn_ref):
    """Both succeed with equal results, or both fail the same way."""
    try:
        want = fn_ref()
    except OracleOut:
        with pytest.raises(Exception) as e:
            fn_native()
        assert type(e.value).__name__ == "OutOfBlocks"
        return None
    except OracleBlockError:
        with pytest.raises(Exception) as e:
            fn_native()
        assert "INVALID_ARGUMENT" in str(e.value)
        return None
    return fn_native(), want


@pytest.mark.parametrize("seed", range(8))
def test_sessions_match_oracle(BM, seed):
    rng = np.random.default_rng(100 + seed)
    nb, bs, nh = int(rng.integers(12, 64)), int(rng.choice([1, 2, 4, 16])), int(rng.integers(0, 24))
    bm, ref = BM.BlockManager(nb, bs, nh), BlockManagerOracle(nb, bs, nh)
    ids, next_id, done = [], 0, 0
    for step in range(400):
        resident = sorted(ref.tables)
        op = rng.choice(["add", "prefix", "fork", "append", "append", "append", "plan", "free", "swap_out",
                         "swap_in", "bad"])
        if op == "add":
            n = int(rng.integers(0, 4 * bs))
            r = run_both(bm, ref, lambda: bm.add_sequence(next_id, n), lambda: ref.add_sequence(next_id, n))
            if r:
                assert r[0].tolist() == r[1]
            ids.append(next_id)
            next_id += 1
        elif op == "prefix" and resident:
            p = resident[rng.integers(len(resident))]
            n = int(rng.integers(0, 4 * bs))
            k = int(rng.integers(0, n + 1))
            r = run_both(bm, ref, lambda: bm.add_sequence(next_id, n, p, k), lambda: ref.add_sequence(next_id, n, p, k))
            if r:
                assert r[0].tolist() == r[1]
            ids.append(next_id)
            next_id += 1
        elif op == "fork" and resident:
            p = resident[rng.integers(len(resident))]
            run_both(bm, ref, lambda: bm.fork(p, next_id), lambda: ref.fork(p, next_id))
            ids.append(next_id)
            next_id += 1
        elif op in ("append", "plan") and resident:
            sel = [resident[i] for i in rng.permutation(len(resident))[:int(rng.integers(1, len(resident) + 1))]]
            if op == "append":
                r = run_both(bm, ref, lambda: bm.append_slots(sel), lambda: ref.append_slots(sel))
                if r:
                    (slots, pairs), (rs, rp) = r
                    assert slots.tolist() == rs and [tuple(x) for x in pairs.tolist()] == rp
                    done += 1
            else:
                width = max(len(ref.tables[s]) for s in sel) + 1
                def ref_plan():
                    s, p = ref.append_slots(sel)
                    t, l = ref.block_tables(sel, width, pad=7)
                    return s, p, t, l
                r = run_both(bm, ref, lambda: bm.plan_decode(sel, width, pad=7), ref_plan)
                if r:
                    (s, p, t, l), (rs, rp, rt, rl) = r
                    assert s.tolist() == rs and [tuple(x) for x in p.tolist()] == rp
                    assert t.tolist() == rt and l.tolist() == rl
                    done += 1
        elif op == "free" and ids:
            s = ids[rng.integers(len(ids))]
            run_both(bm, ref, lambda: bm.free_sequence(s), lambda: ref.free_sequence(s))
        elif op == "swap_out" and resident:
            s = resident[rng.integers(len(resident))]
            r = run_both(bm, ref, lambda: bm.swap_out(s), lambda: ref.swap_out(s))
            if r:
                assert [tuple(x) for x in r[0].tolist()] == r[1]
        elif op == "swap_in" and ref.swapped:
            s = sorted(ref.swapped)[rng.integers(len(ref.swapped))]
            r = run_both(bm, ref, lambda: bm.swap_in(s), lambda: ref.swap_in(s))
            if r:
                assert [tuple(x) for x in r[0].tolist()] == r[1]
        elif op == "bad" and resident:
            s = resident[0]
            run_both(bm, ref, lambda: bm.append_slots([s, s]), lambda: ref.append_slots([s, s]))
            run_both(bm, ref, lambda: bm.fork(s, s), lambda: ref.fork(s, s))
        snapshot(bm, ref, ids)
    assert done > 10


def test_plan_decode_checks_width_before_changing_anything(BM):
    bm = BM.BlockManager(8, 4)
    bm.add_sequence(0, 4)                                   # one full block: the next token needs a new one
    with pytest.raises(Exception) as e:
        bm.plan_decode([0], max_blocks=1)
    assert "INVALID_ARGUMENT" in str(e.value)
    assert bm.sequence_info(0) == (4, 1, False) and bm.num_free_blocks() == (7, 0)
    s, p, t, l = bm.plan_decode([0], max_blocks=2, pad=-1)
    assert s.tolist() == [4 * 1 + 0] and t.tolist() == [[0, 1]] and l.tolist() == [5] and len(p) == 0


def test_plan_decode_output_buffers_are_checked(BM):
    """The manager writes the plan through raw host pointers: caller buffers that are too small, of the
    wrong dtype, strided or on a device are refused before the call, and nothing changes."""
    import torch
    bm = BM.BlockManager(16, 4)
    bm.add_sequence(0, 3)
    bm.add_sequence(1, 5)
    good = (torch.empty(2, dtype=torch.int64), torch.empty((2, 2), dtype=torch.int64),
            torch.empty((2, 3), dtype=torch.int32), torch.empty(2, dtype=torch.int32))
    bad = [
        (torch.empty(1, dtype=torch.int64),) + good[1:],                                  # slots too small
        good[:2] + (torch.empty((2, 3), dtype=torch.int64),) + good[3:],                  # tables int64
        good[:2] + (torch.empty((3, 2), dtype=torch.int32).t(),) + good[3:],             # strided
        good[:3] + (np.empty(2, np.int64),),                                              # lens int64
        good[:1] + (torch.empty((2, 2), dtype=torch.int64, device="meta"),) + good[2:],  # not host memory
    ]
    for out in bad:
        with pytest.raises(ValueError):
            bm.plan_decode([0, 1], 3, 0, out)
        assert bm.sequence_info(0) == (3, 1, False) and bm.sequence_info(1) == (5, 2, False)
    s, p, t, l = bm.plan_decode([0, 1], 3, -1, good)
    assert s.tolist() == [3, 4 * 2 + 1] and l.tolist() == [4, 6] and t.tolist() == [[0, -1, -1], [1, 2, -1]]
    assert len(p) == 0


def test_out_of_blocks_is_all_or_nothing(BM):
    bm = BM.BlockManager(3, 2)
    bm.add_sequence(0, 2)
    bm.add_sequence(1, 2)
    bm.add_sequence(2, 1)                                   # pool now full; 2 has room in its block
    with pytest.raises(BM.OutOfBlocks):
        bm.append_slots([2, 0])                             # 0 needs a block: whole call refused
    assert bm.sequence_info(2)[0] == 1
    assert bm.append_slots([2])[0].tolist() == [2 * 2 + 1]
