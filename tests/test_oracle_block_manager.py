"""Pins for the block-manager oracle (CPU only).

* A worked scenario, decided by hand from the pages' rules (on-demand blocks, reference-counted
  sharing, copy-on-write, release at zero, page-aligned prefix sharing), with every slot, pair and
  table written out.
* Content semantics by brute force: a simulated physical pool receives every token through the
  returned slots, every copy-on-write pair as a whole-block copy, and every swap as block moves
  between a device and a host pool. After each operation every resident sequence, read through its
  block table, must hold exactly its own token history, which the test tracks independently.
* Bookkeeping invariants after each operation: a block's count equals the number of table entries
  naming it; the free stack holds exactly the blocks with count zero, once each; a table has
  ceil(len / block_size) entries; host blocks are either free or held by one swapped sequence.
* Failed operations leave the state unchanged.
* Planted mistakes (a skipped copy-on-write, a count that never drops, prefix sharing of a partial
  block, a swap that forgets to release) are each caught by the checks above.
"""
import copy

import numpy as np
import pytest

from oracle.block_manager import BlockManagerOracle, OracleBlockError, OutOfBlocks


def test_worked_scenario():
    bm = BlockManagerOracle(num_blocks=8, block_size=4, num_host_blocks=4)
    # A: 6-token prompt -> blocks 0, 1 (the stack pops 0 first); every token written.
    assert bm.add_sequence("A", 6) == [0, 1, 2, 3, 4, 5]
    assert bm.tables["A"] == [0, 1] and bm.num_free_blocks() == 6
    # B forks A: shares both blocks.
    bm.fork("A", "B")
    assert bm.ref[:2] == [2, 2]
    # Both append. A writes into shared block 1 -> copy-on-write into block 2; B then holds block 1
    # alone and writes in place.
    slots, pairs = bm.append_slots(["A", "B"])
    assert pairs == [(1, 2)] and slots == [2 * 4 + 2, 1 * 4 + 2]
    assert bm.tables == {"A": [0, 2], "B": [0, 1]} and bm.ref[:3] == [2, 1, 1]
    # C shares A's prompt prefix of 7 tokens: only the first FULL block (tokens 0..3) is shared;
    # tokens 4..8 of its 9-token prompt go to fresh blocks 3 and 4.
    assert bm.add_sequence("C", 9, prefix_seq="A", prefix_tokens=7) == [12, 13, 14, 15, 16]
    assert bm.tables["C"] == [0, 3, 4] and bm.ref[0] == 3
    # A's 8th token fills block 2; its 9th needs a new block (5).
    assert bm.append_slots(["A"]) == ([11], [])
    assert bm.append_slots(["A"]) == ([20], [])
    assert bm.tables["A"] == [0, 2, 5]
    # Free B: block 1 returns to the free stack (count 0), block 0 keeps count 2.
    bm.free_sequence("B")
    assert bm.free[-1] == 1 and bm.ref[0] == 2
    # Swap C out: host blocks 0, 1, 2 in table order; device 3, 4 are freed, 0 stays for A.
    assert bm.swap_out("C") == [(0, 0), (3, 1), (4, 2)]
    assert bm.ref[0] == 1 and bm.free[-2:] == [3, 4]
    # Swap C back in: it gets the top of the stack (4, 3, then 1), all private.
    assert bm.swap_in("C") == [(0, 4), (1, 3), (2, 1)]
    assert bm.tables["C"] == [4, 3, 1] and bm.num_free_host_blocks() == 4
    rows, lens = bm.block_tables(["A", "C"], max_blocks=4, pad=-1)
    assert rows == [[0, 2, 5, -1], [4, 3, 1, -1]] and lens == [9, 9]


class World:
    """Independent ground truth: token histories and a simulated device + host memory."""

    def __init__(self, bm):
        self.bm = bm
        self.mem = np.full(bm.num_blocks * bm.block_size, -1, np.int64)
        self.host = np.full(max(len(bm.host_free), 1) * bm.block_size, -1, np.int64)
        self.hist = {}
        self.next_token = 0

    def new_tokens(self, n):
        t = list(range(self.next_token, self.next_token + n))
        self.next_token += n
        return t

    def copy_block(self, dst_mem, dst, src_mem, src):
        bs = self.bm.block_size
        dst_mem[dst * bs:(dst + 1) * bs] = src_mem[src * bs:(src + 1) * bs]

    def add(self, seq, n, prefix=-1, prefix_tokens=0):
        if prefix != -1:
            common = min(prefix_tokens, len(self.hist[prefix]))
            shared = common // self.bm.block_size * self.bm.block_size
            toks = self.hist[prefix][:shared] + self.new_tokens(n - shared)
        else:
            toks = self.new_tokens(n)
        slots = self.bm.add_sequence(seq, n, prefix, prefix_tokens)
        first = n - len(slots)
        for t, s in zip(toks[first:], slots):
            self.mem[s] = t
        self.hist[seq] = toks

    def fork(self, parent, child):
        self.bm.fork(parent, child)
        self.hist[child] = list(self.hist[parent])

    def append(self, seqs):
        slots, pairs = self.bm.append_slots(seqs)
        for src, dst in pairs:                     # copies first, then the new tokens
            self.copy_block(self.mem, dst, self.mem, src)
        for s, slot in zip(seqs, slots):
            t = self.new_tokens(1)[0]
            self.mem[slot] = t
            self.hist[s].append(t)

    def free(self, seq):
        self.bm.free_sequence(seq)
        del self.hist[seq]

    def swap_out(self, seq):
        for dev, host in self.bm.swap_out(seq):
            self.copy_block(self.host, host, self.mem, dev)

    def swap_in(self, seq):
        for host, dev in self.bm.swap_in(seq):
            self.copy_block(self.mem, dev, self.host, host)

    def check(self):
        bm, bs = self.bm, self.bm.block_size
        for seq, table in bm.tables.items():
            L = bm.lens[seq]
            assert len(table) == -(-L // bs)
            got = [int(self.mem[table[t // bs] * bs + t % bs]) for t in range(L)]
            assert got == self.hist[seq], f"sequence {seq} reads wrong tokens"
        for seq, host in bm.swapped.items():
            L = bm.lens[seq]
            got = [int(self.host[host[t // bs] * bs + t % bs]) for t in range(L)]
            assert got == self.hist[seq], f"swapped sequence {seq} lost tokens"
        counts = [0] * bm.num_blocks
        for table in bm.tables.values():
            for b in table:
                counts[b] += 1
        assert counts == bm.ref
        assert sorted(bm.free) == [b for b in range(bm.num_blocks) if counts[b] == 0]
        held = [h for host in bm.swapped.values() for h in host]
        assert len(held) == len(set(held)) and not set(held) & set(bm.host_free)
        assert len(set(bm.host_free)) == len(bm.host_free)


def random_session(bm, seed, steps=300):
    rng = np.random.default_rng(seed)
    w = World(bm)
    next_id = 0
    for _ in range(steps):
        resident = list(bm.tables)
        op = rng.choice(["add", "prefix", "fork", "append", "append", "append", "free", "swap_out", "swap_in"])
        before = copy.deepcopy(bm.__dict__)
        try:
            if op == "add":
                w.add(next_id, int(rng.integers(0, 3 * bm.block_size)))
                next_id += 1
            elif op == "prefix" and resident:
                p = resident[rng.integers(len(resident))]
                n = int(rng.integers(0, 3 * bm.block_size))
                w.add(next_id, n, p, int(rng.integers(0, n + 1)))
                next_id += 1
            elif op == "fork" and resident:
                w.fork(resident[rng.integers(len(resident))], next_id)
                next_id += 1
            elif op == "append" and resident:
                k = int(rng.integers(1, len(resident) + 1))
                w.append([resident[i] for i in rng.permutation(len(resident))[:k]])
            elif op == "free" and (resident or bm.swapped):
                pool = resident + list(bm.swapped)
                w.free(pool[rng.integers(len(pool))])
            elif op == "swap_out" and resident:
                w.swap_out(resident[rng.integers(len(resident))])
            elif op == "swap_in" and bm.swapped:
                sw = list(bm.swapped)
                w.swap_in(sw[rng.integers(len(sw))])
        except OutOfBlocks:
            assert bm.__dict__ == before, f"{op} changed the state before failing"
        w.check()
    return w


@pytest.mark.parametrize("seed", range(6))
def test_random_sessions_keep_contents_and_counts(seed):
    bm = BlockManagerOracle(num_blocks=24, block_size=4, num_host_blocks=12)
    w = random_session(bm, seed)
    assert w.next_token > 100                         # the session did real work


def test_argument_errors():
    bm = BlockManagerOracle(4, 4)
    bm.add_sequence(0, 3)
    with pytest.raises(OracleBlockError):
        bm.add_sequence(0, 1)                         # duplicate id
    with pytest.raises(OracleBlockError):
        bm.append_slots([0, 0])                       # one token per sequence per call
    with pytest.raises(OracleBlockError):
        bm.fork(7, 8)                                 # unknown parent
    with pytest.raises(OracleBlockError):
        bm.swap_out(0)                                # no host pool at all -> OutOfBlocks
    with pytest.raises(OracleBlockError):
        bm.block_tables([0], max_blocks=0)


# --- planted mistakes ------------------------------------------------------------------------------
class NoCopyOnWrite(BlockManagerOracle):
    def append_slots(self, seqs):
        saved = self.ref
        self.ref = [min(r, 1) for r in saved]         # pretends nothing is shared
        try:
            out = BlockManagerOracle.append_slots(self, seqs)
        finally:
            fresh = self.ref
            self.ref = [max(a, b) if a else 0 for a, b in zip(saved, fresh)]
        return out


class NeverRelease(BlockManagerOracle):
    def _release(self, b):
        pass


class SharesPartialBlocks(BlockManagerOracle):
    def _blocks_for(self, tokens):
        return -(-tokens // self.block_size)

    def add_sequence(self, seq, num_tokens, prefix_seq=-1, prefix_tokens=0):
        if prefix_seq != -1 and prefix_seq in self.tables:
            prefix_tokens = min(num_tokens, -(-prefix_tokens // self.block_size) * self.block_size)
        return BlockManagerOracle.add_sequence(self, seq, num_tokens, prefix_seq, prefix_tokens)


class SwapForgetsRelease(BlockManagerOracle):
    def swap_out(self, seq):
        table = list(self.tables[seq])
        pairs = BlockManagerOracle.swap_out(self, seq)
        for b in table:                               # undo the release
            if self.ref[b] == 0:
                self.free.remove(b)
            self.ref[b] += 1
        return pairs


@pytest.mark.parametrize("mutant", [NoCopyOnWrite, NeverRelease, SharesPartialBlocks, SwapForgetsRelease])
def test_planted_mistakes_are_caught(mutant):
    caught = False
    for seed in range(6):
        try:
            random_session(mutant(num_blocks=24, block_size=4, num_host_blocks=12), seed)
        except (AssertionError, OracleBlockError, IndexError, ValueError):
            caught = True
            break
    assert caught, f"{mutant.__name__} went unnoticed"
