"""Oracle of the host block manager -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU baseline may import this module; the product
path never does.

A plain dictionary-and-list model of the paging scheme the pages describe, with one fixed allocation
policy so that two implementations of it can be compared decision by decision:

* A pool of num_blocks physical blocks is created up front (tutorial page, sec. 3.2 "关键性能优化",
  block preallocation). Free blocks sit on a stack: it starts as 0, 1, 2, ... from the top, and a
  released block goes back on top (last released, first reused).
* Each sequence owns a block table mapping logical block i to a physical block (tutorial sec. 2.1
  "基本数据结构设计"; page "vLLM的诞生背景", section "PagedAttention的破局思路"). Blocks are taken only
  when a token needs one (on-demand allocation, same section).
* Sharing is by reference count (tutorial sec. 2.3 "显存共享机制"): fork() gives a child every block of
  its parent (beam search, sharing within a request); add_sequence() with a prefix shares the
  parent's FULL blocks covering the common prefix (sharing between requests), since sharing only
  works at page-aligned boundaries (page "PagedAttention 与连续批处理", section "对 agent 开发者的启示").
* Writing a token into a block whose count is above one first copies that block to a fresh one
  (copy-on-write, page "vLLM的诞生背景", section "PagedAttention的局限性"); the (old, new) pair is what
  the device's copy_blocks consumes.
* free() releases a finished sequence's blocks (page "PagedAttention 与连续批处理", section
  "连续批处理": a finished request's pages are released); a block returns to the free stack when its
  count reaches zero.
* swap_out()/swap_in() move a sequence's blocks to a host pool and back (same page, section
  "PagedAttention：把显存做成虚拟内存": pages of inactive sequences go to CPU memory). Reading taken:
  each block of the swapped sequence gets its own host block; a block still shared by a resident
  sequence stays on the device for it (its count drops by one). After swap_in the sequence holds
  private blocks.

Every operation either succeeds completely or raises and leaves the state unchanged.
"""


class OracleBlockError(Exception):
    pass


class OutOfBlocks(OracleBlockError):
    pass


class BlockManagerOracle:
    def __init__(self, num_blocks, block_size, num_host_blocks=0):
        if num_blocks <= 0 or block_size <= 0 or num_host_blocks < 0:
            raise OracleBlockError("bad sizes")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = list(range(num_blocks - 1, -1, -1))          # top of the stack is the end
        self.host_free = list(range(num_host_blocks - 1, -1, -1))
        self.ref = [0] * num_blocks
        self.tables = {}                                         # seq -> list of device blocks
        self.lens = {}                                           # seq -> tokens stored
        self.swapped = {}                                        # seq -> list of host blocks

    # --- helpers -------------------------------------------------------------------------------
    def _take(self):
        b = self.free.pop()
        assert self.ref[b] == 0
        self.ref[b] = 1
        return b

    def _release(self, b):
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free.append(b)

    def _blocks_for(self, tokens):
        return -(-tokens // self.block_size)

    def _known(self, seq):
        return seq in self.tables or seq in self.swapped

    # --- operations ----------------------------------------------------------------------------
    def add_sequence(self, seq, num_tokens, prefix_seq=-1, prefix_tokens=0):
        """A new sequence holding num_tokens prompt tokens. Returns the slots of the tokens that must
        be written (those not inside shared blocks), in token order."""
        if self._known(seq) or num_tokens < 0 or prefix_tokens < 0 or prefix_tokens > num_tokens:
            raise OracleBlockError("bad add_sequence")
        shared = []
        if prefix_seq != -1:
            if prefix_seq not in self.tables:
                raise OracleBlockError("prefix sequence not resident")
            common = min(prefix_tokens, self.lens[prefix_seq])
            shared = self.tables[prefix_seq][:common // self.block_size]
        need = self._blocks_for(num_tokens) - len(shared)
        if need > len(self.free):
            raise OutOfBlocks("pool exhausted")
        for b in shared:
            self.ref[b] += 1
        table = list(shared) + [self._take() for _ in range(need)]
        self.tables[seq] = table
        self.lens[seq] = num_tokens
        bs = self.block_size
        return [table[t // bs] * bs + t % bs for t in range(len(shared) * bs, num_tokens)]

    def fork(self, parent, child):
        """The child shares every block of the parent (reference counts up by one)."""
        if parent not in self.tables or self._known(child):
            raise OracleBlockError("bad fork")
        for b in self.tables[parent]:
            self.ref[b] += 1
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]

    def append_slots(self, seqs):
        """One new token for each sequence, in the given order. Returns (slots, cow_pairs)."""
        if len(set(seqs)) != len(seqs) or any(s not in self.tables for s in seqs):
            raise OracleBlockError("bad append")
        bs = self.block_size
        need = 0
        for s in seqs:
            L = self.lens[s]
            if L % bs == 0 or self.ref[self.tables[s][L // bs]] > 1:
                need += 1
        if need > len(self.free):
            raise OutOfBlocks("pool exhausted")
        slots, pairs = [], []
        for s in seqs:
            table, L = self.tables[s], self.lens[s]
            if L % bs == 0:
                table.append(self._take())
            else:
                last = table[L // bs]
                if self.ref[last] > 1:
                    new = self._take()
                    pairs.append((last, new))
                    self._release(last)
                    table[L // bs] = new
            slots.append(table[L // bs] * bs + L % bs)
            self.lens[s] = L + 1
        return slots, pairs

    def free_sequence(self, seq):
        if seq in self.tables:
            for b in self.tables.pop(seq):
                self._release(b)
        elif seq in self.swapped:
            self.host_free.extend(self.swapped.pop(seq))
        else:
            raise OracleBlockError("unknown sequence")
        del self.lens[seq]

    def swap_out(self, seq):
        """Returns the (device block, host block) pairs to copy, in table order."""
        if seq not in self.tables:
            raise OracleBlockError("not resident")
        table = self.tables[seq]
        if len(table) > len(self.host_free):
            raise OutOfBlocks("host pool exhausted")
        host = [self.host_free.pop() for _ in table]
        pairs = list(zip(table, host))
        for b in table:
            self._release(b)
        del self.tables[seq]
        self.swapped[seq] = host
        return pairs

    def swap_in(self, seq):
        """Returns the (host block, device block) pairs to copy, in table order."""
        if seq not in self.swapped:
            raise OracleBlockError("not swapped")
        host = self.swapped[seq]
        if len(host) > len(self.free):
            raise OutOfBlocks("pool exhausted")
        table = [self._take() for _ in host]
        pairs = list(zip(host, table))
        self.host_free.extend(host)
        del self.swapped[seq]
        self.tables[seq] = table
        return pairs

    def block_tables(self, seqs, max_blocks, pad=0):
        rows, lens = [], []
        for s in seqs:
            if s not in self.tables:
                raise OracleBlockError("not resident")
            t = self.tables[s]
            if len(t) > max_blocks:
                raise OracleBlockError("table wider than max_blocks")
            rows.append(t + [pad] * (max_blocks - len(t)))
            lens.append(self.lens[s])
        return rows, lens

    def num_free_blocks(self):
        return len(self.free)

    def num_free_host_blocks(self):
        return len(self.host_free)
