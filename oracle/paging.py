"""Block allocation semantics of the paged cache -- TEST INFRASTRUCTURE ONLY.

A plain restatement, in Python, of what the pages say a paged KV cache does
with its blocks, with the documented deterministic policies of the library's
block manager so the two can be compared exactly:

* "KV Cache 深度解析" §三: fixed 16-token blocks, a per-sequence block table,
  blocks allocated on demand (at most one partly used block per sequence),
  physical blocks shared by several sequences (beam branches, common prefixes);
* "大模型推理为何这么慢" (PagedAttention section): blocks are allocated when a
  request needs more space and released as soon as it finishes;
* "llm-inference-optimization" notes §二 (``PagedKVCache.append_token``): a
  sequence takes a new block when it has none or its last one is full, and
  the token goes to the next offset of the last block.

Sharing is by reference count; writing into a shared block that still has
free slots first moves the writer to a private copy (copy-on-write).
Policies: free blocks are a LIFO stack that initially yields 0, 1, 2, ...;
a new sequence gets the lowest unused id.
"""
from __future__ import annotations

BLOCK = 16
POISON = 2**31 - 1


class ToyBlockManager:
    def __init__(self, num_blocks: int, max_seqs: int, max_blocks_per_seq: int):
        self.free = list(range(num_blocks - 1, -1, -1))   # pop() yields 0, 1, 2, ...
        self.ref = [0] * num_blocks
        self.max_seqs, self.max_blocks = max_seqs, max_blocks_per_seq
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}

    def _alloc(self) -> int:
        b = self.free.pop()
        self.ref[b] = 1
        return b

    def _release(self, b: int) -> None:
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free.append(b)

    def add_sequence(self) -> int:
        s = next(i for i in range(self.max_seqs) if i not in self.tables)
        self.tables[s], self.lens[s] = [], 0
        return s

    def fork(self, parent: int) -> int:
        c = self.add_sequence()
        self.tables[c] = list(self.tables[parent])
        self.lens[c] = self.lens[parent]
        for b in self.tables[c]:
            self.ref[b] += 1
        return c

    def free_sequence(self, s: int) -> None:
        for b in reversed(self.tables.pop(s)):
            self._release(b)
        del self.lens[s]

    def append_token(self, s: int):
        """Slot for sequence s's next token, and the copy (src, dst) it needs, if any."""
        table, pos, copy = self.tables[s], self.lens[s], None
        if pos % BLOCK == 0:
            table.append(self._alloc())
        elif self.ref[table[-1]] > 1:
            fresh = self._alloc()
            copy = (table[-1], fresh)
            self._release(table[-1])
            table[-1] = fresh
        self.lens[s] = pos + 1
        return table[pos // BLOCK] * BLOCK + pos % BLOCK, copy

    def blocks_needed(self, seq_ids) -> int:
        """Blocks a batch of appends would take (new blocks and copies)."""
        lens, fresh, need = dict(self.lens), set(), 0
        for s in seq_ids:
            pos = lens[s]
            lens[s] += 1
            if pos % BLOCK == 0:
                need += 1
                fresh.add(s)
            elif s not in fresh and self.ref[self.tables[s][-1]] > 1:
                need += 1
                fresh.add(s)
        return need

    def export(self):
        table = [[POISON] * self.max_blocks for _ in range(self.max_seqs)]
        lens = [0] * self.max_seqs
        for s, t in self.tables.items():
            table[s][:len(t)] = t
            lens[s] = self.lens[s]
        return table, lens
