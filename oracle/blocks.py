"""Block-manager oracle — TEST INFRASTRUCTURE ONLY.

A plain, sequential restatement of the paged KV cache's block bookkeeping, in
the order the pages describe it:

  * one pool of equal blocks, carved once; the blocks not in use form a free
    pool from which a new block is taken ("从源码剖析 vLLM 的显存管理与连续批处理",
    §2.1 BlockTable.append_token, §2.2 the KV-cache pool);
  * a sequence takes a new physical block when its next token starts a new
    logical block, and its block table maps the logical block to it (§2.1);
  * a block carries a reference count; requests with a common prefix point at
    the same physical blocks and the count goes up; a write into a shared block
    first copies it (copy-on-write); a block whose count drops to zero returns
    to the free pool ("vLLM框架解析：PagedAttention技术如何实现LLM推理20倍加速",
    §2.2 the Block structure with ref_count, §2.3 block sharing steps 1-3, and
    the §3.1 flow chart: shared block -> count up, otherwise a new block);
  * requests are admitted in order while blocks remain, and admission stops at
    the first request that does not fit (§3.2 of the first page: schedule()
    with block_manager.can_allocate, "else: break").

Readings where the pages leave a step open (each is the plainest one):
  * the free pool is first in, first out: a block freed earlier is reused
    earlier (the flow chart puts new blocks on an LRU queue);
  * one step appends num_new_tokens[s] tokens to every sequence s, in index
    order; within a sequence the copy-on-write block is taken before the new
    ones, and new blocks in logical order;
  * a sequence whose first new token falls inside its last, partly filled
    block writes into that block; if the block's count is above one it is
    first replaced by a private copy (count of the old block down by one);
  * the step's slots are packed in sequence order (offsets = running sum of
    num_new_tokens); a sequence that is not served gets slot -1 for each of
    its tokens, no new block and no length change;
  * a fork makes a child share the first `length` tokens of its parent: the
    child's table takes the parent's first ceil(length / B) block ids, each of
    whose counts goes up by one, and its length becomes `length`; the child
    must hold no tokens and differ from the parent (else ERR_REF_COUNT), and
    0 <= length <= the parent's length (else ERR_CONTEXT_LEN);
  * a negative token count is ERR_CONTEXT_LEN (the sequence is skipped);
  * freeing a sequence lowers the count of each of its blocks in logical
    order; a block reaching zero joins the free pool at that moment; the
    sequence's row is cleared (-1) and its length set to 0.

Plain Python loops over small pools; it shares nothing with the CUDA library
and imports neither it nor the other oracle module.  Only tests/, the smoke
check and bench.py's CPU baseline use it.
"""

from __future__ import annotations

from collections import deque

import numpy as np

# Error flags of a step (same meaning as the library's device error bits).
ERR_CONTEXT_LEN = 2      # a sequence would exceed its block-table row, or a bad length
ERR_NO_FREE_BLOCK = 32   # the free pool ran out; that sequence and every later one were not served
ERR_REF_COUNT = 64       # a count would drop below zero, or a fork into a sequence that holds blocks


class BlockManager:
    """Reference counts, free pool, block tables and lengths of one pool."""

    def __init__(self, num_blocks: int, num_seqs: int, max_blocks_per_seq: int, block_size: int):
        self.N, self.B = int(num_blocks), int(block_size)
        self.ref = np.zeros(self.N, dtype=np.int64)
        self.free = deque(range(self.N))               # head = next block handed out
        self.freed_total = 0                           # blocks returned so far (the ring's tail position - N)
        self.taken_total = 0                           # blocks handed out so far (the ring's head position)
        self.tables = np.full((num_seqs, max_blocks_per_seq), -1, dtype=np.int64)
        self.lens = np.zeros(num_seqs, dtype=np.int64)

    # ---- helpers
    def blocks_of(self, length: int) -> int:
        return (int(length) + self.B - 1) // self.B

    def _take(self) -> int:
        b = self.free.popleft()
        self.taken_total += 1
        self.ref[b] = 1
        return b

    def _give_back(self, b: int):
        self.free.append(int(b))
        self.freed_total += 1

    # ---- operations
    def append(self, num_new_tokens):
        """One step: every sequence s takes num_new_tokens[s] new token slots.
        Returns (slots [sum n], copy pairs [S][2] (old, new) or (-1, -1),
        error flags)."""
        n_new = [int(x) for x in num_new_tokens]
        S = len(n_new)
        slots = np.full(sum(max(0, n) for n in n_new), -1, dtype=np.int64)
        pairs = np.full((S, 2), -1, dtype=np.int64)
        err = 0
        offset = 0
        stopped = False
        for s in range(S):
            n = n_new[s]
            base = offset
            offset += max(0, n)
            if n < 0:
                err |= ERR_CONTEXT_LEN
                continue
            if n == 0 or stopped:
                continue
            L = int(self.lens[s])
            if L + n > self.tables.shape[1] * self.B:
                err |= ERR_CONTEXT_LEN
                continue
            first_new_block = self.blocks_of(L)
            new_blocks = self.blocks_of(L + n) - first_new_block
            cow = L % self.B != 0 and self.ref[self.tables[s, L // self.B]] > 1
            if new_blocks + (1 if cow else 0) > len(self.free):
                err |= ERR_NO_FREE_BLOCK
                stopped = True            # admission stops here: later sequences wait too
                continue
            if cow:
                old = int(self.tables[s, L // self.B])
                copy = self._take()
                self.ref[old] -= 1
                self.tables[s, L // self.B] = copy
                pairs[s] = (old, copy)
            for j in range(first_new_block, first_new_block + new_blocks):
                self.tables[s, j] = self._take()
            for i in range(n):
                pos = L + i
                slots[base + i] = self.tables[s, pos // self.B] * self.B + pos % self.B
            self.lens[s] = L + n
        return slots, pairs, err

    def fork(self, pairs):
        """pairs: (parent, child, length) in order; the child shares the
        parent's first `length` tokens."""
        err = 0
        for parent, child, length in pairs:
            parent, child, length = int(parent), int(child), int(length)
            if child == parent or self.lens[child] != 0:   # the child's own blocks would be lost
                err |= ERR_REF_COUNT
                continue
            if not 0 <= length <= self.lens[parent]:
                err |= ERR_CONTEXT_LEN
                continue
            for j in range(self.blocks_of(length)):
                b = int(self.tables[parent, j])
                self.tables[child, j] = b
                self.ref[b] += 1
            self.lens[child] = length
        return err

    def release(self, seqs):
        """Free whole sequences, in the given order."""
        err = 0
        for s in seqs:
            s = int(s)
            for j in range(self.blocks_of(self.lens[s])):
                b = int(self.tables[s, j])
                if self.ref[b] <= 0:
                    err |= ERR_REF_COUNT
                else:
                    self.ref[b] -= 1
                    if self.ref[b] == 0:
                        self._give_back(b)
                self.tables[s, j] = -1
            self.lens[s] = 0
        return err

    # ---- the state in the library's array form
    def ring(self):
        """(free_ids [N], head, tail): the free pool as a ring of N entries whose
        live part is positions head .. tail-1 (mod N), oldest first."""
        head = self.taken_total
        tail = self.N + self.freed_total
        ids = np.full(self.N, -1, dtype=np.int64)
        for k, b in enumerate(self.free):
            ids[(head + k) % self.N] = b
        return ids, head, tail
