"""Pins of the block-manager oracle (oracle/blocks.py), CPU only:

  * a hand-worked golden run (tests/golden/block_manager.json): appends that
    take new blocks, forks that share them, a copy-on-write, frees that return
    blocks to the pool first in first out, a step that runs out of blocks and
    one that overflows a table row, with the expected slots, copy pairs,
    counts, tables, lengths and free pool after every operation;
  * invariants over seeded random runs: every count equals the number of
    table entries naming the block, the free pool holds exactly the blocks of
    count zero, once each, every block a step writes into is held by that
    sequence alone, and admission stops at the first sequence that does not
    fit;
  * attention is unchanged by sharing and copy-on-write: after a fork and a
    step that copies the shared partial block (copy done with the attention
    oracle's own block copy), the parent's decode output is bit-identical and
    the child's logical K/V is the parent's prefix plus its new tokens;
  * planted mistakes in a copy of the oracle's source each fail one of the
    above."""

import json
import os
import types

import numpy as np
import pytest
import torch

import oracle
import oracle.blocks as blocks
import workloads

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden", "block_manager.json")


def replay_golden(mod):
    g = json.load(open(GOLDEN))
    m = mod.BlockManager(g["num_blocks"], g["num_seqs"], g["max_blocks_per_seq"], g["block_size"])
    for k, op in enumerate(g["ops"]):
        if op["op"] == "append":
            slots, pairs, err = m.append(op["n"])
            assert slots.tolist() == op["slots"], (k, op)
            assert pairs.tolist() == op["pairs"], (k, op)
        elif op["op"] == "fork":
            err = m.fork(op["pairs"])
        else:
            err = m.release(op["seqs"])
        assert err == op["err"], (k, op)
        st = op["state"]
        assert m.ref.tolist() == st["ref"], (k, "ref")
        assert m.lens.tolist() == st["lens"], (k, "lens")
        assert m.tables.tolist() == st["tables"], (k, "tables")
        assert list(m.free) == st["free"], (k, "free")
        ring, head, tail = m.ring()
        assert (head, tail) == (st["head"], st["tail"]), (k, "head/tail")
        if "ring" in st:
            assert ring.tolist() == st["ring"], (k, "ring")


def test_golden_run():
    replay_golden(blocks)


def check_invariants(m):
    counts = np.zeros(m.N, dtype=np.int64)
    for s in range(m.tables.shape[0]):
        n = m.blocks_of(m.lens[s])
        row = m.tables[s]
        assert np.all(row[n:] == -1)
        assert np.all((row[:n] >= 0) & (row[:n] < m.N))
        np.add.at(counts, row[:n], 1)
    assert np.array_equal(counts, m.ref)
    free = list(m.free)
    assert len(set(free)) == len(free)
    assert set(free) == set(np.nonzero(m.ref == 0)[0].tolist())
    ring, head, tail = m.ring()
    assert tail - head == len(free)
    assert [ring[(head + k) % m.N] for k in range(len(free))] == free


def random_run(mod, seed, steps=150, num_blocks=40, num_seqs=8, max_blocks=8, block_size=4):
    """Seeded random appends, forks and frees; invariants checked after each."""
    rng = np.random.default_rng(seed)
    m = mod.BlockManager(num_blocks, num_seqs, max_blocks, block_size)
    for _ in range(steps):
        r = rng.random()
        active = np.nonzero(m.lens > 0)[0]
        empty = np.nonzero(m.lens == 0)[0]
        if r < 0.6:
            n = rng.integers(0, 7, size=num_seqs)
            n[rng.random(num_seqs) < 0.3] = 0
            before = m.lens.copy()
            slots, pairs, err = m.append(n)
            served = m.lens != before
            offs = np.concatenate([[0], np.cumsum(n)])
            for s in range(num_seqs):
                mine = slots[offs[s]:offs[s + 1]]
                if served[s]:
                    assert np.all(mine >= 0)
                    assert np.all(m.ref[mine // block_size] == 1)          # written blocks are private
                    assert set((mine // block_size).tolist()) <= set(m.tables[s].tolist())
                else:
                    assert np.all(mine == -1)
            if err & mod.ERR_NO_FREE_BLOCK:
                first = min(s for s in range(num_seqs) if n[s] > 0 and not served[s]
                            and before[s] + n[s] <= max_blocks * block_size)
                assert not np.any(served[first:])                          # admission stopped there
        elif r < 0.8 and len(active) and len(empty):
            parent = int(rng.choice(active))
            child = int(rng.choice(empty))
            m.fork([(parent, child, int(rng.integers(0, m.lens[parent] + 1)))])
        elif len(active):
            m.release(rng.choice(active, size=min(len(active), int(rng.integers(1, 3))), replace=False))
        check_invariants(m)
    return m


@pytest.mark.parametrize("seed", range(6))
def test_invariants_over_random_runs(seed):
    random_run(blocks, seed)


def test_sharing_and_copy_on_write_leave_attention_unchanged():
    """A parent with a partly filled last block forks a child; both append a
    token; the parent's block is copied for the writer that goes first (the
    parent, index 0) and the child keeps the original.  With the copy applied
    and the new rows written, the attention of every sequence over its old
    tokens is bit-identical to what it was before the step, and each
    sequence's new row sits right after its own prefix."""
    orc = oracle.default()
    B, Hkv, D = 16, 2, 64
    N, rows = 24, 3
    m = blocks.BlockManager(N, rows, 6, B)
    slots0, _, _ = m.append([37, 0, 0])                 # parent: 37 tokens, 3 blocks, last one holds 5
    assert m.fork([(0, 1, 37), (0, 2, 32)]) == 0        # children share 3 and 2 (full) blocks
    pool = workloads.random_small(seed=5, dtype=torch.float16, lens=(1,), num_q_heads=4, num_kv_heads=Hkv,
                                  head_dim=D, block_size=B, extra_blocks=N - 1)
    k, v = pool.k_cache.clone(), pool.v_cache.clone()
    gen = torch.Generator().manual_seed(9)
    rows37 = torch.randn((37, Hkv, D), generator=gen).to(torch.float16)
    orc.reshape_and_cache(rows37, rows37 + 1, k, v, torch.from_numpy(slots0), B)
    q = torch.randn((rows, 4, D), generator=gen).to(torch.float16)

    def decode(mgr, kk, vv):
        return orc.decode(q, kk, vv, torch.from_numpy(mgr.tables.astype(np.int32)),
                          torch.from_numpy(mgr.lens.astype(np.int32)), 0.125, B, Hkv)

    before = decode(m, k, v)
    slots, pairs, err = m.append([1, 1, 1])
    assert err == 0
    assert pairs[0].tolist() != [-1, -1] and pairs[1].tolist() == [-1, -1]   # parent copies, child 1 keeps
    assert pairs[2].tolist() == [-1, -1]                                      # child 2 starts a new block
    live = pairs[pairs[:, 0] >= 0]
    orc.copy_blocks(k, v, k, v, torch.from_numpy(live), B)
    new = torch.randn((3, Hkv, D), generator=gen).to(torch.float16)
    orc.reshape_and_cache(new, new - 1, k, v, torch.from_numpy(slots), B)
    check_invariants(m)
    # the parent without its new token: the same attention as before the step
    m_prev = types.SimpleNamespace(tables=m.tables, lens=m.lens - np.array([1, 1, 1]))
    again = decode(m_prev, k, v)
    assert np.array_equal(again, before)
    # the child's logical K is the parent's first 37 rows, then its own new row
    kc = orc.pool_index

    def logical_row(mgr, s, t):
        blk = int(mgr.tables[s, t // B])
        return k.view(-1)[[kc(blk, 0, t % B, d, Hkv, B, D, torch.float16) for d in range(D)]]

    for t in (0, 17, 36):
        assert torch.equal(logical_row(m, 1, t), rows37[t, 0])
    assert torch.equal(logical_row(m, 1, 37), new[1, 0])
    assert torch.equal(logical_row(m, 0, 37), new[0, 0])
    assert torch.equal(logical_row(m, 2, 32), new[2, 0])


# ---- planted mistakes

MUTANTS = {
    "copy-on-write skipped": ("cow = L % self.B != 0 and self.ref[self.tables[s, L // self.B]] > 1", "cow = False"),
    "block returned at count one": ("if self.ref[b] == 0:", "if self.ref[b] == 1:"),
    "blocks needed rounded down": ("return (int(length) + self.B - 1) // self.B", "return int(length) // self.B"),
    "free pool last in first out": ("b = self.free.popleft()", "b = self.free.pop()"),
    "fork does not count": ("self.ref[b] += 1", "self.ref[b] += 0"),
    "copy keeps the old count": ("self.ref[old] -= 1", "self.ref[old] -= 0"),
    "admission goes on after a miss": ("stopped = True", "stopped = False"),
    "slot offset off by one": ("* self.B + pos % self.B", "* self.B + (pos + 1) % self.B"),
    "free leaves the row": ("                self.tables[s, j] = -1\n", "                pass\n"),
    "copy taken after the new blocks": ("            if cow:\n                old", "            if False:\n                old"),
}


def load_mutant(name):
    src = open(blocks.__file__).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    mod = types.ModuleType(f"blocks_mutant_{abs(hash(name))}")
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(name):
    mod = load_mutant(name)
    caught = []
    try:
        replay_golden(mod)
    except (AssertionError, IndexError, KeyError, ValueError):
        caught.append("golden")
    for seed in range(6):
        try:
            random_run(mod, seed)
        except (AssertionError, IndexError, KeyError, ValueError):
            caught.append(f"random {seed}")
            break
    assert caught, f"planted mistake '{name}' passed every pin"
