"""The device block manager (pa_blocks_*) against the block-manager oracle
(GPU).  Its result is deterministic, so after every operation the whole state
is compared exactly: block tables, lengths, reference counts, the free ring's
live entries in order with its head and tail, the step's slots and
copy-on-write pairs, and the device error bits.

  * the hand-worked golden run of tests/golden/block_manager.json;
  * seeded random runs (admissions of whole prompts, forks at random prefix
    lengths, decode steps of one token per running sequence, frees, a pool
    small enough to run out) on pools of 8-, 16- and 32-token blocks;
  * a serving loop end to end: prompts written through the slots the device
    hands out, sequences forked from a shared system prompt, decode steps of
    pa_blocks_append + pa_copy_blocks (the copy-on-write pairs) +
    pa_decode_append on the updated tables, each step's attention compared with
    the oracle's (the oracle's own bookkeeping, block copy, write and decode);
  * pa_decode_append with reference counts refuses to write a newest block
    that two sequences hold."""

import json
import os

import numpy as np
import pytest
import torch

import oracle
import oracle.blocks as ob
import workloads
import paged_kv_cache_449_b200 as pa
from pagedutil import as_f64, check_tolerance

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


class DeviceManager:
    """The device state and the four entry points, driven like the oracle."""

    def __init__(self, num_blocks, num_seqs, max_blocks, block_size):
        d = "cuda"
        self.N, self.B = num_blocks, block_size
        self.ref = torch.full((num_blocks,), 7, dtype=torch.int32, device=d)       # init must overwrite
        self.free_ids = torch.full((num_blocks,), -5, dtype=torch.int32, device=d)
        self.state = torch.full((2,), 123, dtype=torch.int64, device=d)
        self.tables = torch.full((num_seqs, max_blocks), -1, dtype=torch.int32, device=d)
        self.lens = torch.zeros(num_seqs, dtype=torch.int32, device=d)
        pa.pa_blocks_init(self.ref, self.free_ids, self.state)

    def append(self, n):
        n = torch.as_tensor(np.asarray(n), dtype=torch.int32).cuda()
        total = int(n.clamp(min=0).sum())
        slots = torch.full((max(total, 1),), -77, dtype=torch.int64, device="cuda")
        pairs = torch.full((self.tables.shape[0], 2), -77, dtype=torch.int64, device="cuda")
        pa.pa_blocks_append(self.tables, self.lens, n, self.ref, self.free_ids, self.state, slots, pairs, self.B)
        return slots[:total].cpu().numpy(), pairs.cpu().numpy()

    def fork(self, pairs):
        f = torch.as_tensor(np.asarray(pairs, dtype=np.int32).reshape(-1, 3)).cuda()
        pa.pa_blocks_fork(self.tables, self.lens, self.ref, f, self.B)

    def release(self, seqs):
        pa.pa_blocks_release(self.tables, self.lens, self.ref, self.free_ids, self.state,
                             torch.as_tensor(np.asarray(seqs, dtype=np.int32)).cuda(), self.B)

    def live_ring(self):
        head, tail = (int(x) for x in self.state.cpu())
        ids = self.free_ids.cpu().numpy()
        return [int(ids[p % self.N]) for p in range(head, tail)], head, tail


def assert_same_state(dev: DeviceManager, m: ob.BlockManager, where):
    assert dev.ref.cpu().tolist() == m.ref.tolist(), (where, "ref")
    assert dev.lens.cpu().tolist() == m.lens.tolist(), (where, "lens")
    assert dev.tables.cpu().tolist() == m.tables.tolist(), (where, "tables")
    live, head, tail = dev.live_ring()
    _, mh, mt = m.ring()
    assert (head, tail) == (mh, mt), (where, "head/tail")
    assert live == list(m.free), (where, "ring")


def test_golden_run_on_the_device():
    g = json.load(open(os.path.join(HERE, "golden", "block_manager.json")))
    dev = DeviceManager(g["num_blocks"], g["num_seqs"], g["max_blocks_per_seq"], g["block_size"])
    pa.pa_get_device_error()
    for k, op in enumerate(g["ops"]):
        if op["op"] == "append":
            slots, pairs = dev.append(op["n"])
            assert slots.tolist() == op["slots"], (k, op)
            assert pairs.tolist() == op["pairs"], (k, op)
        elif op["op"] == "fork":
            dev.fork(op["pairs"])
        else:
            dev.release(op["seqs"])
        assert pa.pa_get_device_error() == op["err"], (k, op)
        st = op["state"]
        assert dev.ref.cpu().tolist() == st["ref"], k
        assert dev.lens.cpu().tolist() == st["lens"], k
        assert dev.tables.cpu().tolist() == st["tables"], k
        live, head, tail = dev.live_ring()
        assert (live, head, tail) == (st["free"], st["head"], st["tail"]), k
        if "ring" in st:
            assert dev.free_ids.cpu().tolist() == st["ring"], k


def choose_op(rng, lens, max_blocks, block_size):
    """A seeded operation for the current lengths: admit whole prompts, fork a
    running sequence at a random prefix, a one-token decode step for every
    running sequence, or free a few; None when nothing applies."""
    num_seqs = len(lens)
    cap = max_blocks * block_size
    r = rng.random()
    running = np.nonzero(lens > 0)[0]
    empty = np.nonzero(lens == 0)[0]
    if r < 0.25 and len(empty):
        n = np.zeros(num_seqs, dtype=np.int64)
        for s in rng.choice(empty, size=min(len(empty), int(rng.integers(1, 6))), replace=False):
            n[s] = int(rng.integers(1, cap // 2))
        return "append", n
    if r < 0.75 and len(running):
        n = np.zeros(num_seqs, dtype=np.int64)
        n[running] = 1
        return "append", n
    if r < 0.87 and len(running) and len(empty):
        p = int(rng.choice(running))
        return "fork", [(p, int(rng.choice(empty)), int(rng.integers(0, lens[p] + 1)))]
    if len(running):
        return "release", rng.choice(running, size=min(len(running), int(rng.integers(1, 4))), replace=False)
    return None


@pytest.mark.parametrize("block_size", [8, 16, 32])
def test_random_runs_match_the_oracle_exactly(block_size):
    S, MB = 48, 64
    N = 600 if block_size == 8 else 300       # small enough that admissions run out of blocks
    m = ob.BlockManager(N, S, MB, block_size)
    dev = DeviceManager(N, S, MB, block_size)
    pa.pa_get_device_error()
    seen = 0
    rng = np.random.default_rng(block_size)
    for k in range(160):
        pick = choose_op(rng, m.lens, MB, block_size)
        if pick is None:
            continue
        op, arg = pick
        if op == "append":
            slots, pairs = dev.append(arg)
            ms, mp, err = m.append(arg)
            assert slots.tolist() == ms.tolist(), (k, op)
            assert pairs.tolist() == mp.tolist(), (k, op)
        elif op == "fork":
            dev.fork(arg)
            err = m.fork(arg)
        else:
            dev.release(arg)
            err = m.release(arg)
        assert pa.pa_get_device_error() == err, (k, op)
        seen |= err
        assert_same_state(dev, m, (k, op))
    assert seen & ob.ERR_NO_FREE_BLOCK        # the run did exhaust the pool at least once


def test_many_sequences_and_long_prompts():
    """More sequences than threads of the launch, and more copy-on-write
    writers into one shared partial block (1201) than threads."""
    S, MB, B, N = 2100, 80, 16, 40000
    m = ob.BlockManager(N, S, MB, B)
    dev = DeviceManager(N, S, MB, B)
    pa.pa_get_device_error()
    rng = np.random.default_rng(5)
    n = np.zeros(S, dtype=np.int64)
    n[:3] = [1250, 37, 1279]                   # 79, 3 and 80 blocks
    for op, arg in (("append", n), ("fork", [(1, c, 37) for c in range(3, 1203)]),
                    ("append", np.where(np.arange(S) < 1203, 1, 0)),
                    ("append", rng.integers(0, 3, size=S)),
                    ("release", np.arange(0, S, 2)), ("append", rng.integers(0, 40, size=S))):
        if op == "append":
            slots, pairs = dev.append(arg)
            ms, mp, err = m.append(arg)
            assert slots.tolist() == ms.tolist() and pairs.tolist() == mp.tolist(), op
        elif op == "fork":
            dev.fork(arg)
            err = m.fork(arg)
        else:
            dev.release(arg)
            err = m.release(arg)
        assert pa.pa_get_device_error() == err, op
        assert_same_state(dev, m, op)


def test_serving_loop_attention_matches_the_oracle():
    """Admit prompts, fork children from a shared system prompt (partial last
    block), run decode steps through the device block manager and compare
    every step's attention with the oracle's bookkeeping + copy + write +
    decode."""
    orc = oracle.default()
    dt, Hq, Hkv, D, B = torch.bfloat16, 32, 8, 128, 16
    S, MB, N = 24, 40, 700
    base = workloads.random_small(seed=61, dtype=dt, lens=(1,), num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                                  block_size=B, extra_blocks=N - 1)
    k_dev, v_dev = base.k_cache.cuda().contiguous(), base.v_cache.cuda().contiguous()
    k_ref, v_ref = base.k_cache.clone(), base.v_cache.clone()
    m = ob.BlockManager(N, S, MB, B)
    dev = DeviceManager(N, S, MB, B)
    pa.pa_get_device_error()
    gen = torch.Generator().manual_seed(62)

    def write(slots, pairs):
        live = pairs[pairs[:, 0] >= 0]
        pa.pa_copy_blocks(k_dev, v_dev, k_dev, v_dev, torch.from_numpy(pairs).cuda())
        if len(live):
            orc.copy_blocks(k_ref, v_ref, k_ref, v_ref, torch.from_numpy(live), B)
        T = len(slots)
        kn = torch.randn((T, Hkv, D), generator=gen).to(dt)
        vn = torch.randn((T, Hkv, D), generator=gen).to(dt)
        pa.pa_reshape_and_cache(kn.cuda(), vn.cuda(), k_dev, v_dev, torch.from_numpy(slots).cuda())
        orc.reshape_and_cache(kn, vn, k_ref, v_ref, torch.from_numpy(slots), B)

    # system prompt in sequence 0 (37 tokens: the last block is partly filled), other prompts
    n = np.zeros(S, dtype=np.int64)
    n[0], n[1], n[2] = 37, 300, 5
    slots, pairs = dev.append(n)
    ms, mp, _ = m.append(n)
    assert slots.tolist() == ms.tolist()
    write(slots, pairs)
    forks = [(0, c, 37) for c in range(3, 12)] + [(1, 12, 160), (1, 13, 299)]
    dev.fork(forks)
    m.fork(forks)
    for step in range(6):
        running = (m.lens > 0).astype(np.int64)
        slots, pairs = dev.append(running)
        ms, mp, _ = m.append(running)
        assert slots.tolist() == ms.tolist() and pairs.tolist() == mp.tolist(), step
        if step == 0:
            assert (mp[:, 0] >= 0).sum() >= 9          # the children copied the shared partial block
        # the step: copies, then pa_decode_append writes each newest token and attends
        live = mp[mp[:, 0] >= 0]
        pa.pa_copy_blocks(k_dev, v_dev, k_dev, v_dev, torch.from_numpy(pairs).cuda())
        if len(live):
            orc.copy_blocks(k_ref, v_ref, k_ref, v_ref, torch.from_numpy(live), B)
        kn = torch.randn((S, Hkv, D), generator=gen).to(dt)
        vn = torch.randn((S, Hkv, D), generator=gen).to(dt)
        q = torch.randn((S, Hq, D), generator=gen).to(dt)
        out = torch.full((S, Hq, D), float("nan"), dtype=dt, device="cuda")
        pa.pa_decode_append(out, q.cuda(), kn.cuda(), vn.cuda(), k_dev, v_dev, dev.tables, dev.lens, D ** -0.5,
                            max_context_len=MB * B, ref_counts=dev.ref)
        # the oracle: write each running sequence's token at its slot, then decode
        order = np.nonzero(running)[0]
        orc.reshape_and_cache(kn[order].contiguous(), vn[order].contiguous(), k_ref, v_ref, torch.from_numpy(ms), B)
        ref = orc.decode(q, k_ref, v_ref, torch.from_numpy(m.tables.astype(np.int32)),
                         torch.from_numpy(m.lens.astype(np.int32)), D ** -0.5, B, Hkv)
        got = as_f64(out)
        check_tolerance(got[order], ref[order], dt)
        assert pa.pa_get_device_error() == 0, step
        assert_same_state(dev, m, step)
    assert torch.equal(k_dev.cpu(), k_ref) and torch.equal(v_dev.cpu(), v_ref)
    # finished sequences return their blocks
    dev.release([0, 3, 4, 12])
    m.release([0, 3, 4, 12])
    assert_same_state(dev, m, "release")


def test_decode_append_refuses_a_shared_newest_block():
    """Two sequences whose newest token falls in one block (a table that
    skipped copy-on-write): with reference counts given, the write is skipped
    and PA_DEVERR_SHARED_BLOCK set; the other sequences are unaffected."""
    b = workloads.random_small(seed=63, dtype=torch.bfloat16, lens=(40, 40, 70), num_q_heads=8, num_kv_heads=2,
                               head_dim=128, block_size=16, extra_blocks=3)
    bt = b.block_tables.clone()
    bt[1, :3] = bt[0, :3]                             # sequence 1 aliases all of sequence 0's blocks
    ref = torch.zeros(b.num_blocks, dtype=torch.int32)
    for s in range(3):
        for j in range((int(b.context_lens[s]) + 15) // 16):
            ref[int(bt[s, j])] += 1
    k, v = b.k_cache.cuda().contiguous(), b.v_cache.cuda().contiguous()
    k0 = k.clone()
    out = torch.empty(b.q.shape, dtype=b.q.dtype, device="cuda")
    pa.pa_get_device_error()
    pa.pa_decode_append(out, b.q.cuda(), b.new_key.cuda(), b.new_value.cuda(), k, v, bt.cuda(),
                        b.context_lens.cuda(), b.scale, ref_counts=ref.cuda())
    assert pa.pa_get_device_error() & pa.DEVERR_SHARED_BLOCK
    newest = int(bt[0, 39 // 16])
    assert torch.equal(k[newest].cpu(), k0[newest].cpu())         # the shared block is untouched
    # sequence 2's block is private: written and attended as usual
    orc = oracle.default()
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    slots = torch.tensor([-1, -1, int(b.slot_mapping[2])], dtype=torch.int64)
    orc.reshape_and_cache(b.new_key, b.new_value, kc, vc, slots, 16)
    ref_out = orc.decode(b.q, kc, vc, bt, b.context_lens, b.scale, 16, 2)
    check_tolerance(as_f64(out), ref_out, b.dtype)      # 0 and 1 attend over the pool as it was
    assert torch.equal(k.cpu()[int(bt[2, 69 // 16])], kc[int(bt[2, 69 // 16])])
