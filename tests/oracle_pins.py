"""Pins for the oracle: checks against things other than the oracle itself —
hand-derived golden values, closed forms, exact special cases, invariants the
pages fix, long-double brute force on tiny inputs, and library routines for the
number formats.  Each pin takes an ``oracle.Oracle`` so the same suite can be
run against copies of the oracle with planted mistakes (test_oracle_mutants).
"""

from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import workloads
from pagedutil import (as_f64, brute_force, logical_kv, materialize_shared, permute_physical,
                       rel_err, relayout_block_size)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _decode(orc, b, **kw):
    return orc.decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale,
                      b.block_size, b.num_kv_heads, **kw)


def _empty_batch(dtype, lens, Hq, Hkv, D, B, N, tables, scale=1.0):
    x = workloads.vec_elems(dtype)
    S = len(lens)
    return workloads.Batch(
        name="hand", dtype=dtype, num_seqs=S, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
        block_size=B, num_blocks=N, scale=scale,
        context_lens=torch.tensor(lens, dtype=torch.int32),
        block_tables=torch.tensor(tables, dtype=torch.int32),
        q=torch.zeros((S, Hq, D), dtype=dtype),
        k_cache=torch.zeros((N, Hkv, D // x, B, x), dtype=dtype),
        v_cache=torch.zeros((N, Hkv, D // x, B, x), dtype=dtype),
        new_key=torch.zeros((0, Hkv, D), dtype=dtype), new_value=torch.zeros((0, Hkv, D), dtype=dtype),
        slot_mapping=torch.zeros((0,), dtype=torch.int64))


# ---------------------------------------------------------------------------- layout & slots

def pin_layout_golden(orc):
    """Hand-derived element offsets of the pool layout; the oracle's reshape
    must put a written element exactly there and touch nothing else."""
    for c in _golden("pool_layout.json")["cases"]:
        dt = DT[c["dtype"]]
        Hkv, B, D = c["Hkv"], c["B"], c["D"]
        assert orc.pool_index(c["b"], c["h"], c["t"], c["d"], Hkv, B, D, dt) == c["index"], c
        x = workloads.vec_elems(dt)
        N = c["b"] + 1
        k = torch.zeros((N, Hkv, D // x, B, x), dtype=dt)
        v = torch.zeros_like(k)
        key = torch.zeros((1, Hkv, D), dtype=dt)
        key[0, c["h"], c["d"]] = 3.0
        val = torch.zeros_like(key)
        val[0, c["h"], c["d"]] = -5.0
        orc.reshape_and_cache(key, val, k, v, torch.tensor([c["b"] * B + c["t"]]), B)
        kf, vf = k.reshape(-1), v.reshape(-1)
        nz = torch.nonzero(kf).flatten().tolist()
        assert nz == [c["index"]], (c, nz)
        assert float(kf[c["index"]]) == 3.0 and float(vf[c["index"]]) == -5.0
        assert torch.nonzero(vf).flatten().tolist() == [c["index"]]


def pin_slot_golden(orc):
    """The append_token walkthrough: the generator's decode slots and the
    oracle's gather both follow slot = table[p // B] * B + p % B."""
    g = _golden("slot_mapping.json")
    B, row = g["block_size"], g["block_table_row"]
    for p, want in zip(g["positions"], g["slots"]):
        tables = np.array([row], dtype=np.int32)
        assert int(workloads._decode_slots(tables, [p + 1], B)[0]) == want
    for n, want in zip(g["appended"], g["blocks_in_use"]):
        assert (n + B - 1) // B == want
    # Needle through the oracle: write a marked token at the golden slot with
    # the oracle's reshape, then decode must fetch it at that logical position.
    D, N = 8, 16
    for p, slot in zip(g["positions"], g["slots"]):
        b = _empty_batch(torch.float32, [p + 1], 1, 1, D, B, N, [row], scale=1.0)
        key = torch.zeros((1, 1, D)); key[0, 0, 0] = 64.0
        val = torch.arange(1, D + 1, dtype=torch.float32).reshape(1, 1, D) * (p + 1)
        orc.reshape_and_cache(key, val, b.k_cache, b.v_cache, torch.tensor([slot]), B)
        b.q[0, 0, 0] = 64.0
        out = _decode(orc, b)
        assert np.array_equal(out[0, 0], val[0, 0].double().numpy()), (p, out[0, 0])


# ---------------------------------------------------------------------------- attention

def _tiny_cases():
    cases = []
    for seed, (dt, B, lens, Hq, Hkv, D) in enumerate([
        (torch.float32, 1, (3, 1, 7), 1, 1, 8),
        (torch.float32, 2, (5, 4, 0, 9), 4, 2, 16),
        (torch.float32, 16, (1, 17, 33, 40), 4, 4, 64),
        (torch.bfloat16, 8, (40, 3, 12), 8, 2, 16),
        (torch.float16, 16, (2, 31, 16), 8, 1, 64),
        (torch.bfloat16, 16, (1, 25), 4, 1, 128),
        (torch.float16, 8, (9, 40, 16, 1), 8, 8, 8),
    ]):
        cases.append(workloads.random_small(seed=seed, dtype=dt, lens=lens, num_q_heads=Hq,
                                            num_kv_heads=Hkv, head_dim=D, block_size=B,
                                            extra_blocks=5))
    return cases


def pin_brute_force(orc):
    """Oracle vs long-double dense attention over the logical K/V (numpy view of
    the layout), tiny inputs: <= 1e-12 relative."""
    for b in _tiny_cases():
        got = _decode(orc, b)
        ref = brute_force(b)
        assert rel_err(got, ref) <= 1e-12, (b.name, rel_err(got, ref))


def pin_dense_equality(orc):
    """Dense K/V written into a shuffled paged pool with the oracle's own
    reshape (slot by slot), vs the same K/V as one contiguous block per
    sequence: bit-identical outputs, and equal to brute force."""
    rng = np.random.default_rng(7)
    S, Hq, Hkv, D, B = 3, 4, 2, 16, 8
    lens = [13, 1, 24]
    dt = torch.bfloat16
    dense_k = [torch.randn(L, Hkv, D).to(dt) for L in lens]
    dense_v = [torch.randn(L, Hkv, D).to(dt) for L in lens]
    q = torch.randn(S, Hq, D).to(dt)
    # paged
    nblk = [(L + B - 1) // B for L in lens]
    N = sum(nblk) + 4
    ids = rng.permutation(N)
    tables = np.full((S, max(nblk)), -1, dtype=np.int32)
    cur = 0
    for s in range(S):
        tables[s, :nblk[s]] = ids[cur:cur + nblk[s]]
        cur += nblk[s]
    paged = _empty_batch(dt, lens, Hq, Hkv, D, B, N, tables, scale=0.25)
    paged.q.copy_(q)
    for s in range(S):
        slots = torch.tensor([int(tables[s, t // B]) * B + t % B for t in range(lens[s])])
        orc.reshape_and_cache(dense_k[s].contiguous(), dense_v[s].contiguous(), paged.k_cache,
                              paged.v_cache, slots, B)
    # contiguous: block size = longest context, block s holds sequence s
    Bc = 24
    cont = _empty_batch(dt, lens, Hq, Hkv, D, Bc, S, [[s] for s in range(S)], scale=0.25)
    cont.q.copy_(q)
    for s in range(S):
        orc.reshape_and_cache(dense_k[s].contiguous(), dense_v[s].contiguous(), cont.k_cache,
                              cont.v_cache, torch.arange(lens[s]) + s * Bc, Bc)
    a, c = _decode(orc, paged), _decode(orc, cont)
    assert np.array_equal(a, c)
    # and the dense definition, straight from the dense arrays
    for s in range(S):
        for h in range(Hq):
            kvh = h // (Hq // Hkv)
            K = as_f64(dense_k[s][:, kvh]).astype(np.longdouble)
            V = as_f64(dense_v[s][:, kvh]).astype(np.longdouble)
            z = np.longdouble(0.25) * (K @ as_f64(q[s, h]).astype(np.longdouble))
            w = np.exp(z - z.max())
            ref = (w[:, None] * V).sum(0) / w.sum()
            assert np.max(np.abs(a[s, h] - ref.astype(np.float64))) <= 1e-12 * max(1.0, np.abs(ref).max())


def pin_permutation_invariance(orc):
    for b in _tiny_cases()[2:5]:
        assert np.array_equal(_decode(orc, b), _decode(orc, permute_physical(b, seed=11)))


def pin_block_size_invariance(orc):
    b = workloads.random_small(seed=21, dtype=torch.float16, lens=(70, 1, 33, 16), num_q_heads=8,
                               num_kv_heads=2, head_dim=64, block_size=16)
    ref = _decode(orc, b)
    for nb in (8, 32):
        assert np.array_equal(ref, _decode(orc, relayout_block_size(b, nb)))


def pin_shared_vs_copied(orc):
    for prefix in (32, 40):  # 40: the prefix ends inside a block (copy-on-write block)
        b = workloads.prefix_sharing(seed=3, prefix_len=prefix, num_seqs=3, suffix_range=(1, 20))
        twin = materialize_shared(b)
        assert twin.num_blocks > b.num_blocks
        assert np.array_equal(_decode(orc, b), _decode(orc, twin))


def pin_closed_forms(orc):
    # L = 1: the output is V[0] exactly.
    b = workloads.random_small(seed=31, dtype=torch.bfloat16, lens=(1, 1, 1), num_q_heads=4,
                               num_kv_heads=2, head_dim=16, block_size=8)
    out = _decode(orc, b)
    for s in range(3):
        for h in range(4):
            _, V = logical_kv(b, s, h // 2)
            assert np.array_equal(out[s, h], V[0])
    # q = 0: uniform weights, the output is the mean of V over the context.
    b = workloads.random_small(seed=32, dtype=torch.float32, lens=(5, 12, 33), num_q_heads=2,
                               num_kv_heads=1, head_dim=8, block_size=8)
    b.q.zero_()
    out = _decode(orc, b)
    for s in range(3):
        _, V = logical_kv(b, s, 0)
        assert np.max(np.abs(out[s, 0] - V.mean(axis=0))) <= 1e-14
    # two tokens with scores 0 and 1: logistic weights (golden).
    g = _golden("two_token_logistic.json")
    D = g["head_dim"]
    tb = _empty_batch(torch.float32, [2], 1, 1, D, 16, 1, [[0]], scale=g["scale"])
    tb.q[0, 0] = torch.tensor(g["q"], dtype=torch.float32)
    orc.reshape_and_cache(torch.tensor(g["keys"], dtype=torch.float32).reshape(2, 1, D),
                          torch.tensor(g["values"], dtype=torch.float32).reshape(2, 1, D),
                          tb.k_cache, tb.v_cache, torch.tensor([0, 1]), 16)
    out = _decode(orc, tb)
    assert np.max(np.abs(out[0, 0] - np.array(g["out"]))) <= g["abs_tol"], out[0, 0]
    # empty context: zeros.
    b = workloads.random_small(seed=33, dtype=torch.float16, lens=(0, 4), num_q_heads=2,
                               num_kv_heads=1, head_dim=8, block_size=8)
    out = _decode(orc, b)
    assert np.array_equal(out[0], np.zeros_like(out[0])) and np.any(out[1] != 0)


def pin_needle(orc):
    """q and one key aligned with score 4096 at position t*: every other weight
    is exp(-4096) = 0 in fp64, so the output is V[t*] exactly.  The needle sits
    in one kv head only; the other head's queries see no needle."""
    b = workloads.random_small(seed=41, dtype=torch.bfloat16, lens=(37, 8, 1), num_q_heads=4,
                               num_kv_heads=2, head_dim=16, block_size=8)
    b.scale = 1.0
    B = b.block_size
    for s in range(b.num_seqs):
        for t in range(int(b.context_lens[s])):
            c = permute_physical(b, seed=t)  # fresh copy
            c.k_cache.zero_()
            c.q.zero_()
            c.q[s, 0:2, 0] = 64.0                      # q heads 0,1 -> kv head 0
            blk = int(c.block_tables[s, t // B])
            c.k_cache[blk, 0, 0, t % B, 0] = 64.0      # dim 0 of token t, kv head 0
            out = _decode(orc, c, seqs=[s])
            _, V = logical_kv(c, s, 0)
            assert np.array_equal(out[0, 0], V[t]) and np.array_equal(out[0, 1], V[t]), (s, t)
            _, V1 = logical_kv(c, s, 1)
            assert np.max(np.abs(out[0, 2] - V1.mean(axis=0))) <= 1e-14   # no needle in head 1


def pin_partitioned(orc):
    """Partition + log-sum-exp merge (fp64) equals the plain definition."""
    for b in _tiny_cases():
        plain = _decode(orc, b)
        for part in (1, 3, 8, 16, 512):
            got = _decode(orc, b, partition_size=part)
            assert rel_err(got, plain) <= 1e-13, (b.name, part)


def pin_reshape_scatter(orc):
    """Reshape vs an independent numpy scatter through the 5-D pool view;
    untouched bytes stay as they were; padding slots (-1) write nothing."""
    for dt, B, D in ((torch.bfloat16, 16, 128), (torch.float32, 8, 64), (torch.float16, 32, 64)):
        b = workloads.random_small(seed=51, dtype=dt, lens=(20, 5), num_q_heads=4, num_kv_heads=2,
                                   head_dim=D, block_size=B, extra_blocks=4, new_tokens=12)
        k0, v0 = b.k_cache.clone(), b.v_cache.clone()
        orc.reshape_and_cache(b.new_key, b.new_value, b.k_cache, b.v_cache, b.slot_mapping, B)
        x = workloads.vec_elems(dt)
        for i, slot in enumerate(b.slot_mapping.tolist()):
            if slot < 0:
                continue
            k0[slot // B, :, :, slot % B, :] = b.new_key[i].reshape(b.num_kv_heads, D // x, x)
            v0[slot // B, :, :, slot % B, :] = b.new_value[i].reshape(b.num_kv_heads, D // x, x)
        kb = k0.view(-1).view(torch.int16 if dt != torch.float32 else torch.int32)
        gb = b.k_cache.view(-1).view(kb.dtype)
        assert torch.equal(kb, gb) and torch.equal(
            v0.view(-1).view(kb.dtype), b.v_cache.view(-1).view(kb.dtype))


# ---------------------------------------------------------------------------- block copies (CoW, swap)

def _bits_rows(pool):
    """A pool as [num_blocks, bytes-per-block / 2] 16-bit words: each block
    (all its heads, tokens and dimensions) is one contiguous row."""
    return pool.contiguous().view(pool.shape[0], -1).view(torch.int16)


def pin_copy_blocks_rows(orc):
    """Whole-block copies vs row copies of the pools viewed as [blocks, bytes]
    (no layout arithmetic): each destination row equals its source row, every
    other row keeps its bytes, K and V pools independently."""
    for dt, B, D, Hkv in ((torch.bfloat16, 16, 128, 2), (torch.float32, 8, 64, 3), (torch.float16, 32, 64, 1)):
        src = workloads.random_small(seed=71, dtype=dt, lens=(40, 9), num_q_heads=Hkv, num_kv_heads=Hkv,
                                     head_dim=D, block_size=B, extra_blocks=6)
        dst = workloads.random_small(seed=72, dtype=dt, lens=(17,), num_q_heads=Hkv, num_kv_heads=Hkv,
                                     head_dim=D, block_size=B, extra_blocks=9)
        n_src, n_dst = src.num_blocks, dst.num_blocks
        pairs = torch.tensor([[0, n_dst - 1], [n_src - 1, 0], [2, 3], [2, 5]], dtype=torch.int64)
        for same in (False, True):   # another pool pair (swap) / the same pool pair (copy-on-write)
            if same:
                dk, dv = src.k_cache.clone(), src.v_cache.clone()
                sk, sv = dk, dv
                pairs_s = torch.tensor([[0, n_src - 1], [1, 4]], dtype=torch.int64)
            else:
                dk, dv = dst.k_cache.clone(), dst.v_cache.clone()
                sk, sv = src.k_cache.clone(), src.v_cache.clone()
                pairs_s = pairs
            want_k, want_v = _bits_rows(dk).clone(), _bits_rows(dv).clone()
            src_k_rows, src_v_rows = _bits_rows(sk).clone(), _bits_rows(sv).clone()
            for a, b_ in pairs_s.tolist():
                want_k[b_] = src_k_rows[a]
                want_v[b_] = src_v_rows[a]
            orc.copy_blocks(dk, dv, sk, sv, pairs_s, B)
            assert torch.equal(_bits_rows(dk), want_k) and torch.equal(_bits_rows(dv), want_v), (dt, same)


def pin_copy_on_write_keeps_attention(orc):
    """Copy-on-write ([P4] §2.3): duplicating a shared block into a free block
    and pointing one sequence at the duplicate leaves every sequence's
    attention output bit-identical in fp64."""
    b = workloads.prefix_sharing(seed=73, prefix_len=40, num_seqs=3, block_size=8, suffix_range=(3, 12))
    before = _decode(orc, b)
    used = set(int(x) for x in b.block_tables[b.block_tables >= 0].tolist())
    free = [i for i in range(b.num_blocks) if i not in used]
    extra = 3 - len(free)
    if extra > 0:   # make room for the copies
        pad = torch.zeros((extra,) + tuple(b.k_cache.shape[1:]), dtype=b.k_cache.dtype)
        k = torch.cat([b.k_cache, pad]).contiguous()
        v = torch.cat([b.v_cache, pad]).contiguous()
        free += list(range(b.num_blocks, b.num_blocks + extra))
    else:
        k, v = b.k_cache.clone(), b.v_cache.clone()
    tables = b.block_tables.clone()
    pairs = []
    for s, dst in zip(range(b.num_seqs), free):
        src = int(tables[s, 0])
        pairs.append([src, dst])
        tables[s, 0] = dst
    orc.copy_blocks(k, v, k, v, torch.tensor(pairs, dtype=torch.int64), b.block_size)
    after = orc.decode(b.q, k, v, tables, b.context_lens, b.scale, b.block_size, b.num_kv_heads)
    np.testing.assert_array_equal(after, before)


def pin_swap_round_trip(orc):
    """Preemption by swapping ([P1] §4.2): a sequence's blocks copied out to a
    second (host) pool and back into other free blocks of the device pool,
    with its table rewritten, attend exactly as before."""
    b = workloads.random_small(seed=74, dtype=torch.bfloat16, lens=(37, 20, 5), num_q_heads=4, num_kv_heads=2,
                               head_dim=64, block_size=8, extra_blocks=8)
    before = _decode(orc, b)
    s = 0
    nblk = (int(b.context_lens[s]) + b.block_size - 1) // b.block_size
    ids = [int(x) for x in b.block_tables[s, :nblk]]
    host_k = torch.zeros((nblk,) + tuple(b.k_cache.shape[1:]), dtype=b.k_cache.dtype)
    host_v = torch.zeros_like(host_k)
    k, v = b.k_cache.clone(), b.v_cache.clone()
    orc.copy_blocks(host_k, host_v, k, v, torch.tensor([[i, j] for j, i in enumerate(ids)]), b.block_size)
    used = set(int(x) for x in b.block_tables[b.block_tables >= 0].tolist())
    free = [i for i in range(b.num_blocks) if i not in used][:nblk]
    assert len(free) == nblk
    k[ids] = 0   # the swapped-out blocks are reused by someone else
    v[ids] = 0
    orc.copy_blocks(k, v, host_k, host_v, torch.tensor([[j, f] for j, f in enumerate(free)]), b.block_size)
    tables = b.block_tables.clone()
    tables[s, :nblk] = torch.tensor(free, dtype=torch.int32)
    after = orc.decode(b.q, k, v, tables, b.context_lens, b.scale, b.block_size, b.num_kv_heads)
    np.testing.assert_array_equal(after, before)


# ---------------------------------------------------------------------------- 8-bit (e4m3) pools

def pin_e4m3_golden(orc):
    """Hand-worked e4m3 decodes and encodes (ties to even, saturation)."""
    g = _golden("e4m3.json")
    for c in g["decode"]:
        v = orc.e4m3_value(c["bits"])
        assert v == c["value"] and math.copysign(1, v) == math.copysign(1, c["value"]), c
    for c in g["encode"]:
        assert orc.e4m3_encode(c["value"]) == c["bits"], c


def pin_e4m3_layout_golden(orc):
    """Hand-worked byte offsets of the 8-bit K and V pool layouts."""
    g = _golden("e4m3_layout.json")
    for c in g["k"]:
        assert orc.e4m3_k_index(c["b"], c["h"], c["t"], c["d"], c["Hkv"], c["B"], c["D"]) == c["index"], c
    for c in g["v"]:
        assert orc.e4m3_v_index(c["b"], c["h"], c["t"], c["d"], c["Hkv"], c["B"], c["D"]) == c["index"], c


def pin_e4m3_against_torch(orc):
    """Every code's value against torch's float8_e4m3fn conversion; every
    finite value encodes back to its code; random fp32 values below the
    saturation threshold (464) encode as torch rounds them."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).tolist()
    for c in range(256):
        v = orc.e4m3_value(c)
        if math.isnan(ref[c]):
            assert math.isnan(v), c
            continue
        assert v == ref[c], c
        assert orc.e4m3_encode(v) == c, c
    rng = np.random.default_rng(81)
    xs = np.concatenate([rng.standard_normal(3000) * s for s in (1e-3, 0.1, 3.0, 100.0)]).astype(np.float32)
    xs = xs[np.abs(xs) < 464]
    want = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).tolist()
    for x, w in zip(xs.tolist(), want):
        assert orc.e4m3_encode(x) == w, (x, w)


def _e4m3_batch(orc, seed, dtype, lens, Hq, Hkv, D, B, extra=6, pow2_scales=False):
    """A random batch whose every token is written into e4m3 pools by the
    oracle's quantising write, with per-kv-head scales."""
    b = workloads.random_small(seed=seed, dtype=dtype, lens=lens, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                               block_size=B, extra_blocks=extra)
    rng = np.random.default_rng(seed)
    if pow2_scales:
        ks = torch.tensor(2.0 ** rng.integers(-6, 2, size=Hkv), dtype=torch.float32)
        vs = torch.tensor(2.0 ** rng.integers(-6, 2, size=Hkv), dtype=torch.float32)
    else:
        ks = torch.tensor(rng.uniform(0.002, 0.05, size=Hkv), dtype=torch.float32)
        vs = torch.tensor(rng.uniform(0.002, 0.05, size=Hkv), dtype=torch.float32)
    kc = torch.zeros((b.num_blocks, Hkv, D // 16, B, 16), dtype=torch.uint8)
    vc = torch.zeros_like(kc)
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        if L == 0:
            continue
        per_head = [logical_kv(b, s, h) for h in range(Hkv)]
        keys = torch.from_numpy(np.stack([k for k, _ in per_head], axis=1)).to(dtype).contiguous()
        vals = torch.from_numpy(np.stack([v for _, v in per_head], axis=1)).to(dtype).contiguous()
        slots = torch.tensor([int(b.block_tables[s, t // B]) * B + t % B for t in range(L)], dtype=torch.int64)
        orc.reshape_and_cache_e4m3(keys, vals, kc, vc, slots, ks, vs, B)
    return b, kc, vc, ks, vs


def pin_e4m3_write_then_single_token(orc):
    """Quantising write then a one-token context: the output is the stored V
    row, e4m3(x / scale) * scale, computed here with torch's e4m3 conversion
    (values below the saturation threshold)."""
    for dt in (torch.bfloat16, torch.float16, torch.float32):
        Hkv, D, B = 2, 32, 8
        x = torch.randn((1, Hkv, D), generator=torch.Generator().manual_seed(82), dtype=torch.float32).to(dt)
        ks = torch.tensor([0.02, 0.5], dtype=torch.float32)
        vs = torch.tensor([0.01, 0.25], dtype=torch.float32)
        kc = torch.zeros((3, Hkv, D // 16, B, 16), dtype=torch.uint8)
        vc = torch.zeros_like(kc)
        orc.reshape_and_cache_e4m3(x, x, kc, vc, torch.tensor([2 * B]), ks, vs, B)
        q = torch.randn((1, 2 * Hkv, D), generator=torch.Generator().manual_seed(83)).to(dt)
        out = orc.decode_e4m3(q, kc, vc, ks, vs, torch.tensor([[2]], dtype=torch.int32),
                              torch.tensor([1], dtype=torch.int32), 0.5, B, Hkv)
        xf = x.to(torch.float32)[0]
        for h in range(Hkv):
            stored = ((xf[h] / vs[h]).to(torch.float8_e4m3fn).to(torch.float64) * float(vs[h])).numpy()
            np.testing.assert_array_equal(out[0, 2 * h], stored)
            np.testing.assert_array_equal(out[0, 2 * h + 1], stored)
            kstored = (xf[h] / ks[h]).to(torch.float8_e4m3fn).view(torch.uint8)
            flat = kc.view(-1)
            for d in range(D):
                assert int(flat[orc.e4m3_k_index(2, h, 0, d, Hkv, B, D)]) == int(kstored[d]), (h, d)


def pin_e4m3_decode_is_dense_decode_of_dequantised_pool(orc):
    """With power-of-two scales every code * scale is exact in fp32.  The same
    logical rows are written into 8-bit pools (quantising write) and, after
    quantising and dequantising them with torch's e4m3 conversion, into fp32
    pools (plain write): e4m3 decode must equal the plain decode bit for bit
    in fp64, and the partitioned form must equal it to 1e-13."""
    for dt, B, D, Hq, Hkv, lens in ((torch.bfloat16, 16, 32, 4, 2, (40, 3, 17)),
                                    (torch.float16, 8, 16, 2, 1, (9, 30)),
                                    (torch.bfloat16, 32, 16, 2, 2, (70, 33))):
        b, kc, vc, ks, vs = _e4m3_batch(orc, 83, dt, lens, Hq, Hkv, D, B, pow2_scales=True)
        x = workloads.vec_elems(torch.float32)
        fk = torch.zeros((b.num_blocks, Hkv, D // x, B, x), dtype=torch.float32)
        fv = torch.zeros_like(fk)
        for s in range(b.num_seqs):
            L = int(b.context_lens[s])
            if L == 0:
                continue
            per_head = [logical_kv(b, s, h) for h in range(Hkv)]
            keys = torch.from_numpy(np.stack([k for k, _ in per_head], axis=1)).to(dt).to(torch.float32)
            vals = torch.from_numpy(np.stack([v for _, v in per_head], axis=1)).to(dt).to(torch.float32)
            dq_k = (keys / ks.view(1, Hkv, 1)).to(torch.float8_e4m3fn).to(torch.float32) * ks.view(1, Hkv, 1)
            dq_v = (vals / vs.view(1, Hkv, 1)).to(torch.float8_e4m3fn).to(torch.float32) * vs.view(1, Hkv, 1)
            slots = torch.tensor([int(b.block_tables[s, t // B]) * B + t % B for t in range(L)], dtype=torch.int64)
            orc.reshape_and_cache(dq_k.contiguous(), dq_v.contiguous(), fk, fv, slots, B)
        q32 = b.q.to(torch.float32).contiguous()
        plain = orc.decode(q32, fk, fv, b.block_tables, b.context_lens, b.scale, B, Hkv)
        got = orc.decode_e4m3(q32, kc, vc, ks, vs, b.block_tables, b.context_lens, b.scale, B, Hkv)
        np.testing.assert_array_equal(got, plain)
        part = orc.decode_e4m3(q32, kc, vc, ks, vs, b.block_tables, b.context_lens, b.scale, B, Hkv,
                               partition_size=16)
        assert rel_err(part, plain) <= 1e-13


def pin_errors(orc):
    from oracle import OracleError
    b = workloads.random_small(seed=61, dtype=torch.float16, lens=(9, 3), num_q_heads=2,
                               num_kv_heads=1, head_dim=8, block_size=8)
    bad = b.block_tables.clone()
    bad[0, 1] = b.num_blocks          # out of range
    for tables, lens, code in ((bad, b.context_lens, "block id"),
                               (b.block_tables, torch.tensor([9, 100], dtype=torch.int32), "context")):
        try:
            orc.decode(b.q, b.k_cache, b.v_cache, tables, lens, b.scale, 8, 1)
        except OracleError as e:
            assert code in str(e)
        else:
            raise AssertionError("oracle accepted bad input")
    try:
        orc.reshape_and_cache(b.new_key, b.new_value, b.k_cache, b.v_cache,
                              torch.tensor([b.num_blocks * 8] * b.new_key.shape[0]), 8)
    except OracleError as e:
        assert "slot" in str(e)
    else:
        raise AssertionError("oracle accepted a slot past the pool")
    try:
        orc.copy_blocks(b.k_cache.clone(), b.v_cache.clone(), b.k_cache, b.v_cache,
                        torch.tensor([[0, b.num_blocks]]), 8)
    except OracleError as e:
        assert "block id" in str(e)
    else:
        raise AssertionError("oracle accepted a block copy past the pool")
    # a negative source id is an empty entry: nothing is copied and nothing is refused
    k2, v2 = b.k_cache.clone(), b.v_cache.clone()
    orc.copy_blocks(k2, v2, k2, v2, torch.tensor([[-1, 0], [-1, -1]]), 8)
    assert torch.equal(k2, b.k_cache) and torch.equal(v2, b.v_cache)


def pin_number_formats(orc):
    """Every fp16 and bf16 bit pattern, and a sample of fp32 patterns, widen
    exactly: L = 1 with q = 0 returns V[0] itself; compared with numpy's
    float16 and torch's bfloat16 conversions to float64."""
    D = 64
    for dt in (torch.float16, torch.bfloat16):
        bits = torch.arange(-32768, 32768, dtype=torch.int32).to(torch.int16)
        vals = bits.view(dt)
        S = vals.numel() // D
        x = workloads.vec_elems(dt)
        b = _empty_batch(dt, [1] * S, 1, 1, D, 8, S, [[s] for s in range(S)])
        rows = vals.reshape(S, D)
        orc.reshape_and_cache(torch.zeros((S, 1, D), dtype=dt), rows.reshape(S, 1, D).contiguous(),
                              b.k_cache, b.v_cache, torch.arange(S) * 8, 8)
        out = _decode(orc, b)[:, 0]
        if dt == torch.float16:
            ref = rows.numpy().view(np.float16).astype(np.float64)
        else:
            ref = rows.to(torch.float64).numpy()
        np.testing.assert_array_equal(out, ref)
    rng = np.random.default_rng(5)
    f32 = rng.integers(0, 2**32, size=64 * D, dtype=np.uint64).astype(np.uint32).view(np.float32)
    f32 = np.where(np.isfinite(f32), f32, 0).astype(np.float32)
    S = f32.size // D
    b = _empty_batch(torch.float32, [1] * S, 1, 1, D, 8, S, [[s] for s in range(S)])
    rows = torch.from_numpy(f32.reshape(S, 1, D).copy())
    orc.reshape_and_cache(torch.zeros_like(rows), rows, b.k_cache, b.v_cache, torch.arange(S) * 8, 8)
    np.testing.assert_array_equal(_decode(orc, b)[:, 0], f32.reshape(S, D).astype(np.float64))


# ---------------------------------------------------------------------------- chunked prefill

def _prefill(orc, b, qs=None, lens=None):
    qs = b.meta["query_start"] if qs is None else qs
    return orc.prefill(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens if lens is None else lens, qs,
                       b.scale, b.block_size, b.num_kv_heads)


def pin_prefill_single_token_chunks_are_decode(orc):
    """Chunks of one token: each query is the newest token of its sequence,
    which is exactly decode ([P1] §4.3 mixes both in one batch)."""
    for dt, B, g in ((torch.bfloat16, 16, 4), (torch.float32, 8, 1)):
        b = workloads.random_small(seed=91, dtype=dt, lens=(1, 17, 40, 5), num_q_heads=2 * g, num_kv_heads=2,
                                   head_dim=32, block_size=B)
        qs = torch.arange(b.num_seqs + 1, dtype=torch.int32)
        np.testing.assert_array_equal(_prefill(orc, b, qs), _decode(orc, b))


def pin_prefill_brute_force(orc):
    """Causal attention by long-double brute force over the logical K/V (a
    separate loop nest): query i of a chunk of Q sees positions 0 .. L-Q+i."""
    for dt, B, Hq, Hkv in ((torch.float32, 8, 4, 2), (torch.float16, 16, 2, 2)):
        b = workloads.chunked_prefill(seed=92, dtype=dt, num_seqs=3, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=16,
                                      block_size=B, context_range=(3, 40), chunk_range=(1, 40))
        got = _prefill(orc, b)
        qs = b.meta["query_start"].tolist()
        g = Hq // Hkv
        for s in range(b.num_seqs):
            L = int(b.context_lens[s])
            Q = qs[s + 1] - qs[s]
            for kvh in range(Hkv):
                K, V = logical_kv(b, s, kvh)
                K, V = K.astype(np.longdouble), V.astype(np.longdouble)
                for i in range(Q):
                    p = L - Q + i
                    for j in range(g):
                        h = kvh * g + j
                        qv = as_f64(b.q[qs[s] + i, h]).astype(np.longdouble)
                        z = (K[:p + 1] @ qv) * np.longdouble(np.float32(b.scale))
                        w = np.exp(z - z.max())
                        ref = (w[:, None] * V[:p + 1]).sum(0) / w.sum()
                        assert rel_err(got[qs[s] + i, h], ref.astype(np.float64)) <= 1e-12, (s, i, h)


def pin_prefill_future_tokens_are_invisible(orc):
    """Changing the K/V of the chunk's last token leaves every earlier query of
    the chunk bit-identical, and changes the last query's output."""
    b = workloads.chunked_prefill(seed=93, dtype=torch.bfloat16, num_seqs=2, num_q_heads=4, num_kv_heads=2,
                                  head_dim=32, block_size=16, context_range=(30, 50), chunk_range=(8, 12))
    before = _prefill(orc, b)
    k, v = b.k_cache.clone(), b.v_cache.clone()
    qs = b.meta["query_start"].tolist()
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        blk = int(b.block_tables[s, (L - 1) // 16])
        k[blk, :, :, (L - 1) % 16, :] = 7.0
        v[blk, :, :, (L - 1) % 16, :] = -9.0
    c = b.__class__(**{**b.__dict__, "k_cache": k, "v_cache": v})
    after = _prefill(orc, c)
    for s in range(b.num_seqs):
        np.testing.assert_array_equal(after[qs[s]:qs[s + 1] - 1], before[qs[s]:qs[s + 1] - 1])
        assert np.abs(after[qs[s + 1] - 1] - before[qs[s + 1] - 1]).max() > 1e-3


def pin_prefill_chunk_split(orc):
    """A chunk of Q tokens equals the same chunk run as two chunks (the first
    Q1 tokens with context L - Q + Q1, then the rest with context L), bit for
    bit: chunking does not change any query's attention."""
    b = workloads.chunked_prefill(seed=94, dtype=torch.float16, num_seqs=3, num_q_heads=4, num_kv_heads=1,
                                  head_dim=16, block_size=8, context_range=(20, 60), chunk_range=(6, 20))
    whole = _prefill(orc, b)
    qs = b.meta["query_start"].tolist()
    for s in range(b.num_seqs):
        Q = qs[s + 1] - qs[s]
        L = int(b.context_lens[s])
        Q1 = Q // 2
        one = b.__class__(**{**b.__dict__, "num_seqs": 1, "q": b.q[qs[s]:qs[s] + Q1].contiguous(),
                             "block_tables": b.block_tables[s:s + 1], "context_lens": torch.tensor([L - Q + Q1],
                                                                                                  dtype=torch.int32)})
        two = b.__class__(**{**b.__dict__, "num_seqs": 1, "q": b.q[qs[s] + Q1:qs[s + 1]].contiguous(),
                             "block_tables": b.block_tables[s:s + 1], "context_lens": torch.tensor([L], dtype=torch.int32)})
        a = _prefill(orc, one, torch.tensor([0, Q1], dtype=torch.int32))
        c = _prefill(orc, two, torch.tensor([0, Q - Q1], dtype=torch.int32))
        np.testing.assert_array_equal(np.concatenate([a, c]), whole[qs[s]:qs[s + 1]])


PINS = [pin_layout_golden, pin_slot_golden, pin_brute_force, pin_dense_equality,
        pin_permutation_invariance, pin_block_size_invariance, pin_shared_vs_copied,
        pin_closed_forms, pin_needle, pin_partitioned, pin_reshape_scatter, pin_errors,
        pin_number_formats, pin_copy_blocks_rows, pin_copy_on_write_keeps_attention, pin_swap_round_trip,
        pin_e4m3_golden, pin_e4m3_layout_golden, pin_e4m3_against_torch, pin_e4m3_write_then_single_token,
        pin_e4m3_decode_is_dense_decode_of_dequantised_pool, pin_prefill_single_token_chunks_are_decode,
        pin_prefill_brute_force, pin_prefill_future_tokens_are_invisible, pin_prefill_chunk_split]
