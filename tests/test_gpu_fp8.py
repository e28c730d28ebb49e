"""8-bit (e4m3) KV pools on the GPU: the quantising write against the
oracle's write byte for byte (ties, saturation, subnormal codes and padding
slots included), and decode (one pass, split with fused merge, split with the
merge kernel) against the oracle's decode over dequantised codes, within the
16-bit tolerance (2e-2 absolute + 2e-2 relative)."""

import numpy as np
import pytest
import torch

import oracle
import workloads
import paged_kv_cache_449_b200 as pa
from pagedutil import as_f64, check_tolerance, compact_for_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.fixture(autouse=True)
def no_device_errors():
    pa.pa_get_device_error()
    yield
    assert pa.pa_get_device_error() == 0


def _fp8_pools(num_blocks, hkv, d, b):
    shape = pa.fp8_pool_shape(num_blocks, hkv, d, b)
    g = torch.Generator().manual_seed(num_blocks)
    k = torch.randint(0, 256, shape, generator=g, dtype=torch.int32).to(torch.uint8)   # untouched bytes pattern
    return k, k.flip(0).contiguous()


def _rows_with_edge_values(T, hkv, d, dtype, scales, seed):
    """N(0,1) rows plus, per row, exact e4m3 midpoints (ties), values past
    the saturation bound and values in the subnormal range, all relative to
    the row's kv-head scale (a power of two keeps them exact)."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((T, hkv, d), generator=g) * 3
    ties = torch.tensor([1.0625, 1.1875, -2.125, 0.0009765625, 3 * 2.0 ** -11, 13.0, 104.0, 464.0])
    big = torch.tensor([470.0, -500.0, 1e6, 448.0])
    tiny = torch.tensor([2.0 ** -9, 5 * 2.0 ** -10, -7 * 2.0 ** -9, 2.0 ** -12])
    edge = torch.cat([ties, big, tiny])
    for h in range(hkv):
        x[:, h, :edge.numel()] = edge * float(scales[h])
    return x.to(dtype)


CASES = [(torch.bfloat16, 128, 16, 8), (torch.float16, 64, 8, 2), (torch.float32, 128, 32, 4),
         (torch.bfloat16, 64, 32, 1), (torch.float16, 128, 16, 2)]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_quantising_write_is_bit_exact(orc, case):
    dt, D, B, Hkv = CASES[case]
    N, T = 9, 20
    ks = torch.tensor([2.0 ** (-3 - h) for h in range(Hkv)], dtype=torch.float32)
    vs = torch.tensor([0.0173 * (h + 1) for h in range(Hkv)], dtype=torch.float32)   # not powers of two
    key = _rows_with_edge_values(T, Hkv, D, dt, ks, 500 + case)
    value = _rows_with_edge_values(T, Hkv, D, dt, vs, 600 + case)
    rng = np.random.default_rng(700 + case)
    slots = torch.from_numpy(rng.choice(N * B, size=T, replace=False).astype(np.int64))
    slots[::7] = -1   # padding tokens
    k0, v0 = _fp8_pools(N, Hkv, D, B)
    kd, vd = k0.cuda(), v0.cuda()
    pa.pa_reshape_and_cache_fp8(key.cuda(), value.cuda(), kd, vd, slots.cuda(), ks.cuda(), vs.cuda())
    torch.cuda.synchronize()
    ko, vo = k0.clone(), v0.clone()
    orc.reshape_and_cache_e4m3(key, value, ko, vo, slots, ks, vs, B)
    assert torch.equal(kd.cpu(), ko) and torch.equal(vd.cpu(), vo)


def _gpu_fp8_decode(b, pools, mode, part=512, dev=None):
    q = b.q.cuda().contiguous()
    out = torch.full_like(q, float("nan"))
    bt, cl = b.block_tables.cuda(), b.context_lens.cuda()
    args = (out, q, pools.k_cache, pools.v_cache, pools.k_scale, pools.v_scale, bt, cl, b.scale)
    if mode == "single":
        pa.pa_decode_fp8(*args, max_context_len=b.max_context_len)
    else:
        pa.pa_decode_splitk_fp8(*args, b.max_context_len, partition_size=part, fused=(mode == "splitk"))
    torch.cuda.synchronize()
    return out


def _oracle_fp8(orc, b, pools, seqs):
    q, _, _, bt, cl = compact_for_oracle(b, seqs)
    used = sorted(set(int(x) for x in b.block_tables[list(seqs)][b.block_tables[list(seqs)] >= 0].tolist()))
    remap = {o: n for n, o in enumerate(used)}
    bt = b.block_tables[list(seqs)].clone()
    for i in range(bt.shape[0]):
        for j in range(bt.shape[1]):
            x = int(bt[i, j])
            if x >= 0:
                bt[i, j] = remap[x]
    idx = torch.tensor(used if used else [0], dtype=torch.int64, device=pools.k_cache.device)
    kc = pools.k_cache[idx].cpu().contiguous()
    vc = pools.v_cache[idx].cpu().contiguous()
    return orc.decode_e4m3(q, kc, vc, pools.k_scale.cpu().contiguous(), pools.v_scale.cpu().contiguous(),
                           bt, cl, b.scale, b.block_size, b.num_kv_heads)


SMALL = [
    # q dtype, D, B, Hq, Hkv, lens, q multiplier (exercises the bf16 query scaling)
    (torch.bfloat16, 128, 16, 32, 8, (1, 15, 16, 17, 250, 0), 1.0),
    (torch.bfloat16, 128, 8, 8, 4, (0, 1, 7, 8, 9, 130), 1e3),
    (torch.bfloat16, 64, 32, 16, 2, (33, 64, 95, 2), 1e-4),
    (torch.float16, 128, 16, 64, 8, (300, 12, 1), 1.0),
    (torch.float16, 64, 8, 2, 2, (77, 0, 5), 20.0),
    (torch.bfloat16, 64, 16, 8, 8, (40, 3, 200), 3e4),
]


@pytest.mark.parametrize("case", range(len(SMALL)))
def test_decode_every_element(orc, case):
    dt, D, B, Hq, Hkv, lens, qmul = SMALL[case]
    b = workloads.random_small(seed=800 + case, dtype=dt, lens=lens, num_q_heads=Hq, num_kv_heads=Hkv,
                               head_dim=D, block_size=B, extra_blocks=5)
    b.q = (b.q.to(torch.float32) * qmul).to(dt)
    b.scale = b.scale / qmul if qmul > 1 else b.scale
    pools = workloads.random_fp8_pools(b, seed=900 + case, device="cuda")
    ref = _oracle_fp8(orc, b, pools, range(b.num_seqs))
    for mode, part in (("single", 0), ("splitk", max(16, B)), ("splitk2", 64), ("splitk", 512)):
        got = _gpu_fp8_decode(b, pools, mode, part or 512)
        check_tolerance(as_f64(got), ref, dt)


def test_write_then_decode_roundtrip(orc):
    """Pools filled by the GPU's quantising write, then decoded: the same as
    the oracle's write followed by its decode."""
    b = workloads.random_small(seed=950, dtype=torch.bfloat16, lens=(40, 17, 100), num_q_heads=8, num_kv_heads=2,
                               head_dim=128, block_size=16, extra_blocks=3)
    ks = torch.tensor([0.011, 0.027], dtype=torch.float32)
    vs = torch.tensor([0.019, 0.007], dtype=torch.float32)
    kc = torch.zeros(pa.fp8_pool_shape(b.num_blocks, 2, 128, 16), dtype=torch.uint8)
    vc = torch.zeros_like(kc)
    kd, vd = kc.cuda(), vc.cuda()
    from pagedutil import logical_kv
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        per_head = [logical_kv(b, s, h) for h in range(2)]
        keys = torch.from_numpy(np.stack([k for k, _ in per_head], axis=1)).to(torch.bfloat16).contiguous()
        vals = torch.from_numpy(np.stack([v for _, v in per_head], axis=1)).to(torch.bfloat16).contiguous()
        slots = torch.tensor([int(b.block_tables[s, t // 16]) * 16 + t % 16 for t in range(L)], dtype=torch.int64)
        pa.pa_reshape_and_cache_fp8(keys.cuda(), vals.cuda(), kd, vd, slots.cuda(), ks.cuda(), vs.cuda())
        orc.reshape_and_cache_e4m3(keys, vals, kc, vc, slots, ks, vs, 16)
    torch.cuda.synchronize()
    assert torch.equal(kd.cpu(), kc) and torch.equal(vd.cpu(), vc)
    pools = workloads.Fp8Pools(kd, vd, ks.cuda(), vs.cuda())
    ref = orc.decode_e4m3(b.q, kc, vc, ks, vs, b.block_tables, b.context_lens, b.scale, 16, 2)
    check_tolerance(as_f64(_gpu_fp8_decode(b, pools, "single")), ref, torch.bfloat16)


@pytest.mark.parametrize("wl,part", [("llama3_8b_decode", 1024), ("llama3_70b_long", 1024)])
def test_full_size_sampled(orc, wl, part):
    b = workloads.CONFIGS[wl](seed=7, device="cuda")
    pools = workloads.random_fp8_pools(b, seed=8, device="cuda")
    seqs = sorted(set(np.random.default_rng(9).choice(b.num_seqs, size=4, replace=False).tolist()))
    ref = _oracle_fp8(orc, b, pools, seqs)
    for mode in ("single", "splitk"):
        got = _gpu_fp8_decode(b, pools, mode, part)
        check_tolerance(as_f64(got[seqs]), ref, b.dtype)
        assert torch.isfinite(got.float()).all()


def test_fp32_queries_are_refused():
    b = workloads.random_small(seed=960, dtype=torch.float32, lens=(5,), num_q_heads=2, num_kv_heads=2,
                               head_dim=64, block_size=16)
    pools = workloads.random_fp8_pools(b, seed=1, device="cuda")
    with pytest.raises(pa.PagedAttentionError) as e:
        _gpu_fp8_decode(b, pools, "single")
    assert e.value.status == 2


@pytest.mark.parametrize("make", [
    lambda: workloads.llama3_8b_decode(seed=1100, device="cuda", num_seqs=24, num_blocks=4096),
    lambda: workloads.continuous_batching_mix(seed=1101, device="cuda", num_seqs=40, block_size=8),
    lambda: workloads.random_small(seed=1102, dtype=torch.float16, lens=(0, 1, 16, 17, 300), num_q_heads=8,
                                   num_kv_heads=2, head_dim=64, block_size=32),
    lambda: workloads.random_small(seed=1103, dtype=torch.bfloat16, lens=(5, 33, 64, 2), num_q_heads=8,
                                   num_kv_heads=8, head_dim=128, block_size=16),
])
def test_append_fp8_equals_write_then_decode(make):
    b = make()
    pools = workloads.random_fp8_pools(b, seed=1110, device="cuda")
    q, bt, cl = b.q.cuda().contiguous(), b.block_tables.cuda(), b.context_lens.cuda()
    nk, nv = b.new_key.cuda().contiguous(), b.new_value.cuda().contiguous()
    k1, v1 = pools.k_cache.clone(), pools.v_cache.clone()
    k2, v2 = pools.k_cache.clone(), pools.v_cache.clone()
    ref = torch.full_like(q, float("nan"))
    pa.pa_reshape_and_cache_fp8(nk, nv, k1, v1, b.slot_mapping.cuda(), pools.k_scale, pools.v_scale)
    pa.pa_decode_fp8(ref, q, k1, v1, pools.k_scale, pools.v_scale, bt, cl, b.scale, max_context_len=b.max_context_len)
    got = torch.full_like(q, float("nan"))
    pa.pa_decode_append_fp8(got, q, nk, nv, k2, v2, pools.k_scale, pools.v_scale, bt, cl, b.scale,
                            max_context_len=b.max_context_len)
    torch.cuda.synchronize()
    assert torch.equal(k2, k1) and torch.equal(v2, v1)
    bits = lambda t: t.contiguous().view(-1).view(torch.int16)
    assert torch.equal(bits(got), bits(ref))


# ---------------------------------------------------------------------------- needles

@pytest.mark.parametrize("qdt,D,B,mode,part", [
    (torch.bfloat16, 128, 16, "single", None),    # deep ring of 3 stages: two blocks per softmax step
    (torch.float16, 128, 16, "splitk", 64),
    (torch.bfloat16, 64, 16, "splitk2", 128),
    (torch.bfloat16, 128, 32, "single", None),
    (torch.float16, 64, 8, "single", None),
])
def test_needle_every_position(orc, qdt, D, B, mode, part):
    """Scales 1, K codes 0 except e4m3(64) in dim 0 of one logical token t*
    of kv head 1, q = 64 e_0 in that head's query heads: t*'s score is 4096
    and every other weight underflows to exactly 0, so those heads' output is
    the dequantised V row of t* bit for bit.  Sweeping t* over every position
    of sequences long enough that each warp of a thread block takes several
    blocks pins the gather, the in-block offsets of both 8-bit tile layouts,
    the pairing of blocks per softmax step (odd counts, a partial last block)
    and the partition boundaries."""
    b = workloads.random_small(seed=1200, dtype=qdt, lens=(600, 1, 290, 529), num_q_heads=8, num_kv_heads=2,
                               head_dim=D, block_size=B, extra_blocks=3)
    b.scale = 1.0
    g = b.group
    b.q.zero_()
    b.q[:, g:2 * g, 0] = 64.0
    shape = pa.fp8_pool_shape(b.num_blocks, b.num_kv_heads, D, B)
    gen = torch.Generator().manual_seed(1201)
    vc = torch.randint(0, 256, shape, generator=gen, dtype=torch.int32).to(torch.uint8)
    vc[(vc & 0x7f) == 0x7f] = 0   # no NaN codes
    ones = torch.ones(b.num_kv_heads, dtype=torch.float32, device="cuda")
    pools = workloads.Fp8Pools(torch.zeros(shape, dtype=torch.uint8, device="cuda"), vc.cuda(), ones, ones.clone())
    kflat = pools.k_cache.view(-1)
    vflat = vc.view(-1)
    needle = orc.e4m3_encode(64.0)
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        for t in range(L):
            blk = int(b.block_tables[s, t // B])
            at = orc.e4m3_k_index(blk, 1, t % B, 0, b.num_kv_heads, B, D)
            kflat[at] = needle
            out = _gpu_fp8_decode(b, pools, mode, part or 512)
            kflat[at] = 0
            # + 0.0: a -0 code (0x80) reads as +0, the sum of the other tokens' zero-weighted terms
            want = (torch.tensor([orc.e4m3_value(int(vflat[orc.e4m3_v_index(blk, 1, t % B, d, b.num_kv_heads, B, D)]))
                                  for d in range(D)], dtype=torch.float64) + 0.0).to(qdt)
            for h in range(g, 2 * g):
                assert torch.equal(out[s, h].cpu().view(torch.int16), want.view(torch.int16)), (s, t, h)
            assert torch.isfinite(out[s, :g].float()).all()
