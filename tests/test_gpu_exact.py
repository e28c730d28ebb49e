"""Bit-exact properties of the CUDA path (GPU): the KV-cache write against the
oracle byte for byte, indexing by needles, invariance under physical block
permutation and under shared-vs-copied prefix blocks, run-to-run determinism,
and the device-side error word for malformed block tables and slots."""

import numpy as np
import pytest
import torch

import oracle
import workloads
import paged_kv_cache_449_b200 as pa
from pagedutil import (as_f64, check_tolerance, device_batch, gpu_decode, logical_kv, materialize_shared,
                       oracle_decode_sampled, permute_physical, relayout_block_size)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


def _bits(t):
    return t.contiguous().view(-1).view(torch.int32 if t.element_size() == 4 else torch.int16)


def _reshape_vs_oracle(orc, b):
    """GPU reshape on the full pool; the oracle repeats it on the touched
    blocks (copied to the CPU) and every pool byte is compared."""
    dev = {k: getattr(b, k).cuda().contiguous() for k in ("new_key", "new_value", "k_cache", "v_cache")}
    slots = b.slot_mapping.cuda()
    before_k, before_v = dev["k_cache"].clone(), dev["v_cache"].clone()
    pa.pa_reshape_and_cache(dev["new_key"], dev["new_value"], dev["k_cache"], dev["v_cache"], slots)
    torch.cuda.synchronize()
    B = b.block_size
    valid = b.slot_mapping[b.slot_mapping >= 0]
    touched = sorted(set((valid // B).tolist()))
    # untouched blocks keep every byte
    mask = torch.ones(b.num_blocks, dtype=torch.bool, device="cuda")
    if touched:
        mask[torch.tensor(touched, device="cuda")] = False
    assert torch.equal(_bits(dev["k_cache"][mask]), _bits(before_k[mask]))
    assert torch.equal(_bits(dev["v_cache"][mask]), _bits(before_v[mask]))
    if not touched:
        return
    idx = torch.tensor(touched, device="cuda")
    sub_k, sub_v = before_k[idx].cpu().contiguous(), before_v[idx].cpu().contiguous()
    remap = {blk: i for i, blk in enumerate(touched)}
    sub_slots = torch.tensor([remap[s // B] * B + s % B if s >= 0 else -1 for s in b.slot_mapping.tolist()])
    orc.reshape_and_cache(b.new_key.cpu().contiguous(), b.new_value.cpu().contiguous(), sub_k, sub_v,
                          sub_slots, B)
    assert torch.equal(_bits(dev["k_cache"][idx].cpu()), _bits(sub_k))
    assert torch.equal(_bits(dev["v_cache"][idx].cpu()), _bits(sub_v))


def test_reshape_tiny_f32(orc):
    _reshape_vs_oracle(orc, workloads.tiny_mha_f32(seed=0))


def test_reshape_long_context_random_free_slots(orc):
    _reshape_vs_oracle(orc, workloads.llama3_70b_long(seed=0, device="cuda"))


@pytest.mark.parametrize("dtype,D,B", [(torch.bfloat16, 128, 8), (torch.float16, 64, 32), (torch.float32, 128, 16)])
def test_reshape_with_padding_slots(orc, dtype, D, B):
    b = workloads.random_small(seed=3, dtype=dtype, lens=(20, 5, 40), num_q_heads=4, num_kv_heads=2, head_dim=D,
                               block_size=B, extra_blocks=6, new_tokens=40)
    assert (b.slot_mapping < 0).any()
    _reshape_vs_oracle(orc, b)


def test_reshape_then_decode_sees_the_new_token(orc):
    """Write the newest token of every sequence, then decode: the new K/V take
    part exactly as the oracle's write + decode say."""
    b = workloads.continuous_batching_mix(seed=1, device="cuda", num_seqs=24)
    dev = device_batch(b)
    pa.pa_reshape_and_cache(b.new_key.cuda(), b.new_value.cuda(), dev["k_cache"], dev["v_cache"],
                            b.slot_mapping.cuda())
    got = gpu_decode(b, "single", dev=dev)
    kc, vc = b.k_cache.cpu().contiguous(), b.v_cache.cpu().contiguous()
    orc.reshape_and_cache(b.new_key.cpu().contiguous(), b.new_value.cpu().contiguous(), kc, vc,
                          b.slot_mapping, b.block_size)
    assert torch.equal(_bits(dev["k_cache"].cpu()), _bits(kc))
    ref = orc.decode(b.q.cpu().contiguous(), kc, vc, b.block_tables, b.context_lens, b.scale, b.block_size,
                     b.num_kv_heads)
    check_tolerance(as_f64(got), ref, b.dtype)
    assert pa.pa_get_device_error() == 0


# ---------------------------------------------------------------------------- needles

def _needle_batch(dtype, B, lens, Hq=8, Hkv=2, D=128, seed=5):
    b = workloads.random_small(seed=seed, dtype=dtype, lens=lens, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                               block_size=B, extra_blocks=3)
    b.scale = 1.0
    b.q.zero_()
    b.k_cache.zero_()
    return b


@pytest.mark.parametrize("dtype,B,mode,part,D,lens", [
    (torch.bfloat16, 16, "single", None, 128, (70, 1, 33)), (torch.bfloat16, 16, "splitk", 32, 128, (70, 1, 33)),
    (torch.float16, 8, "single", None, 128, (70, 1, 33)), (torch.float16, 32, "splitk", 64, 128, (70, 1, 33)),
    (torch.bfloat16, 8, "splitk", 16, 128, (70, 1, 33)), (torch.float32, 16, "single", None, 128, (70, 1, 33)),
    (torch.float32, 32, "splitk", 32, 128, (70, 1, 33)),
    # deep ring of 4 stages: every warp takes several blocks, two per softmax step
    (torch.bfloat16, 16, "single", None, 64, (300, 1, 161, 16)),
    (torch.float16, 16, "splitk2", 128, 64, (300, 17, 161))])
def test_needle_every_position(dtype, B, mode, part, D, lens):
    """q = 64 e_0 in the query heads of kv head 1; K = 0 except 64 e_0 at one
    logical token t*: that token's score is 4096 and every other weight
    underflows to exactly 0, so the output of those heads is V[t*] bit for
    bit.  Sweeping t* over every position pins the block-table gather, the
    in-block offset, the GQA head mapping, the pairing of blocks per softmax
    step and the partition boundaries."""
    b = _needle_batch(dtype, B, lens, D=D)
    g = b.group
    b.q[:, g:2 * g, 0] = 64.0
    dev = device_batch(b)
    kc = dev["k_cache"]
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        for t in range(L):
            blk = int(b.block_tables[s, t // B])
            kc.zero_()
            kc[blk, 1, 0, t % B, 0] = 64.0                    # kv head 1, dim 0, token t
            out = gpu_decode(b, mode, partition_size=part or 512, dev=dev)
            _, V = logical_kv(b, s, 1)
            want = torch.from_numpy(V[t]).to(dtype)
            for h in range(g, 2 * g):
                assert torch.equal(_bits(out[s, h].cpu()), _bits(want)), (s, t, h)
            # kv head 0's queries (q = 0) see a uniform average: finite, not the needle
            assert torch.isfinite(out[s, :g].float()).all()
    assert pa.pa_get_device_error() == 0


# ---------------------------------------------------------------------------- invariances

def test_permutation_invariance_bit_exact():
    b = workloads.continuous_batching_mix(seed=2, device="cuda", num_seqs=40)
    c = permute_physical(b, seed=9)
    for mode in ("single", "splitk", "splitk2"):
        assert torch.equal(_bits(gpu_decode(b, mode)), _bits(gpu_decode(c, mode)))


@pytest.mark.parametrize("prefix_len", [1024, 1000])
def test_shared_vs_copied_bit_exact(prefix_len):
    b = workloads.prefix_sharing(seed=1, device="cuda", prefix_len=prefix_len, num_seqs=16)
    twin = materialize_shared(b)
    assert twin.num_blocks > b.num_blocks
    for mode in ("single", "splitk", "splitk2"):
        assert torch.equal(_bits(gpu_decode(b, mode)), _bits(gpu_decode(twin, mode)))


def test_block_size_within_tolerance(orc):
    b = workloads.random_small(seed=8, dtype=torch.bfloat16, lens=(300, 17, 64, 1), num_q_heads=32,
                               num_kv_heads=8, head_dim=128, block_size=16)
    ref = orc.decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale, 16, 8)
    for nb in (8, 32):
        c = relayout_block_size(b, nb)
        for mode in ("single", "splitk", "splitk2"):
            check_tolerance(as_f64(gpu_decode(c, mode)), ref, b.dtype)


def test_run_to_run_deterministic():
    b = workloads.llama3_8b_decode(seed=3, device="cuda", num_seqs=16, num_blocks=4096)
    dev = device_batch(b)
    for mode in ("single", "splitk", "splitk2"):
        first = gpu_decode(b, mode, dev=dev)
        for _ in range(3):
            assert torch.equal(_bits(first), _bits(gpu_decode(b, mode, dev=dev)))


# ---------------------------------------------------------------------------- processing order

def _orders(b):
    S = b.num_seqs
    g = torch.Generator().manual_seed(17)
    return [pa.longest_first(b.context_lens), torch.arange(S - 1, -1, -1, dtype=torch.int32),
            torch.randperm(S, generator=g).to(torch.int32)]


@pytest.mark.parametrize("make", [
    # 48 x 8 and 200 x 8 CTAs: more than one wave of resident CTAs, so the
    # L2 warm-up of later CTAs runs as well.
    lambda: workloads.llama3_8b_decode(seed=21, device="cuda", num_seqs=48, num_blocks=4096),
    lambda: workloads.continuous_batching_mix(seed=22, device="cuda", num_seqs=200, block_size=32),
    lambda: workloads.random_small(seed=23, dtype=torch.float32, lens=(0, 5, 16, 300, 33, 1), num_q_heads=4,
                                   num_kv_heads=4, head_dim=64, block_size=8),
])
def test_seq_order_is_bit_identical(make):
    b = make()
    dev = device_batch(b)
    for mode in ("single", "splitk", "splitk2"):
        ref = gpu_decode(b, mode, partition_size=256, dev=dev)
        for order in _orders(b):
            got = gpu_decode(b, mode, partition_size=256, dev=dev, seq_order=order.cuda())
            assert torch.equal(_bits(got), _bits(ref)), mode
    assert pa.pa_get_device_error() == 0


def test_seq_order_append_is_bit_identical():
    b = workloads.continuous_batching_mix(seed=24, device="cuda", num_seqs=64, block_size=16)
    nk, nv = b.new_key.cuda().contiguous(), b.new_value.cuda().contiguous()
    outs, pools = [], []
    for order in [None] + _orders(b):
        d = device_batch(b)
        d["k_cache"], d["v_cache"] = d["k_cache"].clone(), d["v_cache"].clone()
        out = torch.full_like(d["q"], float("nan"))
        pa.pa_decode_append(out, d["q"], nk, nv, d["k_cache"], d["v_cache"], d["block_tables"], d["context_lens"],
                            b.scale, max_context_len=b.max_context_len,
                            seq_order=None if order is None else order.cuda())
        torch.cuda.synchronize()
        outs.append(out)
        pools.append((d["k_cache"], d["v_cache"]))
    for out, (k, v) in zip(outs[1:], pools[1:]):
        assert torch.equal(_bits(out), _bits(outs[0]))
        assert torch.equal(_bits(k), _bits(pools[0][0])) and torch.equal(_bits(v), _bits(pools[0][1]))


def test_seq_order_out_of_range_is_flagged_and_skipped():
    b = workloads.random_small(seed=25, dtype=torch.bfloat16, lens=(40, 20, 70), num_q_heads=4, num_kv_heads=2,
                               head_dim=128, block_size=16)
    dev = device_batch(b)
    ref = gpu_decode(b, "single", dev=dev)
    pa.pa_get_device_error()
    order = torch.tensor([2, 99, 0], dtype=torch.int32, device="cuda")   # sequence 1 left out
    for mode in ("single", "splitk", "splitk2"):
        got = gpu_decode(b, mode, dev=dev, seq_order=order)
        assert pa.pa_get_device_error() & pa.DEVERR_SEQ_ORDER
        for s in (0, 2):
            check_tolerance(as_f64(got[s]), as_f64(ref[s]), b.dtype)
        if mode == "single":
            assert torch.isnan(got[1].float()).all()   # never written
    assert pa.pa_get_device_error() == 0


# ---------------------------------------------------------------------------- error word

def test_out_of_range_block_id_is_flagged_not_read():
    b = workloads.random_small(seed=9, dtype=torch.bfloat16, lens=(40, 20), num_q_heads=4, num_kv_heads=2,
                               head_dim=128, block_size=16)
    pa.pa_get_device_error()
    bad = b.block_tables.clone()
    bad[0, 1] = b.num_blocks + 1000
    bad[1, 0] = -7
    c = b.__class__(**{**b.__dict__, "block_tables": bad})
    for mode in ("single", "splitk", "splitk2"):
        out = gpu_decode(c, mode)
        assert torch.isfinite(out.float()).all()
        assert pa.pa_get_device_error() & pa.DEVERR_BLOCK_ID
    assert pa.pa_get_device_error() == 0


def test_context_len_above_bound_is_flagged():
    b = workloads.random_small(seed=10, dtype=torch.float16, lens=(40, 20), num_q_heads=4, num_kv_heads=2,
                               head_dim=64, block_size=16)
    pa.pa_get_device_error()
    gpu_decode(b, "single", max_context_len=25)        # 40 > 25
    assert pa.pa_get_device_error() & pa.DEVERR_CONTEXT_LEN


def test_slot_past_pool_is_flagged_not_written():
    b = workloads.random_small(seed=11, dtype=torch.bfloat16, lens=(10, 10), num_q_heads=4, num_kv_heads=2,
                               head_dim=128, block_size=16, new_tokens=4)
    k, v = b.k_cache.cuda(), b.v_cache.cuda()
    k0 = k.clone()
    slots = torch.tensor([b.num_blocks * 16 + 3, -1, -1, b.num_blocks * 16 * 5], device="cuda")
    pa.pa_get_device_error()
    pa.pa_reshape_and_cache(b.new_key.cuda(), b.new_value.cuda(), k, v, slots)
    assert pa.pa_get_device_error() & pa.DEVERR_SLOT
    assert torch.equal(_bits(k), _bits(k0))


def test_host_side_errors_raise():
    b = workloads.random_small(seed=12, dtype=torch.bfloat16, lens=(10,), num_q_heads=4, num_kv_heads=2,
                               head_dim=128, block_size=16)
    dev = device_batch(b)
    out = torch.empty_like(dev["q"])
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_decode_splitk(out, dev["q"], dev["k_cache"], dev["v_cache"], dev["block_tables"],
                            dev["context_lens"], b.scale, 10, partition_size=512,
                            workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 3
    with pytest.raises(pa.PagedAttentionError):
        pa.pa_decode(out, dev["q"][:, :3].contiguous(), dev["k_cache"], dev["v_cache"], dev["block_tables"],
                     dev["context_lens"], b.scale)   # 3 q heads over 2 kv heads


# ---------------------------------------------------------------------------- append (write + decode in one launch)

@pytest.mark.parametrize("make", [
    lambda: workloads.tiny_mha_f32(seed=0),
    lambda: workloads.continuous_batching_mix(seed=4, device="cuda", num_seqs=40, block_size=8),
    lambda: workloads.llama3_8b_decode(seed=5, device="cuda", num_seqs=24, num_blocks=4096),
    lambda: workloads.random_small(seed=6, dtype=torch.float16, lens=(0, 1, 16, 17, 300), num_q_heads=8,
                                   num_kv_heads=2, head_dim=64, block_size=32),
])
def test_append_equals_reshape_then_decode(orc, make):
    b = make()
    # separate pools for the two routes
    d1, d2 = device_batch(b), device_batch(b)
    d2["k_cache"], d2["v_cache"] = d2["k_cache"].clone(), d2["v_cache"].clone()
    nk, nv = b.new_key.cuda().contiguous(), b.new_value.cuda().contiguous()
    pa.pa_reshape_and_cache(nk, nv, d1["k_cache"], d1["v_cache"], b.slot_mapping.cuda())
    ref_gpu = gpu_decode(b, "single", dev=d1)
    out = torch.full_like(d2["q"], float("nan"))
    pa.pa_decode_append(out, d2["q"], nk, nv, d2["k_cache"], d2["v_cache"], d2["block_tables"], d2["context_lens"],
                        b.scale, max_context_len=b.max_context_len)
    torch.cuda.synchronize()
    assert torch.equal(_bits(out), _bits(ref_gpu))
    assert torch.equal(_bits(d2["k_cache"]), _bits(d1["k_cache"]))
    assert torch.equal(_bits(d2["v_cache"]), _bits(d1["v_cache"]))
    # and the oracle's write + decode
    seqs = list(range(0, b.num_seqs, max(1, b.num_seqs // 8)))
    kc, vc = b.k_cache.cpu().contiguous(), b.v_cache.cpu().contiguous()
    orc.reshape_and_cache(b.new_key.cpu().contiguous(), b.new_value.cpu().contiguous(), kc, vc, b.slot_mapping,
                          b.block_size)
    c = b.__class__(**{**b.__dict__, "k_cache": kc, "v_cache": vc})
    check_tolerance(as_f64(out[seqs]), oracle_decode_sampled(orc, c, seqs), b.dtype)
    assert pa.pa_get_device_error() == 0


@pytest.mark.parametrize("fp8", [False, True])
def test_prepared_call_repeats_the_entry(fp8):
    """A prepared decode step makes the same call as the entry point: outputs
    and pools bit-identical, also after the buffers' contents change between
    calls (new queries and new tokens written in place)."""
    b = workloads.llama3_8b_decode(seed=1300, device="cuda", num_seqs=24, num_blocks=4096)
    q, nk, nv = b.q.cuda().contiguous(), b.new_key.cuda().contiguous(), b.new_value.cuda().contiguous()
    bt, cl = b.block_tables.cuda(), b.context_lens.cuda()
    if fp8:
        pools = workloads.random_fp8_pools(b, seed=1301, device="cuda")
        k0, v0, extra = pools.k_cache, pools.v_cache, (pools.k_scale, pools.v_scale)
        entry, prepare = pa.pa_decode_append_fp8, pa.prepare_decode_append_fp8
    else:
        k0, v0, extra = b.k_cache.cuda(), b.v_cache.cuda(), ()
        entry, prepare = pa.pa_decode_append, pa.prepare_decode_append
    k1, v1, k2, v2 = k0.clone(), v0.clone(), k0.clone(), v0.clone()
    ref, got = torch.empty_like(q), torch.empty_like(q)
    step = prepare(got, q, nk, nv, k2, v2, *extra, bt, cl, b.scale, max_context_len=b.max_context_len)
    g = torch.Generator(device="cuda").manual_seed(1302)
    for _ in range(3):
        entry(ref, q, nk, nv, k1, v1, *extra, bt, cl, b.scale, max_context_len=b.max_context_len)
        step(torch.cuda.current_stream())
        torch.cuda.synchronize()
        assert torch.equal(_bits(got), _bits(ref))
        assert torch.equal(k1, k2) and torch.equal(v1, v2)
        q.copy_(torch.randn(q.shape, generator=g, device="cuda").to(q.dtype))
        nk.copy_(torch.randn(nk.shape, generator=g, device="cuda").to(nk.dtype))
        nv.copy_(torch.randn(nv.shape, generator=g, device="cuda").to(nv.dtype))
    assert pa.pa_get_device_error() == 0
