"""Whole-block copies (GPU): copy-on-write duplicates inside one pool pair and
swap-out / swap-in between a device pool pair and a page-locked host pool pair,
compared byte for byte with the oracle's block copy, and attention that is
unchanged (bit for bit) after a block moves and its table entry follows it."""

import pytest
import torch

import oracle
import workloads
import paged_kv_cache_449_b200 as pa
from pagedutil import device_batch, gpu_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


def _bits(t):
    return t.contiguous().view(-1).view(torch.int32 if t.element_size() == 4 else torch.int16)


def _free_blocks(b):
    used = set(int(x) for x in b.block_tables[b.block_tables >= 0].tolist())
    return [i for i in range(b.num_blocks) if i not in used]


CASES = [(torch.bfloat16, 128, 16, 8), (torch.float16, 64, 8, 2), (torch.float32, 64, 32, 4),
         (torch.bfloat16, 64, 32, 1), (torch.float32, 128, 8, 2)]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_copy_on_write_matches_oracle(orc, case):
    dt, D, B, Hkv = CASES[case]
    b = workloads.random_small(seed=400 + case, dtype=dt, lens=(3 * B + 1, B, 5), num_q_heads=Hkv,
                               num_kv_heads=Hkv, head_dim=D, block_size=B, extra_blocks=12)
    free = _free_blocks(b)
    used = [int(x) for x in b.block_tables[b.block_tables >= 0].tolist()]
    pairs = torch.tensor([[s, d] for s, d in zip(used, free)], dtype=torch.int64)
    k, v = b.k_cache.cuda().contiguous(), b.v_cache.cuda().contiguous()
    pa.pa_get_device_error()
    pa.pa_copy_blocks(k, v, k, v, pairs.cuda())
    torch.cuda.synchronize()
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    orc.copy_blocks(kc, vc, kc, vc, pairs, B)
    assert torch.equal(_bits(k.cpu()), _bits(kc)) and torch.equal(_bits(v.cpu()), _bits(vc))
    assert pa.pa_get_device_error() == 0


@pytest.mark.parametrize("case", range(len(CASES)))
def test_swap_out_and_back_in(orc, case):
    dt, D, B, Hkv = CASES[case]
    b = workloads.random_small(seed=410 + case, dtype=dt, lens=(4 * B + 3, 2 * B, 7), num_q_heads=2 * Hkv,
                               num_kv_heads=Hkv, head_dim=D, block_size=B, extra_blocks=10)
    dev = device_batch(b)
    before = gpu_decode(b, "single", dev=dev)
    s = 0
    nblk = (int(b.context_lens[s]) + B - 1) // B
    ids = [int(x) for x in b.block_tables[s, :nblk]]
    host_k = torch.zeros((nblk,) + tuple(b.k_cache.shape[1:]), dtype=dt).pin_memory()
    host_v = torch.zeros_like(host_k).pin_memory()
    out_map = torch.tensor([[i, j] for j, i in enumerate(ids)], dtype=torch.int64)
    pa.pa_get_device_error()
    pa.pa_copy_blocks(host_k, host_v, dev["k_cache"], dev["v_cache"], out_map.cuda())
    torch.cuda.synchronize()
    ok_k, ok_v = torch.zeros_like(host_k), torch.zeros_like(host_v)
    orc.copy_blocks(ok_k, ok_v, b.k_cache.contiguous(), b.v_cache.contiguous(), out_map, B)
    assert torch.equal(_bits(host_k), _bits(ok_k)) and torch.equal(_bits(host_v), _bits(ok_v))
    # the swapped-out blocks are reused; the sequence comes back into other free blocks
    dev["k_cache"][ids] = 0
    dev["v_cache"][ids] = 0
    free = _free_blocks(b)[:nblk]
    in_map = torch.tensor([[j, f] for j, f in enumerate(free)], dtype=torch.int64).pin_memory()
    pa.pa_copy_blocks(dev["k_cache"], dev["v_cache"], host_k, host_v, in_map)   # mapping read from host memory
    tables = b.block_tables.clone()
    tables[s, :nblk] = torch.tensor(free, dtype=torch.int32)
    dev["block_tables"] = tables.cuda()
    after = gpu_decode(b, "single", dev=dev)
    assert torch.equal(_bits(after[s]), _bits(before[s]))
    assert pa.pa_get_device_error() == 0


def test_out_of_range_pair_is_flagged_and_skipped():
    b = workloads.random_small(seed=420, dtype=torch.bfloat16, lens=(40, 20), num_q_heads=4, num_kv_heads=2,
                               head_dim=128, block_size=16, extra_blocks=4)
    k, v = b.k_cache.cuda().contiguous(), b.v_cache.cuda().contiguous()
    k0, v0 = k.clone(), v.clone()
    free = _free_blocks(b)
    pairs = torch.tensor([[b.num_blocks, free[0]], [0, -1], [-3, free[1]]], dtype=torch.int64, device="cuda")
    pa.pa_get_device_error()
    pa.pa_copy_blocks(k, v, k, v, pairs)
    assert pa.pa_get_device_error() & pa.DEVERR_BLOCK_ID
    assert torch.equal(_bits(k), _bits(k0)) and torch.equal(_bits(v), _bits(v0))


def test_unpinned_host_pool_is_refused():
    b = workloads.random_small(seed=421, dtype=torch.float16, lens=(16,), num_q_heads=2, num_kv_heads=2,
                               head_dim=64, block_size=16, extra_blocks=2)
    k, v = b.k_cache.cuda().contiguous(), b.v_cache.cuda().contiguous()
    host = torch.zeros_like(b.k_cache)   # pageable
    with pytest.raises(ValueError):
        pa.pa_copy_blocks(host, host, k, v, torch.tensor([[0, 0]], dtype=torch.int64, device="cuda"))


@pytest.mark.parametrize("prefix_len", [1024, 1000])
def test_materialising_a_shared_prefix_by_copy_is_bit_exact(prefix_len):
    """Every sequence gets private copies of the shared prefix blocks (what a
    write into a shared block forces): attention is unchanged bit for bit."""
    b = workloads.prefix_sharing(seed=430, prefix_len=prefix_len, num_seqs=12, suffix_range=(16, 96))
    n_full = prefix_len // b.block_size
    spare = n_full * b.num_seqs
    x = b.k_cache.shape
    k = torch.cat([b.k_cache, torch.zeros((spare,) + tuple(x[1:]), dtype=b.k_cache.dtype)]).cuda().contiguous()
    v = torch.cat([b.v_cache, torch.zeros((spare,) + tuple(x[1:]), dtype=b.v_cache.dtype)]).cuda().contiguous()
    shared = [int(t) for t in b.block_tables[0, :n_full]]
    tables = b.block_tables.clone()
    pairs, nxt = [], b.num_blocks
    for s in range(b.num_seqs):
        for j, src in enumerate(shared):
            pairs.append([src, nxt])
            tables[s, j] = nxt
            nxt += 1
    dev = device_batch(b)
    ref = gpu_decode(b, "single", dev=dev)
    pa.pa_get_device_error()
    pa.pa_copy_blocks(k, v, k, v, torch.tensor(pairs, dtype=torch.int64, device="cuda"))
    dev.update(k_cache=k, v_cache=v, block_tables=tables.cuda())
    c = b.__class__(**{**b.__dict__, "num_blocks": nxt})
    got = gpu_decode(c, "single", dev=dev)
    assert torch.equal(_bits(got), _bits(ref))
    assert pa.pa_get_device_error() == 0
