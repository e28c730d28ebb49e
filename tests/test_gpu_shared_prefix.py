"""Parity of the shared-prefix decode (pa_decode_shared_prefix) with the
oracle (GPU).

Every row of a batch begins with the same physical blocks (a system prompt
shared by reference, "vLLM核心架构总览" §4.1 comparison table; "vLLM框架解析"
§2.3).  The entry attends that prefix once per kv head for all sequences (a
tensor-core pass) and each sequence's own blocks in a decode pass, and merges
the two; the result must be the oracle's plain decode of each sequence over
its whole context, within the 16-bit tolerance.  The appending form must also
leave the pools bit-identical to pa_decode_append's."""

import numpy as np
import pytest
import torch

import oracle
import workloads
import paged_kv_cache_449_b200 as pa
from pagedutil import as_f64, check_tolerance, device_batch, oracle_decode_sampled

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.fixture(autouse=True)
def no_device_errors():
    pa.pa_get_device_error()
    yield
    assert pa.pa_get_device_error() == 0


def _bits(t):
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


def _batch(seed, dtype, D, B, Hq, Hkv, prefix_blocks, suffix_lens):
    return workloads.prefix_sharing(seed=seed, device="cuda", prefix_len=prefix_blocks * B,
                                    num_seqs=len(suffix_lens), block_size=B, dtype=dtype, num_q_heads=Hq,
                                    num_kv_heads=Hkv, head_dim=D, suffix_lens=suffix_lens)


def _dev(b):
    """Device copies of the batch's tensors, pools included (the GPU's writes
    must not reach the pools the oracle reads)."""
    d = device_batch(b)
    d["k_cache"], d["v_cache"] = d["k_cache"].clone(), d["v_cache"].clone()
    return d


def _shared_prefix(b, dev, append, ref_counts=None, prefix_blocks=None):
    out = torch.full_like(dev["q"], float("nan"))
    key = b.new_key.cuda().contiguous() if append else None
    value = b.new_value.cuda().contiguous() if append else None
    pa.pa_decode_shared_prefix(out, dev["q"], key, value, dev["k_cache"], dev["v_cache"], dev["block_tables"],
                               dev["context_lens"], b.scale,
                               b.meta["shared_blocks"] if prefix_blocks is None else prefix_blocks,
                               max_context_len=b.max_context_len, ref_counts=ref_counts)
    torch.cuda.synchronize()
    return out


def _written(orc, b):
    """The batch after the oracle's write of each sequence's newest token."""
    kc, vc = b.k_cache.cpu().contiguous(), b.v_cache.cpu().contiguous()
    orc.reshape_and_cache(b.new_key.cpu().contiguous(), b.new_value.cpu().contiguous(), kc, vc, b.slot_mapping,
                          b.block_size)
    return b.__class__(**{**b.__dict__, "k_cache": kc, "v_cache": vc})


# dtype, D, B, Hq, Hkv, prefix blocks, sequences, suffix range: query rows span
# one to three CTAs of two 128-row tiles with a ragged last tile; prefixes of
# one to many 64-key tiles, ending inside a tile or on its edge
SMALL = [
    (torch.bfloat16, 128, 16, 32, 8, 5, 70, (1, 100)),      # group 4: 32 sequences per tile
    (torch.float16, 64, 8, 8, 8, 24, 300, (1, 40)),         # group 1: 128 per tile, 3 tiles of 64 keys
    (torch.bfloat16, 128, 32, 16, 2, 9, 40, (1, 90)),       # group 8: 16 per tile, prefix ends mid-tile
    (torch.float16, 128, 16, 4, 2, 1, 9, (1, 33)),          # a one-block prefix
    (torch.bfloat16, 64, 16, 8, 4, 64, 130, (1, 200)),      # 16 tiles of keys
    (torch.float16, 128, 8, 32, 8, 13, 33, (1, 70)),        # 8-token blocks, 104-key prefix
    (torch.bfloat16, 128, 16, 8, 2, 128, 3, (1, 50)),       # few sequences, long prefix: 16 key partitions
    (torch.float16, 64, 32, 4, 2, 40, 5, (1, 100)),         # 20 key partitions of one tile each
    (torch.bfloat16, 128, 16, 8, 1, 7, 1, (1, 30)),         # one sequence, one kv head
    (torch.float16, 128, 16, 8, 8, 3, 700, (1, 20)),        # group 1: three row CTAs, 188 rows in the last tile
]


@pytest.mark.parametrize("case", range(len(SMALL)))
@pytest.mark.parametrize("append", [False, True])
def test_small_cases_every_element(orc, case, append):
    dt, D, B, Hq, Hkv, P, S, (lo, hi) = SMALL[case]
    rng = np.random.default_rng(4100 + case)
    suffix = rng.integers(lo, hi, size=S, endpoint=True)
    if not append:
        suffix[rng.choice(S, min(3, S), replace=False)] = 0   # contexts that end with the prefix
    b = _batch(4000 + case, dt, D, B, Hq, Hkv, P, suffix)
    dev = _dev(b)
    got = _shared_prefix(b, dev, append)
    ref_b = _written(orc, b) if append else b
    check_tolerance(as_f64(got), oracle_decode_sampled(orc, ref_b, range(S)), dt)


@pytest.mark.parametrize("append", [False, True])
def test_prefix_sharing_workload_sampled(orc, append):
    """The 128-sequence, 1024-token-prefix workload: sampled sequences
    against the oracle, and the pools against pa_decode_append's."""
    b = workloads.prefix_sharing(seed=0, device="cuda")
    d1, d2 = _dev(b), _dev(b)
    got = _shared_prefix(b, d2, append)
    seqs = sorted(set([int(b.context_lens.argmax()), int(b.context_lens.argmin())] +
                      [int(x) for x in np.random.default_rng(41).choice(b.num_seqs, 8, replace=False)]))
    ref_b = _written(orc, b) if append else b
    check_tolerance(as_f64(got[seqs]), oracle_decode_sampled(orc, ref_b, seqs), b.dtype)
    assert torch.isfinite(got.float()).all()
    if append:
        out = torch.empty_like(d1["q"])
        pa.pa_decode_append(out, d1["q"], b.new_key.cuda(), b.new_value.cuda(), d1["k_cache"], d1["v_cache"],
                            d1["block_tables"], d1["context_lens"], b.scale, max_context_len=b.max_context_len)
        torch.cuda.synchronize()
        assert torch.equal(_bits(d2["k_cache"]), _bits(d1["k_cache"]))
        assert torch.equal(_bits(d2["v_cache"]), _bits(d1["v_cache"]))
        check_tolerance(as_f64(got), as_f64(out), b.dtype)


def test_a_shorter_shared_prefix_gives_the_same_attention(orc):
    """Declaring fewer shared blocks than the rows share moves blocks from the
    prefix pass to the decode pass; the attention stays the oracle's."""
    b = _batch(4200, torch.bfloat16, 128, 16, 32, 8, 12, np.arange(1, 41))
    dev = _dev(b)
    ref = oracle_decode_sampled(orc, b, range(b.num_seqs))
    for P in (1, 4, 11, 12):
        check_tolerance(as_f64(_shared_prefix(b, dev, False, prefix_blocks=P)), ref, b.dtype)


def test_prepared_call_repeats_the_entry():
    b = _batch(4300, torch.float16, 128, 16, 32, 8, 20, np.arange(5, 69))
    d1, d2 = _dev(b), _dev(b)
    nk, nv = b.new_key.cuda().contiguous(), b.new_value.cuda().contiguous()
    ref, got = torch.empty_like(d1["q"]), torch.empty_like(d2["q"])
    step = pa.prepare_decode_shared_prefix(got, d2["q"], nk, nv, d2["k_cache"], d2["v_cache"], d2["block_tables"],
                                           d2["context_lens"], b.scale, 20, max_context_len=b.max_context_len)
    for _ in range(2):
        pa.pa_decode_shared_prefix(ref, d1["q"], nk, nv, d1["k_cache"], d1["v_cache"], d1["block_tables"],
                                   d1["context_lens"], b.scale, 20, max_context_len=b.max_context_len)
        step()
        torch.cuda.synchronize()
        assert torch.equal(_bits(got), _bits(ref))
        assert torch.equal(d1["k_cache"], d2["k_cache"]) and torch.equal(d1["v_cache"], d2["v_cache"])


def test_a_row_with_another_prefix_is_flagged(orc):
    """A row whose first blocks differ from row 0's sets DEVERR_PREFIX; the
    other rows keep the oracle's attention."""
    b = _batch(4400, torch.bfloat16, 128, 16, 32, 8, 6, np.arange(3, 43))
    dev = _dev(b)
    spare = int(dev["block_tables"][5, 6])   # a block of row 5's own
    dev["block_tables"][9, 2] = spare
    pa.pa_get_device_error()
    got = _shared_prefix(b, dev, False)
    assert pa.pa_get_device_error() & pa.DEVERR_PREFIX
    keep = [s for s in range(b.num_seqs) if s != 9]
    check_tolerance(as_f64(got[keep]), oracle_decode_sampled(orc, b, keep), b.dtype)


def test_a_context_inside_the_prefix_is_refused(orc):
    """A context that does not reach past the prefix when appending (the
    newest token would land in a shared block) sets DEVERR_CONTEXT_LEN and
    gets a zero row; the pools are not written for it."""
    b = _batch(4500, torch.float16, 64, 16, 8, 2, 4, np.arange(1, 21))
    dev = _dev(b)
    dev["context_lens"][3] = 4 * 16           # exactly the prefix
    k0, v0 = dev["k_cache"].clone(), dev["v_cache"].clone()
    pa.pa_get_device_error()
    got = _shared_prefix(b, dev, True)
    assert pa.pa_get_device_error() & pa.DEVERR_CONTEXT_LEN
    assert torch.count_nonzero(got[3]) == 0
    prefix_ids = dev["block_tables"][0, :4].long()
    assert torch.equal(dev["k_cache"][prefix_ids], k0[prefix_ids])
    assert torch.equal(dev["v_cache"][prefix_ids], v0[prefix_ids])
    keep = [s for s in range(b.num_seqs) if s != 3]
    c = _written(orc, b)
    check_tolerance(as_f64(got[keep]), oracle_decode_sampled(orc, c, keep), b.dtype)


def test_host_side_refusals():
    b = _batch(4600, torch.bfloat16, 128, 16, 32, 8, 4, np.arange(1, 9))
    dev = _dev(b)
    out = torch.empty_like(dev["q"])
    args = (out, dev["q"], None, None, dev["k_cache"], dev["v_cache"], dev["block_tables"], dev["context_lens"],
            b.scale)
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_decode_shared_prefix(*args, 4, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 3
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_decode_shared_prefix(*args, 0)
    assert e.value.status == 1
    with pytest.raises(ValueError):
        pa.pa_decode_shared_prefix(out, dev["q"], b.new_key.cuda(), None, *args[4:], 4)


def test_a_shared_newest_block_is_not_written(orc):
    """With reference counts given, a sequence whose newest token's block is
    also another sequence's (a table that skipped copy-on-write) is not
    written and sets DEVERR_SHARED_BLOCK, as with pa_decode_append; the other
    sequences are written and attended as usual."""
    b = _batch(4700, torch.bfloat16, 128, 16, 8, 2, 4, [5, 5, 20])
    bt = b.block_tables.clone()
    bt[1, 4] = bt[0, 4]                       # sequence 1's own block aliases sequence 0's
    counts = torch.zeros(b.num_blocks, dtype=torch.int32)
    for s in range(b.num_seqs):
        for j in range((int(b.context_lens[s]) + 15) // 16):
            counts[int(bt[s, j])] += 1
    c = b.__class__(**{**b.__dict__, "block_tables": bt})
    dev = _dev(c)
    k0 = dev["k_cache"].clone()
    pa.pa_get_device_error()
    got = _shared_prefix(c, dev, True, ref_counts=counts.cuda())
    assert pa.pa_get_device_error() & pa.DEVERR_SHARED_BLOCK
    shared = int(bt[0, 4])
    assert torch.equal(dev["k_cache"][shared], k0[shared])        # the shared block is untouched
    kc, vc = b.k_cache.cpu().clone(), b.v_cache.cpu().clone()
    slots = torch.tensor([-1, -1, int(b.slot_mapping[2])], dtype=torch.int64)
    orc.reshape_and_cache(b.new_key.cpu(), b.new_value.cpu(), kc, vc, slots, 16)
    ref = orc.decode(b.q.cpu(), kc, vc, bt, b.context_lens, b.scale, 16, b.num_kv_heads)
    check_tolerance(as_f64(got), ref, b.dtype)      # 0 and 1 attend over the pool as it was
