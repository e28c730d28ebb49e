"""Chunked prefill on the GPU against the oracle's causal prefill (every
element), across dtypes, head dims, block sizes, GQA groups and chunk shapes
(single-token chunks, whole-context chunks, ragged chunks); single-token
chunks against the decode kernel; malformed chunks flagged on the device."""

import numpy as np
import pytest
import torch

import oracle
import workloads
import paged_kv_cache_449_b200 as pa
from pagedutil import as_f64, check_tolerance, device_batch, gpu_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.fixture(autouse=True)
def no_device_errors():
    pa.pa_get_device_error()
    yield
    assert pa.pa_get_device_error() == 0


def _gpu_prefill(b, qs=None):
    qs = b.meta["query_start"] if qs is None else qs
    dev = device_batch(b)
    out = torch.full_like(dev["q"], float("nan"))
    Q = (qs[1:] - qs[:-1]).max().item() if qs.numel() > 1 else 0
    pa.pa_prefill(out, dev["q"], dev["k_cache"], dev["v_cache"], dev["block_tables"], dev["context_lens"],
                  qs.cuda(), b.scale, max_context_len=b.max_context_len, max_query_len=int(Q))
    torch.cuda.synchronize()
    return out


CASES = [
    # dtype, D, B, Hq, Hkv, context range, chunk range
    (torch.bfloat16, 128, 16, 32, 8, (1, 90), (1, 90)),
    (torch.bfloat16, 128, 8, 8, 8, (20, 70), (10, 70)),
    (torch.float16, 64, 32, 16, 2, (30, 130), (1, 40)),
    (torch.float16, 128, 16, 8, 1, (40, 80), (33, 80)),
    (torch.bfloat16, 64, 8, 4, 2, (1, 50), (1, 5)),
    (torch.bfloat16, 64, 32, 8, 4, (60, 200), (60, 200)),
    (torch.bfloat16, 128, 32, 16, 4, (100, 300), (20, 200)),
    (torch.float16, 128, 32, 32, 8, (64, 64), (64, 64)),
    (torch.float16, 64, 8, 8, 2, (30, 150), (5, 100)),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_prefill_every_element(orc, case):
    dt, D, B, Hq, Hkv, ctx, chunk = CASES[case]
    b = workloads.chunked_prefill(seed=1000 + case, dtype=dt, num_seqs=5, num_q_heads=Hq, num_kv_heads=Hkv,
                                  head_dim=D, block_size=B, context_range=ctx, chunk_range=chunk)
    ref = orc.prefill(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.meta["query_start"], b.scale,
                      B, Hkv)
    got = _gpu_prefill(b)
    check_tolerance(as_f64(got), ref, dt)


@pytest.mark.parametrize("block_size", [16, 8, 32])
def test_prefill_llama3_8b_shape(orc, block_size):
    """Llama-3-8B heads, every element, at each pool block size (8-token blocks
    pair two V tiles per MMA step; 32-token blocks gather two chunks per load)."""
    b = workloads.chunked_prefill(seed=1010, num_seqs=4, context_range=(512, 1024), chunk_range=(64, 256),
                                  block_size=block_size)
    ref = orc.prefill(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.meta["query_start"], b.scale,
                      b.block_size, b.num_kv_heads)
    got = _gpu_prefill(b)
    check_tolerance(as_f64(got), ref, b.dtype)
    assert torch.isfinite(got.float()).all()


def test_single_token_chunks_match_decode():
    b = workloads.llama3_8b_decode(seed=1020, num_seqs=12, num_blocks=2048)
    qs = torch.arange(b.num_seqs + 1, dtype=torch.int32)
    pre = _gpu_prefill(b, qs)
    dec = gpu_decode(b, "single")
    check_tolerance(as_f64(pre), as_f64(dec), b.dtype)


def test_chunk_longer_than_context_is_flagged():
    b = workloads.random_small(seed=1030, dtype=torch.bfloat16, lens=(10, 20), num_q_heads=4, num_kv_heads=2,
                               head_dim=64, block_size=16)
    qs = torch.tensor([0, 12, 14], dtype=torch.int32)   # 12 queries over a 10-token context
    b.q = torch.randn((14, 4, 64)).to(torch.bfloat16)
    pa.pa_get_device_error()
    out = _gpu_prefill(b, qs)
    assert pa.pa_get_device_error() & pa.DEVERR_CONTEXT_LEN
    assert torch.isnan(out[:12].float()).all()        # sequence 0 left unwritten
    assert torch.isfinite(out[12:].float()).all()


@pytest.mark.parametrize("block_size", [16, 8, 32])
def test_refused_block_ids_are_flagged_and_masked(orc, block_size):
    """Block ids outside the pool (negative, or past its end) are flagged and
    never fetched: a whole key tile of them (no block of the tile fetchable),
    and a single one among fetchable blocks (with 8-token blocks, the partner
    of a fetchable block in one 16-key MMA step).  Untouched sequences still
    match the oracle; rows of the damaged sequences stay finite."""
    b = workloads.chunked_prefill(seed=1040, num_seqs=3, context_range=(200, 400), chunk_range=(40, 150),
                                  block_size=block_size)
    ref = orc.prefill(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.meta["query_start"], b.scale,
                      b.block_size, b.num_kv_heads)
    bad = b.block_tables.clone()
    per_tile = 64 // b.block_size
    bad[1, :per_tile] = -7                       # the first 64-key tile of sequence 1: nothing to fetch
    bad[2, per_tile + 1] = b.num_blocks + 3      # one block of sequence 2's second key tile
    b.block_tables = bad
    pa.pa_get_device_error()
    got = _gpu_prefill(b)
    assert pa.pa_get_device_error() & pa.DEVERR_BLOCK_ID
    qs = b.meta["query_start"]
    s0 = slice(int(qs[0]), int(qs[1]))
    check_tolerance(as_f64(got[s0]), ref[s0], b.dtype)
    assert torch.isfinite(got.float()).all()


def test_empty_chunk_between_sequences(orc):
    """A sequence with no new tokens (query_start repeats) launches nothing for
    itself and leaves its neighbours exact."""
    b = workloads.chunked_prefill(seed=1050, num_seqs=3, context_range=(150, 300), chunk_range=(30, 90))
    qs = b.meta["query_start"]
    n0, n2 = int(qs[1] - qs[0]), int(qs[3] - qs[2])
    b.q = torch.cat([b.q[: n0], b.q[int(qs[2]):]]).contiguous()
    new_qs = torch.tensor([0, n0, n0, n0 + n2], dtype=torch.int32)
    ref = orc.prefill(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, new_qs, b.scale, b.block_size,
                      b.num_kv_heads)
    got = _gpu_prefill(b, new_qs)
    check_tolerance(as_f64(got), ref, b.dtype)


@pytest.mark.parametrize("qmul", [6.0, 0.01])
def test_prefill_peaked_and_flat_scores(orc, qmul):
    """Queries scaled so that scores span many powers of two (the softmax
    reference moves often, P reaches 2^8 and tiny values) or almost none (a
    flat softmax over the whole context)."""
    b = workloads.chunked_prefill(seed=1060, num_seqs=3, context_range=(300, 600), chunk_range=(50, 200))
    b.q = (b.q.float() * qmul).to(b.dtype).contiguous()
    ref = orc.prefill(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.meta["query_start"], b.scale,
                      b.block_size, b.num_kv_heads)
    got = _gpu_prefill(b)
    check_tolerance(as_f64(got), ref, b.dtype)
