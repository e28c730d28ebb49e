"""pa_decode_splitk_static: split-K decode for callers that cannot allocate
device memory when they launch work (runtime plugins handed only their inputs
and outputs, latency-critical loops that must not trigger cudaMalloc's
implicit synchronisation).  Its partials live in a fixed array inside the
library's device image instead of a caller-provided workspace.

The GPU test calls it through the C ABI twice in a row, on two different
batches.  Each output must equal, bit for bit, the existing pa_decode_splitk
entry point run in the same (two-kernel) form on the same inputs, and must
match the oracle within the bf16 tolerance the other tests use; the second
call runs over whatever the first left in the shared array.  A small fp32
case is compared with the oracle at the fp32 tolerance.  This file is
collected last so a run that stops at the first failure has already run every
other test."""

import ctypes

import pytest
import torch

import oracle
import workloads
import paged_kv_cache_449_b200 as pa
from paged_kv_cache_449_b200 import build as pabuild
from pagedutil import as_f64, check_tolerance, device_batch, oracle_decode_sampled


@pytest.fixture(scope="module")
def lib():
    pabuild.build()
    return pa.load()


def _existing(b, dev, part):
    out = torch.empty_like(dev["q"])
    pa.pa_decode_splitk(out, dev["q"], dev["k_cache"], dev["v_cache"], dev["block_tables"], dev["context_lens"],
                        b.scale, b.max_context_len, partition_size=part, fused=False)
    return out


def _static(b, dev, part):
    out = torch.full_like(dev["q"], float("nan"))
    pa.pa_decode_splitk_static(out, dev["q"], dev["k_cache"], dev["v_cache"], dev["block_tables"],
                               dev["context_lens"], b.scale, b.max_context_len, partition_size=part)
    return out


@pytest.mark.gpu
def test_static_scratch_matches_existing_entry_on_two_calls(lib):
    orc = oracle.default()
    first = workloads.llama3_8b_decode(seed=11, device="cuda", num_seqs=32, num_blocks=8192)
    second = workloads.continuous_batching_mix(seed=12, device="cuda", num_seqs=96, block_size=8)
    pa.pa_get_device_error()
    for b, part in ((first, 256), (second, 512)):
        need = pa.pa_decode_splitk_workspace_size(b.num_seqs, b.num_q_heads, b.head_dim, b.max_context_len, part)
        assert need <= pa.SPLITK_STATIC_SCRATCH_BYTES
        dev = device_batch(b)
        got = _static(b, dev, part)
        ref = _existing(b, dev, part)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
        seqs = [0, 1, int(b.context_lens.argmax()), b.num_seqs - 1]
        check_tolerance(as_f64(got[seqs]), oracle_decode_sampled(orc, b, seqs), b.dtype)
    assert pa.pa_get_device_error() == 0


@pytest.mark.gpu
def test_static_scratch_fp32_against_oracle(lib):
    b = workloads.random_small(seed=13, dtype=torch.float32, lens=(1, 40, 333, 0, 97), num_q_heads=8,
                               num_kv_heads=2, head_dim=64, block_size=16)
    dev = device_batch(b)
    ref = oracle_decode_sampled(oracle.default(), b, range(b.num_seqs))
    for _ in range(2):
        got = _static(b, dev, 32)
        torch.cuda.synchronize()
        check_tolerance(as_f64(got), ref, b.dtype)
    assert pa.pa_get_device_error() == 0


def _size_args(num_seqs, max_context_len, out_ptr):
    # head_dim 64, one query head per kv head, 16-token blocks and partitions:
    # the partials need num_seqs * ceil(max_context_len / 16) * (64 + 2) * 4 bytes.
    return [out_ptr, 16, 16, 16, 16, 16, ctypes.c_float(0.125), 16, num_seqs, 1, 1, 64,
            (max_context_len + 15) // 16, max_context_len, 1 << 20, 2, 16, None]


def test_static_scratch_refuses_requests_beyond_its_size(lib):
    # Refused on the host before any device work, so this runs without a GPU.
    # 64 seqs x 64 q heads x ceil(32768/512) = 64 partitions x 130 floats x 4 B = 136 MB.
    args = [16, 16, 16, 16, 16, 16, ctypes.c_float(0.088), 16, 64, 64, 8, 128, 2048, 32768, 100000, 2, 512, None]
    assert lib.pa_decode_splitk_static(*args) == 3  # PA_ERR_WORKSPACE
    # The size limit itself: with 50 sequences, 1271 partitions fit the array
    # and 1272 do not.  The binding's constant is the header's.
    per_partition = 50 * (64 + 2) * 4
    assert 1271 * per_partition <= pa.SPLITK_STATIC_SCRATCH_BYTES < 1272 * per_partition
    assert lib.pa_decode_splitk_static(*_size_args(50, 1272 * 16, 16)) == 3
    # The largest request that fits passes the size check.  Its `out` pointer
    # is misaligned, so it is refused later, by the argument checks, before any
    # launch: PA_ERR_INVALID_ARG with a GPU, PA_ERR_CUDA without one (no
    # device to look the array up on).
    assert lib.pa_decode_splitk_static(*_size_args(50, 1271 * 16, 17)) in (1, 4)
