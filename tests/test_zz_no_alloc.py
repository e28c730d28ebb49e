"""pa_decode_splitk_static: split-K decode for callers that cannot allocate
device memory when they launch work (runtime plugins handed only their inputs
and outputs, latency-critical loops that must not trigger cudaMalloc's
implicit synchronisation).  Its partials live in a fixed array inside the
library's device image instead of a caller-provided workspace.

The GPU test calls it through the C ABI twice in a row, on two different
batches, and checks each output against the existing pa_decode_splitk entry
point within the bf16 tolerance the other tests use; the second call runs over
whatever the first left in the shared array.  This file is collected last so a
run that stops at the first failure has already run every other test."""

import ctypes

import pytest
import torch

import workloads
import paged_kv_cache_449_b200 as pa
from pagedutil import as_f64, check_tolerance, device_batch


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
def test_static_scratch_matches_existing_entry_on_two_calls():
    first = workloads.llama3_8b_decode(seed=11, device="cuda", num_seqs=32, num_blocks=8192)
    second = workloads.continuous_batching_mix(seed=12, device="cuda", num_seqs=96, block_size=8)
    for b, part in ((first, 256), (second, 512)):
        need = pa.pa_decode_splitk_workspace_size(b.num_seqs, b.num_q_heads, b.head_dim, b.max_context_len, part)
        assert need <= pa.SPLITK_STATIC_SCRATCH_BYTES
        dev = device_batch(b)
        got = _static(b, dev, part)
        ref = _existing(b, dev, part)
        torch.cuda.synchronize()
        check_tolerance(as_f64(got), as_f64(ref), b.dtype)
    assert pa.pa_get_device_error() == 0


def test_static_scratch_refuses_requests_beyond_its_size():
    # 64 seqs x 64 q heads x ceil(32768/512)=64 partitions x 130 floats x 4 B = 136 MB > 16 MiB.
    # Refused on the host before any device work, so this runs without a GPU.
    lib = pa.load()
    args = [16, 16, 16, 16, 16, 16, ctypes.c_float(0.088), 16, 64, 64, 8, 128, 2048, 32768, 100000, 2, 512, None]
    assert lib.pa_decode_splitk_static(*args) == 3  # PA_ERR_WORKSPACE
