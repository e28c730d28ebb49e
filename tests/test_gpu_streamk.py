"""The work-balanced (stream-K) decode on shapes that stress its schedule:
one long sequence cut into hundreds of pieces, fewer tiles than warps,
empty sequences between full ones, and the arrival counters it must leave
at zero (GPU)."""

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


def _run(b, ws):
    dev = device_batch(b)
    out = torch.full_like(dev["q"], float("nan"))
    pa.pa_decode_streamk(out, dev["q"], dev["k_cache"], dev["v_cache"], dev["block_tables"], dev["context_lens"],
                         b.scale, max_context_len=b.max_context_len, workspace=ws)
    torch.cuda.synchronize()
    return out


def _counters_zero(b, ws):
    return bool((ws.counters == 0).all())


CASES = [
    # one long sequence over every warp: hundreds of pieces merged
    dict(dtype=torch.bfloat16, lens=(9000,), Hq=8, Hkv=1, D=128, B=16),
    dict(dtype=torch.float16, lens=(4100,), Hq=4, Hkv=4, D=64, B=8),
    # fewer tiles than warps
    dict(dtype=torch.bfloat16, lens=(3, 1, 17), Hq=4, Hkv=2, D=128, B=16),
    # empty sequences interleaved with long and short ones
    dict(dtype=torch.bfloat16, lens=(0, 700, 0, 0, 5, 1300, 0), Hq=32, Hkv=8, D=128, B=32),
    dict(dtype=torch.float32, lens=(0, 333, 17, 1000), Hq=8, Hkv=2, D=128, B=16),
    dict(dtype=torch.float32, lens=(65, 2, 640), Hq=2, Hkv=1, D=64, B=32),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_streamk_against_oracle_and_counters(orc, case):
    c = CASES[case]
    b = workloads.random_small(seed=200 + case, dtype=c["dtype"], lens=c["lens"], num_q_heads=c["Hq"],
                               num_kv_heads=c["Hkv"], head_dim=c["D"], block_size=c["B"], extra_blocks=4)
    ws = pa.StreamKWorkspace()
    ref = oracle_decode_sampled(orc, b, range(b.num_seqs))
    first = _run(b, ws)
    check_tolerance(as_f64(first), ref, b.dtype)
    assert _counters_zero(b, ws)
    again = _run(b, ws)                      # the same workspace, reused
    assert torch.equal(first.view(torch.uint8), again.view(torch.uint8))
    assert _counters_zero(b, ws)
    assert pa.pa_get_device_error() == 0


def test_streamk_mix_reuses_workspace_across_batches(orc):
    ws = pa.StreamKWorkspace()
    for seed in range(3):
        b = workloads.continuous_batching_mix(seed=seed, device="cuda", num_seqs=48, block_size=(8, 16, 32)[seed])
        got = _run(b, ws)
        seqs = list(range(0, 48, 5))
        check_tolerance(as_f64(got[seqs]), oracle_decode_sampled(orc, b, seqs), b.dtype)
        assert _counters_zero(b, ws)
