"""Parity of the CUDA decode path with the oracle (GPU).

Every comparison goes through the C ABI (libpa.so via the binding).  Small
cases compare every output element; the full-size workloads compare seeded
samples of sequences (the oracle computes each sampled sequence from the same
pool contents).  Tolerances: fp32 1e-5 relative; fp16/bf16 2e-2 absolute +
2e-2 relative, plus the per-row rms and ulp figures (check_tolerance)."""

import numpy as np
import pytest
import torch

import oracle
import workloads
import paged_kv_cache_449_b200 as pa
from pagedutil import (as_f64, check_tolerance, device_batch, gpu_decode, materialize_shared,
                       oracle_decode_sampled, permute_physical, relayout_block_size)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.fixture(autouse=True)
def no_device_errors():
    pa.pa_get_device_error()
    yield
    assert pa.pa_get_device_error() == 0


def _full_check(orc, b, modes=("single", "splitk", "splitk2"), parts=(512, 16)):
    ref = oracle_decode_sampled(orc, b, range(b.num_seqs))
    for mode in modes:
        # a partition is a whole number of blocks
        split_parts = sorted(set(max(p, b.block_size) for p in parts))
        for part in (split_parts if mode.startswith("splitk") else (None,)):
            got = gpu_decode(b, mode, partition_size=part or 512)
            check_tolerance(as_f64(got), ref, b.dtype)


SMALL = [
    # dtype, D, B, Hq, Hkv, lens
    (torch.float32, 64, 16, 4, 4, (1, 17, 33, 100)),
    (torch.float32, 128, 8, 8, 1, (0, 5, 9, 64, 3)),
    (torch.float32, 64, 32, 4, 2, (31, 32, 33, 70)),
    (torch.bfloat16, 128, 16, 32, 8, (1, 15, 16, 17, 250)),
    (torch.bfloat16, 128, 8, 8, 4, (0, 1, 7, 8, 9, 130)),
    (torch.bfloat16, 128, 32, 16, 2, (33, 64, 95, 2)),
    (torch.bfloat16, 64, 16, 8, 8, (40, 3, 200)),
    (torch.float16, 128, 16, 64, 8, (300, 12, 1)),
    (torch.float16, 64, 8, 2, 2, (77, 0, 5)),
    (torch.float16, 64, 32, 8, 1, (129, 31)),
]


@pytest.mark.parametrize("case", range(len(SMALL)))
def test_small_cases_every_element(orc, case):
    dt, D, B, Hq, Hkv, lens = SMALL[case]
    b = workloads.random_small(seed=100 + case, dtype=dt, lens=lens, num_q_heads=Hq, num_kv_heads=Hkv,
                               head_dim=D, block_size=B, extra_blocks=9)
    _full_check(orc, b)


@pytest.mark.parametrize("case", range(len(SMALL)))
def test_many_short_sequences_every_element(orc, case):
    # More than 4 CTAs per SM: the one-pass kernel runs its small-CTA shape
    # (several CTAs per SM) instead of one large CTA per SM.
    dt, D, B, Hq, Hkv, _ = SMALL[case]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    S = (4 * sms + 1 + Hkv - 1) // Hkv + 3
    rng = np.random.default_rng(300 + case)
    lens = tuple(int(x) for x in rng.integers(0, 4 * B + 3, size=S))
    b = workloads.random_small(seed=200 + case, dtype=dt, lens=lens, num_q_heads=Hq, num_kv_heads=Hkv,
                               head_dim=D, block_size=B)
    _full_check(orc, b, modes=("single",))


def test_tiny_mha_f32(orc):
    b = workloads.tiny_mha_f32(seed=0)
    _full_check(orc, b, parts=(512, 16, 32))


def _sampled(orc, b, seqs, modes, part=512):
    seqs = sorted(set(int(s) for s in seqs))
    ref = oracle_decode_sampled(orc, b, seqs)
    dev = device_batch(b)
    for mode in modes:
        got = gpu_decode(b, mode, partition_size=part, dev=dev)
        check_tolerance(as_f64(got[seqs]), ref, b.dtype)
        assert torch.isfinite(got.float()).all()


def test_llama3_8b_decode_every_sequence(orc):
    b = workloads.llama3_8b_decode(seed=0, device="cuda")
    _sampled(orc, b, range(b.num_seqs), ("single", "splitk", "splitk2"))


@pytest.mark.parametrize("block_size", [8, 16, 32])
def test_continuous_batching_mix_sampled(orc, block_size):
    b = workloads.continuous_batching_mix(seed=0, device="cuda", block_size=block_size)
    lens = b.context_lens.numpy()
    rng = np.random.default_rng(block_size)
    short = np.nonzero(lens <= 64)[0]
    long = np.nonzero(lens >= 600)[0]
    seqs = list(rng.choice(short, 6, replace=False)) + list(rng.choice(long, 3, replace=False))
    _sampled(orc, b, seqs, ("single", "splitk", "splitk2"))


@pytest.mark.parametrize("prefix_len", [1024, 1000])
def test_prefix_sharing_sampled(orc, prefix_len):
    b = workloads.prefix_sharing(seed=0, device="cuda", prefix_len=prefix_len)
    rng = np.random.default_rng(prefix_len)
    _sampled(orc, b, rng.choice(b.num_seqs, 6, replace=False), ("single", "splitk", "splitk2"))


def test_llama3_70b_long_sampled(orc):
    b = workloads.llama3_70b_long(seed=0, device="cuda")
    lens = b.context_lens.numpy()
    rng = np.random.default_rng(70)
    seqs = [int(lens.argmax()), int(lens.argmin())] + list(rng.choice(b.num_seqs, 8, replace=False))
    _sampled(orc, b, seqs, ("splitk", "splitk2", "single"))


def test_splitk_oracle_form_matches(orc):
    """The GPU split path against the oracle's own partition + LSE-merge form
    at the same partition size (both must equal the plain definition)."""
    b = workloads.random_small(seed=7, dtype=torch.bfloat16, lens=(700, 513, 512, 1, 1500), num_q_heads=16,
                               num_kv_heads=2, head_dim=128, block_size=16)
    ref = oracle_decode_sampled(orc, b, range(b.num_seqs), partition_size=512)
    got = gpu_decode(b, "splitk", partition_size=512)
    check_tolerance(as_f64(got), ref, b.dtype)
