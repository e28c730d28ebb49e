"""The 16-bit parity bar itself (CPU): the per-row rms and ulp figures that
check_tolerance asserts beside the stated 2e-2 bound must pass a result that
differs from the oracle only by rounding, and must fail a plausible
arithmetic slip that the 2e-2 bound lets through: a split-K merge that drops
one of 32 partitions of a long context.  The slip is planted in the oracle's
result on the CPU (its decode over the context with that partition's blocks
left out), never in a kernel."""

import numpy as np
import pytest
import torch

import oracle
import workloads
from pagedutil import check_tolerance, clone_batch, parity_figures

PART = 512


@pytest.fixture(scope="module")
def long_case():
    # one sequence, 32 full partitions of 512 tokens plus a ragged tail
    b = workloads.random_small(seed=41, dtype=torch.bfloat16, lens=(32 * PART + 100,), num_q_heads=8,
                               num_kv_heads=1, head_dim=128, block_size=16, extra_blocks=0)
    orc = oracle.default()
    ref = orc.decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale, b.block_size,
                     b.num_kv_heads)
    return b, orc, ref


def _rounded(x: np.ndarray, dtype) -> np.ndarray:
    return torch.from_numpy(x).to(dtype).double().numpy()


def test_rounding_alone_passes(long_case):
    b, _, ref = long_case
    check_tolerance(_rounded(ref, torch.bfloat16), ref, torch.bfloat16)
    check_tolerance(_rounded(ref, torch.float16), ref, torch.float16)


@pytest.mark.parametrize("dropped", [0, 13, 31])
def test_a_dropped_partition_fails_the_bar(long_case, dropped):
    b, orc, ref = long_case
    per = PART // b.block_size
    row = b.block_tables[0].clone()
    kept = torch.cat([row[:dropped * per], row[(dropped + 1) * per:], torch.full((per,), -1, dtype=row.dtype)])
    slip = clone_batch(b, block_tables=kept[None, :].contiguous(),
                       context_lens=b.context_lens - PART)
    wrong = orc.decode(slip.q, slip.k_cache, slip.v_cache, slip.block_tables, slip.context_lens, slip.scale,
                       slip.block_size, slip.num_kv_heads)
    got = _rounded(wrong, torch.bfloat16)
    # the stated bound alone does not see it ...
    assert np.all(np.abs(got - ref) <= 2e-2 + 2e-2 * np.abs(ref))
    # ... the per-row rms figure does
    assert parity_figures(got, ref, torch.bfloat16)["rms_row_max"] > 8 * 2.0 ** -7
    with pytest.raises(AssertionError, match="per-row rms"):
        check_tolerance(got, ref, torch.bfloat16)
