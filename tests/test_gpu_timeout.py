"""Bounded waits run out without a fault or a hang (GPU), through the test
hooks of include/pa_test.h, which only libpa_test.so (the library compiled
with PA_TEST_HOOKS) exports.  The waits are made to run out by work that is
never issued, never by a fault:

  * one warp waits on an mbarrier that nothing completes: the wait gives up
    after its limit, PA_DEVERR_TIMEOUT is set, and the next launches on the
    same context compute correct results;
  * the decode kernels' own timeout path: one warp of one thread block leaves
    its first ring stage unfilled; the block waits (bounded) for its other
    copies, reports PA_DEVERR_TIMEOUT and ends.  Every other sequence's output
    still matches the oracle, the fused split merge still brings its arrival
    counters back to zero, and with the hook off the next call matches the
    oracle in full.

The prefill kernel's timeout path (tensor memory released on abort) is not
reached by these hooks."""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
import paged_kv_cache_449_b200 as pa
from paged_kv_cache_449_b200 import build as pabuild
from pagedutil import as_f64, check_tolerance, device_batch, gpu_decode, oracle_decode_sampled

pytestmark = pytest.mark.gpu

LIMIT_NS = 200_000          # 0.2 ms: far above a copy's latency, far below the product's 1 s


@pytest.fixture(scope="module")
def test_lib():
    lib = pa.load_library(pabuild.build_test())
    lib.pa_test_set_hooks.restype = ctypes.c_int
    lib.pa_test_set_hooks.argtypes = [ctypes.c_int64, ctypes.c_int]
    lib.pa_test_wait_timeout.restype = ctypes.c_int
    lib.pa_test_wait_timeout.argtypes = [ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
    return lib


@pytest.fixture
def hooked(test_lib, monkeypatch):
    """The binding routed to libpa_test.so for one test; hooks reset after."""
    monkeypatch.setattr(pa, "_lib", test_lib)
    pa.pa_get_device_error()
    yield test_lib
    assert test_lib.pa_test_set_hooks(1_000_000_000, 0) == 0


def test_a_wait_nothing_completes_gives_up(hooked):
    elapsed = torch.zeros(1, dtype=torch.int64, device="cuda")
    assert hooked.pa_test_wait_timeout(LIMIT_NS, elapsed.data_ptr(), None) == 0
    assert pa.pa_get_device_error() == pa.DEVERR_TIMEOUT
    waited = int(elapsed.item())
    assert LIMIT_NS <= waited < 1000 * LIMIT_NS
    # the context is usable: a decode on it matches the oracle
    b = workloads.random_small(seed=81, dtype=torch.bfloat16, lens=(33, 200, 1), num_q_heads=8, num_kv_heads=2,
                               head_dim=128, block_size=16)
    check_tolerance(as_f64(gpu_decode(b, "single")), oracle_decode_sampled(oracle.default(), b, range(3)), b.dtype)
    assert pa.pa_get_device_error() == 0


@pytest.mark.parametrize("mode", ["single", "splitk", "splitk2"])
def test_decode_timeout_path(hooked, mode):
    b = workloads.random_small(seed=82, dtype=torch.bfloat16, lens=(300, 130, 77, 1), num_q_heads=16,
                               num_kv_heads=4, head_dim=128, block_size=16)
    ref = oracle_decode_sampled(oracle.default(), b, range(b.num_seqs))
    dev = device_batch(b)
    counters = pa.Counters()
    assert hooked.pa_test_set_hooks(LIMIT_NS, 1) == 0
    if mode == "single":
        out = gpu_decode(b, mode, dev=dev)
    else:
        out = torch.full_like(dev["q"], float("nan"))
        pa.pa_decode_splitk(out, dev["q"], dev["k_cache"], dev["v_cache"], dev["block_tables"], dev["context_lens"],
                            b.scale, b.max_context_len, partition_size=64, fused=(mode == "splitk"),
                            counters=counters)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == pa.DEVERR_TIMEOUT
    # every other sequence, and sequence 0's other kv heads, are untouched by the failure
    got = as_f64(out)
    g = b.num_q_heads // b.num_kv_heads
    check_tolerance(got[1:], ref[1:], b.dtype)
    check_tolerance(got[0, g:], ref[0, g:], b.dtype)
    if mode == "splitk":
        assert torch.count_nonzero(counters.buf).item() == 0        # arrival counters back at zero
        assert np.all(np.isfinite(got[0, :g]))                      # merged without the empty partition
    # hooks off: the next call on the same context computes the full result
    assert hooked.pa_test_set_hooks(1_000_000_000, 0) == 0
    again = gpu_decode(b, "splitk" if mode != "single" else "single", partition_size=64, dev=dev)
    check_tolerance(as_f64(again), ref, b.dtype)
    assert pa.pa_get_device_error() == 0
