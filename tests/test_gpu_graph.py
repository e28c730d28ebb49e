"""A decode step captured into a CUDA graph (GPU): after one uncaptured call
(which sets the kernels' shared-memory limit and caches device attributes),
the write and decode entry points record into a graph, and replaying it gives
bit-for-bit the eager result, again after the inputs have changed in place.
Each replayed output is also compared with the oracle (the new tokens written
by the oracle's own write, then its decode) at the 16-bit tolerance."""

import pytest
import torch

import oracle
import workloads
import paged_kv_cache_449_b200 as pa
from pagedutil import as_f64, check_tolerance, device_batch

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.contiguous().view(-1).view(torch.int32 if t.element_size() == 4 else torch.int16)


def _copies(b, n):
    out = []
    for _ in range(n):
        d = device_batch(b)
        d["k_cache"], d["v_cache"] = d["k_cache"].clone(), d["v_cache"].clone()
        d["nk"], d["nv"] = b.new_key.cuda().clone(), b.new_value.cuda().clone()
        d["slots"] = b.slot_mapping.cuda().clone()
        d["out"] = torch.full_like(d["q"], float("nan"))
        out.append(d)
    return out


def _steps(b):
    ws = torch.empty(pa.pa_decode_splitk_workspace_size(b.num_seqs, b.num_q_heads, b.head_dim,
                                                        b.max_context_len, 256), dtype=torch.uint8, device="cuda")
    counters = pa.Counters()
    counters.get(b.num_seqs * b.num_kv_heads, "cuda")

    def append(d):
        pa.pa_decode_append(d["out"], d["q"], d["nk"], d["nv"], d["k_cache"], d["v_cache"], d["block_tables"],
                            d["context_lens"], b.scale, max_context_len=b.max_context_len)

    def reshape_then_split(d):
        pa.pa_reshape_and_cache(d["nk"], d["nv"], d["k_cache"], d["v_cache"], d["slots"])
        pa.pa_decode_splitk(d["out"], d["q"], d["k_cache"], d["v_cache"], d["block_tables"], d["context_lens"],
                            b.scale, b.max_context_len, partition_size=256, workspace=ws, counters=counters)

    def reshape_then_two_kernel_split(d):
        pa.pa_reshape_and_cache(d["nk"], d["nv"], d["k_cache"], d["v_cache"], d["slots"])
        pa.pa_decode_splitk(d["out"], d["q"], d["k_cache"], d["v_cache"], d["block_tables"], d["context_lens"],
                            b.scale, b.max_context_len, partition_size=256, workspace=ws, fused=False)

    return {"append": append, "split_fused": reshape_then_split, "split_merge_kernel": reshape_then_two_kernel_split}


def _oracle_step(b, q):
    """The oracle's result of one step: the batch's new tokens written at
    their (decode-consistent) slots, then decode with queries q."""
    orc = oracle.default()
    kc, vc = b.k_cache.cpu().clone(), b.v_cache.cpu().clone()
    orc.reshape_and_cache(b.new_key.cpu(), b.new_value.cpu(), kc, vc, b.slot_mapping, b.block_size)
    return orc.decode(q.cpu(), kc, vc, b.block_tables, b.context_lens, b.scale, b.block_size, b.num_kv_heads)


@pytest.mark.parametrize("which", ["append", "split_fused", "split_merge_kernel"])
def test_graph_replay_equals_eager(which):
    b = workloads.llama3_8b_decode(seed=31, device="cuda", num_seqs=16, num_blocks=2048)
    eager, graphed = _copies(b, 2)
    step = _steps(b)[which]
    pa.pa_get_device_error()
    step(graphed)                      # the uncaptured first call
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(graphed)
    for round_ in range(2):
        if round_ == 1:                # new queries in place: the graph reads them at replay
            newq = torch.randn(eager["q"].shape, generator=torch.Generator(device="cuda").manual_seed(5),
                               device="cuda").to(eager["q"].dtype)
            eager["q"].copy_(newq)
            graphed["q"].copy_(newq)
        step(eager)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(_bits(graphed["out"]), _bits(eager["out"])), (which, round_)
        assert torch.equal(_bits(graphed["k_cache"]), _bits(eager["k_cache"]))
        check_tolerance(as_f64(graphed["out"]), _oracle_step(b, graphed["q"]), b.dtype)
    assert pa.pa_get_device_error() == 0
    del g


def test_graph_replay_fp8():
    b = workloads.llama3_8b_decode(seed=32, device="cuda", num_seqs=16, num_blocks=2048)
    pools = workloads.random_fp8_pools(b, seed=3, device="cuda")
    q, bt, cl = b.q.cuda(), b.block_tables.cuda(), b.context_lens.cuda()
    outs = [torch.full_like(q, float("nan")) for _ in range(2)]

    def step(out):
        pa.pa_decode_fp8(out, q, pools.k_cache, pools.v_cache, pools.k_scale, pools.v_scale, bt, cl, b.scale,
                         max_context_len=b.max_context_len)

    step(outs[1])
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(outs[1])
    outs[1].fill_(float("nan"))
    step(outs[0])
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(_bits(outs[1]), _bits(outs[0]))
    ref = oracle.default().decode_e4m3(b.q.cpu(), pools.k_cache.cpu(), pools.v_cache.cpu(), pools.k_scale.cpu(),
                                       pools.v_scale.cpu(), b.block_tables, b.context_lens, b.scale, b.block_size,
                                       b.num_kv_heads)
    check_tolerance(as_f64(outs[1]), ref, b.dtype)
    del g


def test_graph_replay_shared_prefix():
    """The shared-prefix step -- two launches, the second a programmatic
    dependent launch that meets the first through arrival counters -- captured
    and replayed: bit-identical to the eager call (outputs and pools), also
    after new queries are written in place, and the oracle's attention."""
    b = workloads.prefix_sharing(seed=33, device="cuda", num_seqs=24, prefix_len=256)
    eager, graphed = _copies(b, 2)
    P = b.meta["shared_blocks"]
    need = pa.pa_decode_shared_prefix_workspace_size(b.num_seqs, b.num_q_heads, b.head_dim, P, b.block_size)
    ws = [torch.empty(need, dtype=torch.uint8, device="cuda") for _ in range(2)]
    counters = [torch.zeros(b.num_seqs * b.num_kv_heads, dtype=torch.int32, device="cuda") for _ in range(2)]

    def step(d, i):
        pa.pa_decode_shared_prefix(d["out"], d["q"], d["nk"], d["nv"], d["k_cache"], d["v_cache"], d["block_tables"],
                                   d["context_lens"], b.scale, P, max_context_len=b.max_context_len,
                                   workspace=ws[i], counters=counters[i])

    pa.pa_get_device_error()
    step(graphed, 1)                   # the uncaptured first call
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(graphed, 1)
    for round_ in range(2):
        if round_ == 1:
            newq = torch.randn(eager["q"].shape, generator=torch.Generator(device="cuda").manual_seed(6),
                               device="cuda").to(eager["q"].dtype)
            eager["q"].copy_(newq)
            graphed["q"].copy_(newq)
        step(eager, 0)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(_bits(graphed["out"]), _bits(eager["out"])), round_
        assert torch.equal(_bits(graphed["k_cache"]), _bits(eager["k_cache"]))
        assert torch.equal(_bits(graphed["v_cache"]), _bits(eager["v_cache"]))
        check_tolerance(as_f64(graphed["out"]), _oracle_step(b, graphed["q"]), b.dtype)
    assert int(counters[0].abs().sum()) == 0 and int(counters[1].abs().sum()) == 0   # left at zero
    assert pa.pa_get_device_error() == 0
    del g


def test_graph_replay_of_a_block_manager_step():
    """A serving step of three launches -- pa_blocks_append, pa_copy_blocks,
    pa_decode_append, each a programmatic dependent launch of the one before --
    captured once and replayed: after the same number of steps the block
    manager's state, the pools and the output are bit-identical to an eager
    twin's."""
    b = workloads.llama3_8b_decode(seed=34, device="cuda", num_seqs=16, num_blocks=2048)
    B, N, S = b.block_size, b.num_blocks, b.num_seqs
    mb = b.max_blocks_per_seq + 2
    lens0 = (b.context_lens - 1).to(torch.int64)

    def state():
        tables = torch.full((S, mb), -1, dtype=torch.int32)
        ref = torch.zeros(N, dtype=torch.int32)
        for s in range(S):
            n = int((lens0[s] + B - 1) // B)
            tables[s, :n] = b.block_tables[s, :n]
            ref[b.block_tables[s, :n].long()] = 1
        free = torch.nonzero(ref == 0).flatten().to(torch.int32)
        ring = torch.full((N,), -1, dtype=torch.int32)
        ring[:free.numel()] = free
        return dict(tables=tables.cuda(), lens=lens0.to(torch.int32).cuda(), ref=ref.cuda(), ring=ring.cuda(),
                    state=torch.tensor([0, free.numel()], dtype=torch.int64, device="cuda"),
                    ones=torch.ones(S, dtype=torch.int32, device="cuda"),
                    slots=torch.empty(S, dtype=torch.int64, device="cuda"),
                    pairs=torch.empty((S, 2), dtype=torch.int64, device="cuda"),
                    k=b.k_cache.cuda().clone(), v=b.v_cache.cuda().clone(), q=b.q.cuda(),
                    nk=b.new_key.cuda(), nv=b.new_value.cuda(), out=torch.empty_like(b.q.cuda()))

    def step(d):
        pa.pa_blocks_append(d["tables"], d["lens"], d["ones"], d["ref"], d["ring"], d["state"], d["slots"],
                            d["pairs"], B)
        pa.pa_copy_blocks(d["k"], d["v"], d["k"], d["v"], d["pairs"])
        pa.pa_decode_append(d["out"], d["q"], d["nk"], d["nv"], d["k"], d["v"], d["tables"], d["lens"], b.scale,
                            max_context_len=mb * B, ref_counts=d["ref"])

    eager, graphed = state(), state()
    pa.pa_get_device_error()
    step(graphed)                      # the uncaptured first step
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(graphed)
    step(eager)
    for _ in range(2):
        step(eager)
        g.replay()
    torch.cuda.synchronize()
    for key in ("tables", "lens", "ref", "ring", "state", "slots", "pairs"):
        assert torch.equal(graphed[key], eager[key]), key
    assert torch.equal(_bits(graphed["out"]), _bits(eager["out"]))
    assert torch.equal(_bits(graphed["k"]), _bits(eager["k"])) and torch.equal(_bits(graphed["v"]), _bits(eager["v"]))
    assert pa.pa_get_device_error() == 0
    del g
