"""Benchmark of the paged decode hot path: one step = write the newest token of
every sequence into the KV pool (pa_reshape_and_cache) + paged decode attention
over every sequence's whole context (pa_decode_append by default: both in one
launch; or pa_reshape_and_cache followed by pa_decode / pa_decode_splitk, --mode).

Default workload: Llama-3-8B-shaped single-layer decode, bf16 — 64 sequences,
32 q / 8 kv heads, head_dim 128, block size 16, context lengths uniform on
[128, 2048], a 16384-block pool with shuffled ids, synthetic N(0,1) data.

Prints one JSON line (rank 0).  `value` is KV GB/s over the whole step:
algorithmic bytes (sum_s L_s*Hkv*D*2*e + Q + out + block-table entries +
context_lens, plus the new tokens' K/V read and written) / step time, summed
over ranks and divided by the max-over-ranks time.  Timing: CUDA events on the
launching stream around the K timed steps.  L2: by default every step's inputs
are larger than L2 and the steps rotate over enough independent copies of the
workload (pools, tables, queries) that a step never finds in L2 what an
earlier step left there; --l2 flush instead writes a 256 MiB buffer between
steps and times each step with its own events.

Multi-GPU: sequences are independent, so each rank runs its own batch (weak
scaling, no data-path collective); only the timing reduction crosses ranks.

--impl reference times the fp64 CPU oracle (the only reference available: the
pages ship no code) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np
import torch

METRIC = "paged decode KV GB/s & tokens/s (Llama-3-8B shape) as % of B200 HBM peak"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
PCIE_GEN5_X16_GBS = 64.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama3_8b_decode",
                    choices=["tiny_mha_f32", "llama3_8b_decode", "continuous_batching_mix", "prefix_sharing",
                             "llama3_70b_long"])
    ap.add_argument("--block-size", type=int, default=None)
    ap.add_argument("--op", choices=["decode", "copy_blocks", "swap_out", "swap_in", "prefill", "block_step"],
                    default="decode",
                    help="decode: the hot-path step (default); copy_blocks: every block of the batch duplicated "
                         "into free blocks of the same pools (copy-on-write / fork); swap_out / swap_in: every "
                         "block of the batch copied to / from a pinned host pool (preemption by swapping); "
                         "block_step: a decode step through the device block manager (pa_blocks_append + "
                         "pa_copy_blocks + pa_decode_append)")
    ap.add_argument("--mode", choices=["append", "single", "splitk", "splitk2", "shared_prefix"], default="append",
                    help="append: one pa_decode_append launch per step (write + decode); the others launch "
                         "pa_reshape_and_cache then pa_decode (single) or pa_decode_splitk with fused (splitk) or "
                         "kernel (splitk2) merge")
    ap.add_argument("--partition-size", type=int, default=1024)
    ap.add_argument("--kv", choices=["bf16", "fp8"], default="bf16",
                    help="KV pool format: the workload's 16-bit/32-bit elements, or 8-bit e4m3 codes with per-kv-head "
                         "scales (pa_reshape_and_cache_fp8 + pa_decode_fp8 / pa_decode_splitk_fp8)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--l2", choices=["rotate", "flush"], default="rotate",
                    help="rotate: inputs larger than L2, rotated over independent copies, K steps timed as one "
                         "region; flush: a 256 MiB write between steps, per-step events")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="capture each rotated copy's step into a CUDA graph once and replay it in the timed region")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-configuration lines (by default the headline run also times every other "
                         "configuration and widened row and reports them under `configs`)")
    ap.add_argument("--cpu-sample-seconds", type=float, default=15.0)
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------- helpers

def cpu_model():
    """The host CPU's model name (Linux /proc/cpuinfo), or the platform's."""
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def cuda_runtime():
    """The CUDA runtime library torch loaded (for cudaMemcpyAsync), or None."""
    import ctypes
    import glob
    here = os.path.dirname(torch.__file__)
    for path in (glob.glob(os.path.join(here, "..", "nvidia", "cuda_runtime", "lib", "libcudart.so*"))
                 + glob.glob(os.path.join(here, "lib", "libcudart*.so*"))):
        try:
            lib = ctypes.CDLL(path)
        except OSError:
            continue
        fn = lib.cudaMemcpyAsync
        fn.restype = ctypes.c_int
        fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p]
        lib.cudaEventRecord.restype = ctypes.c_int
        lib.cudaEventRecord.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        lib.cudaStreamWaitEvent.restype = ctypes.c_int
        lib.cudaStreamWaitEvent.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint]
        return lib
    return None


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def make_workload(name, seed, device, block_size=None):
    import workloads
    kw = {"seed": seed, "device": device}
    if block_size is not None and name != "tiny_mha_f32":
        kw["block_size"] = block_size
    return workloads.CONFIGS[name](**kw)


# DRAM bytes (read + write) per launch of the timed decode kernel, from one
# Nsight Compute capture (dram__bytes_read.sum + dram__bytes_write.sum; summaries
# in profiles/).  Keyed by a hash of the kernel sources: once the kernels change,
# the figure no longer describes them and the bench reports null.
NCU_TRAFFIC = {
    "407f0ade94d110ef": {
        ("llama3_8b_decode_bf16", "append"): 292.750e6 + 3.574e6,
        ("continuous_batching_mix_bf16_B16", "append"): 211.576e6 + 3.781e6,
        ("llama3_70b_long_bf16", "splitk"): 2.519721e9 + 7.594e6,
        ("llama3_8b_decode_bf16+e4m3", "append"): 146.834e6 + 3.286e6,
        ("llama3_70b_long_bf16+e4m3", "splitk"): 1.260204e9 + 6.536e6,
    },
    "b608f02ff2d38061": {
        ("chunked_prefill_bfloat16", "prefill"): 118.548e6 + 19.906e6,
        ("chunked_prefill_bfloat16_B8", "prefill"): 118.360e6 + 20.081e6,
        ("chunked_prefill_bfloat16_B32", "prefill"): 118.734e6 + 21.116e6,
    },
    # the shared-prefix step: its prefix pass plus its decode pass
    "8551f531244d8acb": {
        ("prefix_sharing_f16_p1024", "shared_prefix"): 5.319e6 + 0.0 + 153.343e6 + 0.265e6,
    },
}


# the sources each recorded kernel is compiled from (its launch configuration
# lives in pa_api.cu)
DECODE_SOURCES = ("pa_api.cu", "pa_decode.cuh", "pa_e4m3.cuh", "pa_warp.cuh", "pa_device.cuh", "pa_reshape.cuh")
PREFILL_SOURCES = ("pa_api.cu", "pa_prefill_tc.cuh", "pa_prefill.cuh", "pa_device.cuh")
# the shared-prefix step runs both kernels
SHARED_PREFIX_SOURCES = tuple(sorted(set(DECODE_SOURCES + PREFILL_SOURCES)))


def sources_of(mode):
    return SHARED_PREFIX_SOURCES if mode == "shared_prefix" else DECODE_SOURCES


def code_of(text):
    """A source's code without its comments, tokens joined by single spaces
    (string literals kept whole, so a "//" inside one is not a comment)."""
    import re
    tokens = re.findall(r'"(?:\\.|[^"\\])*"|//[^\n]*|/\*.*?\*/|\S+', text, flags=re.S)
    return " ".join(t for t in tokens if not (t.startswith("//") or t.startswith("/*")))


def kernel_source_hash(names=DECODE_SOURCES):
    """Hash of the named kernel sources' code: comments and whitespace are
    dropped, so that a comment-only edit (which changes no instruction) keeps
    the DRAM traffic taken for the same code."""
    import hashlib
    h = hashlib.sha256()
    for name in sorted(names):
        with open(os.path.join(ROOT, "paged_kv_cache_449_b200", "csrc", name), encoding="utf-8") as fh:
            text = fh.read()
        h.update(name.encode())
        h.update(code_of(text).encode())
    return h.hexdigest()[:16]


def step_bytes(batch, fp8=None):
    """Algorithmic bytes of one step: the decode's (K/V + Q + out + block-table
    entries + context_lens) and the reshape's (new K/V read + written, slots);
    with 8-bit pools the K/V codes are one byte each (plus the scales)."""
    T = int(batch.slot_mapping.numel())
    row = T * batch.num_kv_heads * batch.head_dim
    if fp8 is not None:
        return fp8.algorithmic_bytes(batch), 2 * row * (batch.elem_bytes + 1) + 8 * T + 2 * batch.num_kv_heads * 4
    return batch.algorithmic_bytes(), 2 * 2 * row * batch.elem_bytes + 8 * T


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.device_index = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.device_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        if not getattr(self, "lines", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            parts = [p.strip() for p in l.split(",")]
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- distributed plumbing

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def reduce_max(value: float, world: int) -> float:
    """Max of a scalar over ranks (timing only; not on the data path)."""
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- the GPU arm

class Step:
    """One hot-path step through the C ABI on device-resident inputs."""

    def __init__(self, batch, mode, partition_size, independent=True, fp8=None, longest_first=False):
        import paged_kv_cache_449_b200 as pa
        self.pa = pa
        self.b = batch
        self.mode = mode
        self.part = partition_size
        self.fp8 = fp8 is not None
        dev = "cuda"

        def own(t):  # independent: a device copy with its own memory, never an alias of the batch's
            t = t.to(dev).contiguous()
            return t.clone() if independent else t

        if self.fp8:   # 8-bit pools (e4m3 codes) with per-kv-head scales
            self.k, self.v = own(fp8.k_cache), own(fp8.v_cache)
            self.ks, self.vs = own(fp8.k_scale), own(fp8.v_scale)
        else:
            self.k = own(batch.k_cache)
            self.v = own(batch.v_cache)
        # The per-step inputs live in one device buffer (256-byte aligned
        # views), so a step's upload from the host is a single copy.
        specs = [("q", batch.q), ("nk", batch.new_key), ("nv", batch.new_value), ("slots", batch.slot_mapping),
                 ("bt", batch.block_tables), ("cl", batch.context_lens)]
        if longest_first:   # the start order a scheduler that knows the lengths passes (seq_order)
            specs.append(("order", pa.longest_first(batch.context_lens)))
        offs, total = [], 0
        for _, t in specs:
            offs.append(total)
            total += (t.numel() * t.element_size() + 255) // 256 * 256
        self.inbuf = torch.empty(total, dtype=torch.uint8, device=dev)
        for (name, t), off in zip(specs, offs):
            view = self.inbuf[off:off + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
            view.copy_(t)
            setattr(self, name, view)
        if not longest_first:
            self.order = None
        self.out = torch.empty_like(self.q)
        self.mcl = batch.max_context_len
        if mode == "shared_prefix":   # every row begins with the batch's shared blocks
            need = pa.pa_decode_shared_prefix_workspace_size(batch.num_seqs, batch.num_q_heads, batch.head_dim,
                                                             batch.meta["shared_blocks"], batch.block_size)
        else:
            need = pa.pa_decode_splitk_workspace_size(batch.num_seqs, batch.num_q_heads, batch.head_dim, self.mcl,
                                                      self.part)
        self.ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        self.counters = pa.Counters()
        self.kernels_per_step = {"append": 1, "splitk2": 3}.get(mode, 2)
        # the one-launch step over these fixed buffers, marshalled once (a
        # serving loop's form of the call)
        self.prepared = None
        if mode == "append":
            if self.fp8:
                self.prepared = pa.prepare_decode_append_fp8(
                    self.out, self.q, self.nk, self.nv, self.k, self.v, self.ks, self.vs, self.bt, self.cl,
                    batch.scale, max_context_len=self.mcl, seq_order=self.order)
            else:
                self.prepared = pa.prepare_decode_append(
                    self.out, self.q, self.nk, self.nv, self.k, self.v, self.bt, self.cl, batch.scale,
                    max_context_len=self.mcl, seq_order=self.order)
        elif mode == "shared_prefix":
            if self.fp8:
                raise ValueError("the shared-prefix entry takes 16-bit pools")
            self.prepared = pa.prepare_decode_shared_prefix(
                self.out, self.q, self.nk, self.nv, self.k, self.v, self.bt, self.cl, batch.scale,
                batch.meta["shared_blocks"], max_context_len=self.mcl, workspace=self.ws)

    def reshape(self, stream):
        if self.mode in ("append", "shared_prefix"):
            return  # the newest token is written by the decode launch itself
        if self.fp8:
            self.pa.pa_reshape_and_cache_fp8(self.nk, self.nv, self.k, self.v, self.slots, self.ks, self.vs,
                                             stream=stream)
            return
        self.pa.pa_reshape_and_cache(self.nk, self.nv, self.k, self.v, self.slots, stream=stream)

    def decode(self, stream):
        if self.prepared is not None:
            self.prepared(stream)
            return
        if self.fp8:
            if self.mode == "append":
                self.pa.pa_decode_append_fp8(self.out, self.q, self.nk, self.nv, self.k, self.v, self.ks, self.vs,
                                             self.bt, self.cl, self.b.scale, max_context_len=self.mcl, stream=stream,
                                             seq_order=self.order)
            elif self.mode in ("splitk", "splitk2"):
                self.pa.pa_decode_splitk_fp8(self.out, self.q, self.k, self.v, self.ks, self.vs, self.bt, self.cl,
                                             self.b.scale, self.mcl, partition_size=self.part, workspace=self.ws,
                                             fused=(self.mode == "splitk"), counters=self.counters, stream=stream)
            else:
                self.pa.pa_decode_fp8(self.out, self.q, self.k, self.v, self.ks, self.vs, self.bt, self.cl,
                                      self.b.scale, max_context_len=self.mcl, stream=stream)
            return
        if self.mode == "append":
            self.pa.pa_decode_append(self.out, self.q, self.nk, self.nv, self.k, self.v, self.bt, self.cl, self.b.scale,
                                     max_context_len=self.mcl, stream=stream, seq_order=self.order)
        elif self.mode in ("splitk", "splitk2"):
            self.pa.pa_decode_splitk(self.out, self.q, self.k, self.v, self.bt, self.cl, self.b.scale, self.mcl,
                                     partition_size=self.part, workspace=self.ws, fused=(self.mode == "splitk"),
                                     counters=self.counters, stream=stream)
        else:
            self.pa.pa_decode(self.out, self.q, self.k, self.v, self.bt, self.cl, self.b.scale,
                              max_context_len=self.mcl, stream=stream)


def l2_bytes():
    try:
        return int(torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size)
    except (AttributeError, RuntimeError):
        return 126 << 20


def rotation_copies(unique_bytes, l2):
    """Independent input copies to rotate over so that, between two uses of a
    copy, at least twice the L2 capacity of other inputs has been streamed;
    0 when the workload is too small for that (then L2 is flushed instead)."""
    if unique_bytes <= 0:
        return 0
    r = max(2, math.ceil(2 * l2 / unique_bytes) + 1)
    return r if r <= 16 else 0


def run_gpu(args, world, rank, local):
    import paged_kv_cache_449_b200 as pa
    from paged_kv_cache_449_b200 import build as pabuild
    pabuild.build()
    pa.load()
    batch = make_workload(args.workload, args.seed + rank, "cuda", args.block_size)
    mode = args.mode
    fp8 = None
    if args.kv == "fp8":
        import workloads
        fp8 = workloads.random_fp8_pools(batch, seed=args.seed + rank, device="cuda")
    stream = torch.cuda.current_stream()
    l2 = l2_bytes()
    unique = batch.unique_kv_bytes() // (2 if fp8 is not None else 1)
    copies = rotation_copies(unique, l2) if args.l2 == "rotate" else 0
    # the first copy may use the batch's own device tensors; the others are clones
    steps = [Step(batch, mode, args.partition_size, independent=i > 0, fp8=fp8) for i in range(max(1, copies))]
    step = steps[0]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if copies == 0 else None
    decode_bytes, reshape_bytes = step_bytes(batch, fp8)

    def one(i, ev=None, on=None):
        s_ = on if on is not None else stream
        st = steps[i % len(steps)]
        if ev is not None:
            ev[0].record(s_)
        if st.mode not in ("append", "shared_prefix"):  # there the whole step is the one entry call
            st.reshape(s_)
        if ev is not None:
            ev[1].record(s_)
        st.decode(s_)
        if ev is not None:
            ev[2].record(s_)

    for i in range(args.warmup):
        if flush is not None:
            flush.zero_()
        one(i)
    torch.cuda.synchronize()
    if pa.pa_get_device_error() != 0:
        raise RuntimeError("device error word set during warm-up")
    graphs = None
    if args.graph:   # one graph per rotated copy, captured after the uncaptured warm-up calls
        graphs = []
        for i in range(len(steps)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                one(i, on=torch.cuda.current_stream())   # launches on the capturing stream
            graphs.append(g)
        torch.cuda.synchronize()

        def one(i, ev=None):
            if ev is not None:
                ev[0].record(stream)
                ev[1].record(stream)
            graphs[i % len(graphs)].replay()
            if ev is not None:
                ev[2].record(stream)

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    region = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        # Untimed steps while the sampler starts: the GPU is under load (and
        # at load clocks) when the timed region begins.
        t_busy, i = time.perf_counter() + 0.3, 0
        while time.perf_counter() < t_busy:
            if flush is not None:
                flush.zero_()
            one(i)
            i += 1
            if i % 16 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        barrier(world)
        if flush is None:
            # Rotated inputs: the K steps back to back, one timed region; the
            # per-step events inside it split reshape from decode.
            region[0].record(stream)
            for i in range(args.steps):
                one(i, events[i] if mode not in ("append", "shared_prefix") and graphs is None else None)
            region[1].record(stream)
        else:
            for i in range(args.steps):
                flush.zero_()
                one(i, events[i])
        torch.cuda.synchronize()
    barrier(world)
    if flush is None:
        local_step = region[0].elapsed_time(region[1]) / args.steps
        if mode in ("append", "shared_prefix") or graphs is not None:   # one entry call, or one graph replay
            decode_ms, reshape_ms = [local_step], [0.0]
        else:
            decode_ms = [e[1].elapsed_time(e[2]) for e in events]
            reshape_ms = [e[0].elapsed_time(e[1]) for e in events]
    else:
        step_ms = [e[0].elapsed_time(e[2]) for e in events]
        local_step = sum(step_ms) / len(step_ms)
        decode_ms = [e[1].elapsed_time(e[2]) for e in events]
        reshape_ms = [e[0].elapsed_time(e[1]) for e in events]
    local_decode = sum(decode_ms) / len(decode_ms)
    if pa.pa_get_device_error() != 0:
        raise RuntimeError("device error word set during the timed steps")

    # ---- end to end through the public API: pinned host inputs -> device -> step -> host output
    e2e = None
    if not args.no_e2e:
        host_in = step.inbuf.cpu().pin_memory()
        host_out = [torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory() for _ in range(2)]
        h2d = host_in.numel() * host_in.element_size()
        d2h = host_out[0].numel() * host_out[0].element_size()

        # The copies go straight to the CUDA runtime's cudaMemcpyAsync (the one
        # torch loads) on precomputed pointers: per step the host then spends a
        # few microseconds issuing them, not the tens a tensor copy costs.
        cudart = cuda_runtime()
        rcs = []
        in_ptr = host_in.data_ptr()
        out_ptrs = [t.data_ptr() for t in host_out]

        def upload(st, s):
            if cudart is None:
                with torch.cuda.stream(s):
                    st.inbuf.copy_(host_in, non_blocking=True)
                return
            rcs.append(cudart.cudaMemcpyAsync(st.inbuf_ptr, in_ptr, h2d, 1, s.cuda_stream))

        def download(st, i, s):
            if cudart is None:
                with torch.cuda.stream(s):
                    host_out[i % 2].copy_(st.out, non_blocking=True)
                return
            rcs.append(cudart.cudaMemcpyAsync(out_ptrs[i % 2], st.out_ptr, d2h, 2, s.cuda_stream))

        for st in steps:
            st.inbuf_ptr, st.out_ptr = st.inbuf.data_ptr(), st.out.data_ptr()

        def serial_step(i):
            st = steps[i % len(steps)]
            upload(st, stream)
            st.reshape(stream)
            st.decode(stream)
            download(st, i, stream)

        def pipelined(n, ev0, ev1):
            """n steps; step i+1's inputs go up on one copy stream while step i
            computes, and step i's output comes down on another (opposite
            directions: separate copy engines) once its kernels end.  A rotated
            copy's inputs are overwritten only after its previous step ended, and
            its output only after that output was read back."""
            up_s, down_s = torch.cuda.Stream(), torch.cuda.Stream()
            R = len(steps)
            up = [torch.cuda.Event() for _ in range(n)]
            done = [torch.cuda.Event() for _ in range(n)]
            down = [torch.cuda.Event() for _ in range(n)]
            for e in up + done + down:   # created (on first record) before the timed region
                e.record(stream)
            torch.cuda.synchronize()
            if cudart is not None:   # the runtime's own calls on the raw handles: a few us of host time less a step
                def rec(e, s_):
                    rcs.append(cudart.cudaEventRecord(e.cuda_event, s_.cuda_stream))

                def wait(s_, e):
                    rcs.append(cudart.cudaStreamWaitEvent(s_.cuda_stream, e.cuda_event, 0))
            else:
                def rec(e, s_):
                    e.record(s_)

                def wait(s_, e):
                    s_.wait_event(e)
            up_s.wait_stream(stream)
            down_s.wait_stream(stream)
            ev0.record(up_s)
            upload(steps[0], up_s)
            rec(up[0], up_s)
            for i in range(n):
                st = steps[i % R]
                wait(stream, up[i])
                if i - R >= 0:
                    wait(stream, down[i - R])
                st.reshape(stream)
                st.decode(stream)
                rec(done[i], stream)
                if i + 1 < n:
                    if i + 1 - R >= 0:
                        wait(up_s, done[i + 1 - R])
                    upload(steps[(i + 1) % R], up_s)
                    rec(up[i + 1], up_s)
                wait(down_s, done[i])
                download(st, i, down_s)
                rec(down[i], down_s)
            stream.wait_stream(up_s)
            stream.wait_stream(down_s)
            ev1.record(stream)

        e2e_modes = {}
        for kind in (("pipelined", "serial") if flush is None and len(steps) >= 2 else ("serial",)):
            for i in range(args.warmup):
                if flush is not None:
                    flush.zero_()
                serial_step(i)
            torch.cuda.synchronize()
            barrier(world)
            if kind == "pipelined":
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                pipelined(args.steps, ev[0], ev[1])
                torch.cuda.synchronize()
                e2e_modes[kind] = ev[0].elapsed_time(ev[1]) / args.steps
            elif flush is None:
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                ev[0].record(stream)
                for i in range(args.steps):
                    serial_step(i)
                ev[1].record(stream)
                torch.cuda.synchronize()
                e2e_modes[kind] = ev[0].elapsed_time(ev[1]) / args.steps
            else:
                e2e_events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
                for i in range(args.steps):
                    flush.zero_()
                    e2e_events[i][0].record(stream)
                    serial_step(i)
                    e2e_events[i][1].record(stream)
                torch.cuda.synchronize()
                e2e_modes[kind] = sum(e[0].elapsed_time(e[1]) for e in e2e_events) / args.steps
            barrier(world)
        if any(rc != 0 for rc in rcs):
            raise RuntimeError(f"cudaMemcpyAsync failed with {set(rcs) - {0}}")
        e2e_ms = e2e_modes.get("pipelined", e2e_modes["serial"])
        e2e_serial_ms_max = reduce_max(e2e_modes["serial"], world)
        e2e_ms_max = reduce_max(e2e_ms, world)
        e2e = {"value": None, "unit": "GB/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms_max, "_local_bytes": decode_bytes + reshape_bytes,
               "pipelined": "pipelined" in e2e_modes,
               "how": ("step i+1's inputs uploaded on a copy stream while step i computes; step i's output "
                       "read back on another copy stream when its kernels end" if "pipelined" in e2e_modes
                       else "upload, step, read-back serialised on one stream")
                      + ("; copies and event records / waits by the CUDA runtime's own calls, the step by its "
                         "prepared C-ABI call" if cudart is not None
                         else "; copies by torch tensor copies, the step by its prepared C-ABI call"),
               "serial_ms_per_step": e2e_serial_ms_max}

    step_ms_max = reduce_max(local_step, world)
    decode_ms_max = reduce_max(local_decode, world)
    total_bytes = reduce_sum(decode_bytes + reshape_bytes, world)
    total_decode_bytes = reduce_sum(decode_bytes, world)
    total_seqs = reduce_sum(batch.num_seqs, world)
    if e2e is not None:
        e2e["value"] = total_bytes / (e2e["ms_per_step"] * 1e-3) / 1e9
        e2e["serial_value"] = total_bytes / (e2e["serial_ms_per_step"] * 1e-3) / 1e9
        e2e.pop("_local_bytes")
    clk = clocks.summary()
    peak, peak_kind = measured_peaks()
    # Shared-prefix blocks are read from HBM once per step however many
    # sequences name them: the roofline counts them once.
    roof_bytes = batch.algorithmic_bytes(unique=True) if fp8 is None else decode_bytes
    achieved = roof_bytes / (local_decode * 1e-3) / 1e9
    value = total_bytes / (step_ms_max * 1e-3) / 1e9
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms_max, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32"}[batch.dtype]
        + ("+e4m3 KV (f16 MMA on widened codes)" if fp8 is not None else ""),
        "data": "synthetic (seeded N(0,1) K/V/Q, seeded lengths and shuffled block ids)",
        "config": {
            "workload": batch.name,
            "global_batch": int(total_seqs),
            "num_q_heads": batch.num_q_heads, "num_kv_heads": batch.num_kv_heads,
            "head_dim": batch.head_dim, "block_size": batch.block_size, "num_blocks": batch.num_blocks,
            "context_len_mean": float(batch.context_lens.float().mean()),
            "context_len_max": batch.max_context_len,
            "decode_entry": ({"splitk": "pa_decode_splitk (fused merge)", "splitk2": "pa_decode_splitk (merge kernel)",
                              "append": "pa_decode_append",
                              "shared_prefix": "pa_decode_shared_prefix (appending)"}.get(mode, "pa_decode")
                             if fp8 is None else
                             {"splitk": "pa_decode_splitk_fp8 (fused merge)",
                              "splitk2": "pa_decode_splitk_fp8 (merge kernel)",
                              "append": "pa_decode_append_fp8"}.get(mode, "pa_decode_fp8")),
            "kv_pool": ("e4m3 codes, one fp32 scale per kv head for K and for V (random codes)" if fp8 is not None
                        else "same type as the queries"),
            "partition_size": args.partition_size if mode.startswith("splitk") else None,
            "parallelism": f"replicas x{world} (sequence batches, no collective)",
            "l2": (f"inputs larger than L2 ({unique / 1e6:.0f} MB of distinct KV per step vs "
                   f"{l2 / 1e6:.0f} MB L2), rotated over {len(steps)} independent copies; K steps in one "
                   f"CUDA-event region") if flush is None
            else "flushed between steps (256 MiB write), per-step CUDA events",
            "graph": bool(args.graph),
            "step": ("pa_decode_append" + ("_fp8: newest token of every sequence quantised and written + decode, one "
                                           "launch" if fp8 is not None else
                                           ": newest token of every sequence written + decode, one launch")
                     if mode == "append"
                     else "pa_decode_shared_prefix: the shared prefix once per kv head for all sequences "
                          "(tcgen05 pass), then each sequence's own blocks with its newest token written, "
                          "the two merged; two launches"
                     if mode == "shared_prefix"
                     else "pa_reshape_and_cache_fp8 (newest token of every sequence, quantised) + decode"
                     if fp8 is not None
                     else "pa_reshape_and_cache (newest token of every sequence) + decode"),
        },
        "tokens_per_s": round(total_seqs / (step_ms_max * 1e-3), 1),
        "decode_ms": round(decode_ms_max, 5),
        "reshape_ms": round(sum(reshape_ms) / len(reshape_ms), 5),
        "decode_gbs": round(total_decode_bytes / (decode_ms_max * 1e-3) / 1e9, 2),
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "hbm_peak": f"{peak} GB/s, {peak_kind} copy bandwidth",
        "pct_of_spec_8tbs": round(100 * value / world / SPEC_HBM_GBS, 2),
        "roofline": {
            "bound": "hbm",
            "kernel": {"append": "pa_decode_kernel (append)", "splitk": "pa_decode_kernel<split, fused merge>",
                       "splitk2": "pa_decode_kernel<split> + pa_merge_kernel",
                       "shared_prefix": "pa_prefill_tc_kernel<prefix> + pa_decode_kernel<suffix, append>",
                       }.get(mode, "pa_decode_kernel"),
            "achieved": round(achieved, 2),
            "peak": peak,
            "peak_kind": f"{peak_kind} copy bandwidth (burst)",
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "frac_of_spec_8tbs": round(achieved / SPEC_HBM_GBS, 4),
            "algorithmic_bytes_per_launch": int(roof_bytes),
            "bytes_basis": ("unique: shared-prefix blocks counted once" if roof_bytes != decode_bytes
                            else "logical = unique"),
            "traffic": NCU_TRAFFIC.get(kernel_source_hash(sources_of(mode)), {}).get(
                (batch.name + ("+e4m3" if fp8 is not None else ""), mode)),
        },
        "gpu_launches": int(step.kernels_per_step * args.steps),
        "clocks": clk,
    }
    if e2e is not None:
        result["e2e"] = {k: (round(v, 3) if isinstance(v, float) else v) for k, v in e2e.items()}
    return result, batch


# ----------------------------------------------------------------------------- every configuration

def time_decode_steps(batch, mode, partition_size, fp8, steps, warmup, world, longest_first=False):
    """Device time of one step (write of the newest tokens + decode) on the
    batch: rotated independent copies larger than L2 when the workload allows
    (K steps in one CUDA-event region), else a 256 MiB L2 flush and per-step
    events.  Returns (ms per step, max over ranks; launches per step; L2
    note)."""
    import paged_kv_cache_449_b200 as pa
    stream = torch.cuda.current_stream()
    unique = batch.unique_kv_bytes() // (2 if fp8 is not None else 1)
    copies = rotation_copies(unique, l2_bytes())
    steps_ = [Step(batch, mode, partition_size, independent=i > 0, fp8=fp8, longest_first=longest_first)
              for i in range(max(1, copies))]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if copies == 0 else None

    def one(i):
        st = steps_[i % len(steps_)]
        st.reshape(stream)
        st.decode(stream)

    for i in range(warmup):
        if flush is not None:
            flush.zero_()
        one(i)
    torch.cuda.synchronize()
    barrier(world)
    if flush is None:
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record(stream)
        for i in range(steps):
            one(i)
        ev[1].record(stream)
        torch.cuda.synchronize()
        ms = ev[0].elapsed_time(ev[1]) / steps
        note = f"rotated over {len(steps_)} independent copies larger than L2, one event region"
    else:
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for i in range(steps):
            flush.zero_()
            evs[i][0].record(stream)
            one(i)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in evs) / steps
        note = "256 MiB L2 flush between steps, per-step events"
    barrier(world)
    if pa.pa_get_device_error() != 0:
        raise RuntimeError(f"device error word set on {batch.name}")
    return reduce_max(ms, world), steps_[0].kernels_per_step, note


def profiled_kernel_ms(fn, n, names):
    """Average device duration of each named kernel over n calls of fn, from
    the CUDA activity records of torch.profiler (device timestamps, not a
    replaying profiler).  None where the records are unavailable."""
    try:
        from torch.profiler import ProfilerActivity, profile
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            for i in range(n):
                fn(i)
            torch.cuda.synchronize()
        out = {}
        for ev in prof.key_averages():
            for name in names:
                if name in ev.key:
                    total = getattr(ev, "device_time_total", None)
                    if total is None:
                        total = getattr(ev, "cuda_time_total", 0.0)
                    cnt = out.get(name, (0.0, 0))
                    out[name] = (cnt[0] + total, cnt[1] + ev.count)
        return {k: (t / c / 1e3 if c else None) for k, (t, c) in out.items()}
    except Exception as err:  # the profiler's CUDA activity records are optional
        return {"unavailable": str(err)[:200]}


def block_manager_step(seed, steps, warmup, world, peak):
    """A whole decode step with the device block manager, on the Llama-3-8B
    batch: pa_blocks_append (one token per sequence: a block taken from the
    free ring when the token starts a block) + pa_copy_blocks (the step's
    copy-on-write pairs) + pa_decode_append (write + attend, reference counts
    checked).  The state starts from the batch's tables with each sequence
    one token short; the lengths grow by one per step (steps + warm-up
    tokens, negligible next to ~1000-token contexts)."""
    import paged_kv_cache_449_b200 as pa
    import workloads
    b = workloads.llama3_8b_decode(seed=seed, device="cuda")
    B, N, S = b.block_size, b.num_blocks, b.num_seqs
    total = steps + warmup + 1
    mb = b.max_blocks_per_seq + (total + B - 1) // B + 1
    lens0 = (b.context_lens - 1).to(torch.int64)
    tables = torch.full((S, mb), -1, dtype=torch.int32)
    ref = torch.zeros(N, dtype=torch.int32)
    for s_ in range(S):
        n = int((lens0[s_] + B - 1) // B)
        tables[s_, :n] = b.block_tables[s_, :n]
        ref[b.block_tables[s_, :n].long()] = 1
    free = torch.nonzero(ref == 0).flatten().to(torch.int32)
    ring = torch.full((N,), -1, dtype=torch.int32)
    ring[:free.numel()] = free
    d = "cuda"
    tables, lens, ref, ring = tables.to(d), lens0.to(torch.int32).to(d), ref.to(d), ring.to(d)
    state = torch.tensor([0, free.numel()], dtype=torch.int64, device=d)
    ones = torch.ones(S, dtype=torch.int32, device=d)
    slots = torch.empty(S, dtype=torch.int64, device=d)
    pairs = torch.empty((S, 2), dtype=torch.int64, device=d)
    k, v, q = b.k_cache, b.v_cache, b.q.to(d)
    nk, nv = b.new_key.to(d), b.new_value.to(d)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()

    def one(i):
        pa.pa_blocks_append(tables, lens, ones, ref, ring, state, slots, pairs, B, stream=stream)
        pa.pa_copy_blocks(k, v, k, v, pairs, stream=stream)
        pa.pa_decode_append(out, q, nk, nv, k, v, tables, lens, b.scale, max_context_len=mb * B, stream=stream,
                            ref_counts=ref)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    barrier(world)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record(stream)
    for i in range(steps):
        one(i)
    ev[1].record(stream)
    torch.cuda.synchronize()
    ms = reduce_max(ev[0].elapsed_time(ev[1]) / steps, world)
    per_kernel = profiled_kernel_ms(one, 1, ("pa_blocks_append_kernel", "pa_copy_blocks_kernel", "pa_decode_kernel"))
    if pa.pa_get_device_error() != 0:
        raise RuntimeError("device error word set in the block-manager step")
    # every step adds a token to every sequence: count the bytes at the mean
    # length over the timed steps (step i reads lens0 + warmup + i + 1 tokens)
    grow = warmup + (steps + 1) / 2.0
    mean_tokens = float(lens0.sum()) + S * grow
    e = b.elem_bytes
    tables = sum(math.ceil((float(L) + grow) / B) for L in lens0.tolist()) * 4
    nbytes = int(mean_tokens * b.num_kv_heads * b.head_dim * 2 * e + 2 * S * b.num_q_heads * b.head_dim * e
                 + tables + 4 * S + 4 * S * b.num_kv_heads * b.head_dim * e)   # new K/V rows read + written
    gbs = reduce_sum(nbytes, world) / (ms * 1e-3) / 1e9
    return {"workload": b.name + " + device block manager",
            "entry": "pa_blocks_append + pa_copy_blocks + pa_decode_append (ref counts)",
            "ms_per_step": round(ms, 5), "algorithmic_bytes": int(nbytes), "gb_per_s": round(gbs, 2),
            "frac_of_hbm_peak": round(gbs / world / peak, 4),
            "hbm_peak": f"{peak} GB/s, {measured_peaks()[1]} copy bandwidth",
            "kernel_ms": {k_: (round(v_, 5) if isinstance(v_, float) else v_) for k_, v_ in per_kernel.items()},
            "kernel_ms_how": ("torch.profiler CUDA activity records of one step after the timed ones; a "
                              "kernel's grid may be resident before the launch ahead of it ends (it waits "
                              "for that launch first), so a record can include that wait"),
            "gpu_launches": 3 * steps,
            "bytes_basis": ("K/V at the mean context length over the timed steps (each step appends a token to "
                            "every sequence) + q, out, the new rows, block-table entries and lengths"),
            "l2": "one copy of the pools (290 MB of KV per step, more than twice the L2), K steps in one event region"}


def config_lines(args, world, rank):
    """One entry per configuration of the hot path (and of the widened rows),
    each timed on its own seeded workload with the same rules as the
    headline: device-resident inputs, warm-up, CUDA events, rotated copies
    larger than L2 (or an L2 flush where the workload is smaller than L2)."""
    import paged_kv_cache_449_b200 as pa
    import workloads
    peak, peak_kind = measured_peaks()
    K, W = args.steps, max(3, args.warmup)
    out = {}

    def entry(batch, mode, part=None, fp8=None, note=None, longest_first=False):
        ms, launches, l2 = time_decode_steps(batch, mode, part or args.partition_size, fp8, K, W, world,
                                             longest_first)
        dec, resh = step_bytes(batch, fp8)
        logical = dec + resh
        unique = (batch.algorithmic_bytes(unique=True) if fp8 is None else dec) + resh
        gbs = reduce_sum(unique, world) / (ms * 1e-3) / 1e9
        e = {"workload": batch.name + ("+e4m3" if fp8 is not None else ""), "entry": {
                "append": "pa_decode_append" + ("_fp8" if fp8 is not None else ""),
                "single": "pa_reshape_and_cache + pa_decode",
                "splitk": f"pa_reshape_and_cache + pa_decode_splitk (fused merge, partition {part})",
                "splitk2": f"pa_reshape_and_cache + pa_decode_splitk (merge kernel, partition {part})",
                "shared_prefix": "pa_decode_shared_prefix (appending; prefix pass + own-block pass)"}[mode],
             "seqs": batch.num_seqs, "block_size": batch.block_size, "ms_per_step": round(ms, 5),
             "algorithmic_bytes": int(unique), "gb_per_s": round(gbs, 2),
             "frac_of_hbm_peak": round(gbs / world / peak, 4), "frac_of_spec_8tbs": round(gbs / world / SPEC_HBM_GBS, 4),
             "tokens_per_s": round(reduce_sum(batch.num_seqs, world) / (ms * 1e-3), 1),
             "gpu_launches": launches * K, "l2": l2}
        if unique != logical:
            e["logical_bytes"] = int(logical)
            e["bytes_basis"] = "unique: shared-prefix blocks counted once (logical bytes beside)"
        if note:
            e["note"] = note
        if longest_first:
            e["seq_order"] = "longest first (built on the host from the lengths, uploaded with the step's inputs)"
        traffic = NCU_TRAFFIC.get(kernel_source_hash(sources_of(mode)), {}).get(
            (batch.name + ("+e4m3" if fp8 is not None else ""), mode))
        if traffic is not None and not longest_first:
            e["traffic"] = traffic   # DRAM read + write bytes of the decode launch (profiles/)
        return e

    seed = args.seed + rank
    b = workloads.tiny_mha_f32(seed=seed, device="cuda")
    out["tiny_mha_f32"] = entry(b, "append", note="parity configuration: launch-bound, its GB/s is not a "
                                                  "bandwidth figure")
    del b
    for B in (8, 16, 32):
        b = workloads.continuous_batching_mix(seed=seed, device="cuda", block_size=B)
        out[f"continuous_batching_mix_B{B}"] = entry(b, "append")
        out[f"continuous_batching_mix_B{B}_longest_first"] = entry(b, "append", longest_first=True)
        del b
    b = workloads.prefix_sharing(seed=seed, device="cuda")
    out["prefix_sharing"] = entry(b, "append")
    out["prefix_sharing_shared_prefix"] = entry(b, "shared_prefix")
    del b
    b = workloads.llama3_70b_long(seed=seed, device="cuda")
    out["llama3_70b_long"] = entry(b, "splitk", part=1024)
    two = entry(b, "splitk2", part=1024)
    st = Step(b, "splitk2", 1024)
    stream = torch.cuda.current_stream()
    per_kernel = profiled_kernel_ms(lambda i: (st.reshape(stream), st.decode(stream)), min(K, 20),
                                    ("pa_reshape_kernel", "pa_decode_kernel", "pa_merge_kernel"))
    two["kernel_ms"] = {k: (round(v, 5) if isinstance(v, float) else v) for k, v in per_kernel.items()}
    two["kernel_ms_how"] = ("torch.profiler CUDA activity records over min(steps, 20) steps on one input copy "
                            "(L2 not flushed between them); a kernel's grid may be resident before the launch "
                            "ahead of it ends (it waits for that launch first), so a record can include that "
                            "wait: the step time is the figure to compare")
    out["llama3_70b_long_two_kernel"] = two
    del b, st
    b = workloads.llama3_8b_decode(seed=seed, device="cuda")
    f8 = workloads.random_fp8_pools(b, seed=seed, device="cuda")
    out["llama3_8b_decode_e4m3"] = entry(b, "append", fp8=f8)
    del b, f8
    torch.cuda.empty_cache()
    out["serving_step_with_block_manager"] = block_manager_step(seed, K, W, world, peak)
    torch.cuda.empty_cache()
    # the widened rows measured by their own bench modes, trimmed to the figures
    keep = ("metric", "value", "unit", "ms_per_step", "roofline", "gpu_launches")
    for name, op, workload, steps, bs in (("chunked_prefill", "prefill", args.workload, K, None),
                                          ("chunked_prefill_B8", "prefill", args.workload, K, 8),
                                          ("chunked_prefill_B32", "prefill", args.workload, K, 32),
                                          ("copy_blocks_cow", "copy_blocks", "llama3_8b_decode", K, None),
                                          ("swap_out", "swap_out", "llama3_8b_decode", min(K, 10), None),
                                          ("swap_in", "swap_in", "llama3_8b_decode", min(K, 10), None)):
        sub = argparse.Namespace(**dict(vars(args), op=op, workload=workload, steps=steps, warmup=W,
                                        block_size=bs))
        res = (run_prefill if op == "prefill" else run_blocks)(sub, world, rank, int(os.environ.get("LOCAL_RANK", "0")))
        e = {k: res[k] for k in keep if k in res}
        e["workload"] = res["config"]["workload"]
        if op == "prefill":
            e["block_size"] = res["config"]["block_size"]
        out[name] = e
        torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- the oracle (CPU)

def oracle_sample(batch, seconds_target, seed=0):
    """Times the oracle on a bounded sample of the batch's sequences; returns
    (GB/s over the sample's algorithmic bytes, description, threads)."""
    import oracle
    orc = oracle.default()
    rng = np.random.default_rng(seed)
    order = list(rng.permutation(batch.num_seqs))
    # estimate the cost of one sequence from a first one, then size the sample
    taken, spent, nbytes = [], 0.0, 0
    e = batch.elem_bytes
    per_seq_fixed = 2 * batch.num_q_heads * batch.head_dim * e + 4
    for s in order:
        seqs = [int(s)]
        q, k, v, bt, cl = _compact(batch, seqs)
        t0 = time.perf_counter()
        orc.decode(q, k, v, bt, cl, batch.scale, batch.block_size, batch.num_kv_heads)
        spent += time.perf_counter() - t0
        L = int(batch.context_lens[s])
        nbytes += L * batch.num_kv_heads * batch.head_dim * 2 * e + per_seq_fixed + \
            ((L + batch.block_size - 1) // batch.block_size) * 4
        taken.append(int(s))
        if spent >= seconds_target:
            break
    gbs = nbytes / spent / 1e9
    desc = (f"{len(taken)} of {batch.num_seqs} sequences (seeded sample, "
            f"{sum(int(batch.context_lens[s]) for s in taken)} tokens), single-threaded fp64, {spent:.1f} s")
    return gbs, desc, spent, len(taken)


def oracle_sample_all_cores(batch, seconds_target, seed=0):
    """The oracle over the host's cores: one thread per core, one whole
    sequence per task.  The oracle is a C library called through ctypes,
    which releases the interpreter lock for the call, and it keeps no state
    between calls, so the threads run it in parallel unchanged.  Sequences
    are repeated until the wall time reaches about seconds_target / cores.
    Returns (GB/s over the processed sequences' algorithmic bytes,
    description, cores)."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    orc = oracle.default()
    cores = max(1, os.cpu_count() or 1)
    e = batch.elem_bytes
    per_seq_fixed = 2 * batch.num_q_heads * batch.head_dim * e + 4
    order = [int(x) for x in np.random.default_rng(seed).permutation(batch.num_seqs)]
    tasks, nbytes = [], []
    for s in order:
        tasks.append(_compact(batch, [s]))
        L = int(batch.context_lens[s])
        nbytes.append(L * batch.num_kv_heads * batch.head_dim * 2 * e + per_seq_fixed +
                      ((L + batch.block_size - 1) // batch.block_size) * 4)

    def run(task):
        q, k, v, bt, cl = task
        orc.decode(q, k, v, bt, cl, batch.scale, batch.block_size, batch.num_kv_heads)

    with ThreadPoolExecutor(max_workers=cores) as ex:
        rounds, total, wall = 0, 0, 0.0
        while wall < seconds_target / cores or rounds == 0:
            t0 = time.perf_counter()
            list(ex.map(run, tasks))
            wall += time.perf_counter() - t0
            total += sum(nbytes)
            rounds += 1
            if rounds >= 50:
                break
    gbs = total / wall / 1e9
    desc = (f"all {batch.num_seqs} sequences x {rounds} round(s) on {cores} threads "
            f"(one sequence per task, fp64 oracle), {wall:.2f} s wall")
    return gbs, desc, cores


def _compact(batch, seqs):
    bt = batch.block_tables[seqs]
    used = sorted(set(int(x) for x in bt[bt >= 0].tolist()))
    remap = {old: new for new, old in enumerate(used)}
    nbt = bt.clone()
    flat = nbt.view(-1)
    for i in range(flat.numel()):
        x = int(flat[i])
        if x >= 0:
            flat[i] = remap[x]
    idx = torch.tensor(used if used else [0], dtype=torch.int64, device=batch.k_cache.device)
    return (batch.q[seqs].cpu().contiguous(), batch.k_cache[idx].cpu().contiguous(),
            batch.v_cache[idx].cpu().contiguous(), nbt.contiguous(), batch.context_lens[seqs].contiguous())


def run_reference(args, world, rank):
    """The reference arm: the fp64 oracle on the host cores, bounded sample per step."""
    if rank != 0:
        return None
    import workloads
    device = "cuda" if torch.cuda.is_available() else "cpu"
    batch = make_workload(args.workload, args.seed, device, args.block_size)
    per_step = max(1.0, 60.0 / max(1, args.steps + args.warmup))
    times, gbs_list, desc = [], [], ""
    for i in range(args.warmup + args.steps):
        gbs, desc, spent, n = oracle_sample(batch, per_step, seed=i)
        if i >= args.warmup:
            times.append(spent)
            gbs_list.append(gbs)
    value = statistics.mean(gbs_list)
    return {
        "metric": METRIC, "impl": "reference", "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * statistics.mean(times), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (same seeded workload as the GPU arm)",
        "config": {"workload": batch.name, "global_batch": batch.num_seqs},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": desc,
                         "cpu": cpu_model(), "host_cores": os.cpu_count()},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def measured_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured cuBLAS bf16 (burst)"
    return 1590.0, "fallback bf16"


def run_prefill(args, world, rank, local):
    """Chunked prefill through pa_prefill: Llama-3-8B heads, 8 sequences with
    contexts U[1024, 4096] whose newest U[256, 1024] tokens are the chunk."""
    import paged_kv_cache_449_b200 as pa
    import workloads
    from paged_kv_cache_449_b200 import build as pabuild
    pabuild.build()
    pa.load()
    b = workloads.chunked_prefill(seed=args.seed + rank, device="cuda", block_size=args.block_size or 16)
    qs = b.meta["query_start"]
    chunks = (qs[1:] - qs[:-1]).to(torch.int64)
    lens = b.context_lens.to(torch.int64)
    # every query row sees L - Q + i + 1 keys: QK^T and PV are 2 * D flops per key each
    visible = int(((lens - chunks) * chunks + chunks * (chunks + 1) // 2).sum())
    flops = 4 * b.head_dim * b.num_q_heads * visible
    dev = {k: getattr(b, k).cuda().contiguous() for k in ("q", "k_cache", "v_cache", "block_tables", "context_lens")}
    qsd = qs.cuda()
    out = torch.empty_like(dev["q"])
    maxq = int(chunks.max())
    stream = torch.cuda.current_stream()

    def one():
        pa.pa_prefill(out, dev["q"], dev["k_cache"], dev["v_cache"], dev["block_tables"], dev["context_lens"], qsd,
                      b.scale, max_context_len=b.max_context_len, max_query_len=maxq, stream=stream)

    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize()
    pa.pa_get_device_error()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    barrier(world)
    with ClockSampler(local) as clocks:
        t_busy = time.perf_counter() + 0.3
        while time.perf_counter() < t_busy:
            one()
            torch.cuda.synchronize()
        barrier(world)
        ev[0].record(stream)
        for _ in range(args.steps):
            one()
        ev[1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    if pa.pa_get_device_error() != 0:
        raise RuntimeError("device error word set during the timed steps")
    local_ms = ev[0].elapsed_time(ev[1]) / args.steps
    ms = reduce_max(local_ms, world)
    total = reduce_sum(flops, world)
    peak, kind = measured_tensor_peak()
    achieved = flops / (local_ms * 1e-3) / 1e12
    return {
        "metric": "paged chunked prefill TFLOP/s (Llama-3-8B attention shape)",
        "value": round(total / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) Q/K/V, seeded context and chunk lengths, shuffled block ids)",
        "config": {"workload": b.name, "global_batch": b.num_seqs, "query_tokens": int(chunks.sum()),
                   "context_len_mean": float(lens.float().mean()), "chunk_len_mean": float(chunks.float().mean()),
                   "num_q_heads": b.num_q_heads, "num_kv_heads": b.num_kv_heads, "head_dim": b.head_dim,
                   "block_size": b.block_size, "flops_per_step": flops, "parallelism": f"replicas x{world}",
                   "l2": "not flushed: compute-bound (the K/V of a sequence is reread by its query tiles)",
                   "mma": "tcgen05.mma kind::f16, M = 128 query rows, S / O / P in tensor memory, fp32 accumulate"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 3), "peak": peak, "peak_kind": kind,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": NCU_TRAFFIC.get(kernel_source_hash(PREFILL_SOURCES), {}).get(
                         (b.name if b.block_size == 16 else f"{b.name}_B{b.block_size}", "prefill"))},
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
    }


def run_blocks(args, world, rank, local):
    """Block copies through pa_copy_blocks: every block of the batch's
    sequences, K and V pools, per step."""
    import paged_kv_cache_449_b200 as pa
    from paged_kv_cache_449_b200 import build as pabuild
    pabuild.build()
    pa.load()
    batch = make_workload(args.workload, args.seed + rank, "cuda", args.block_size)
    B = batch.block_size
    k = batch.k_cache.contiguous()
    v = batch.v_cache.contiguous()
    ids = []
    for s in range(batch.num_seqs):
        n = (int(batch.context_lens[s]) + B - 1) // B
        ids += [int(x) for x in batch.block_tables[s, :n].tolist()]
    ids = sorted(set(ids))
    n = len(ids)
    block_bytes = batch.num_kv_heads * B * batch.head_dim * batch.elem_bytes
    stream = torch.cuda.current_stream()
    if args.op == "copy_blocks":
        used = set(ids)
        free = [i for i in range(batch.num_blocks) if i not in used][:n]
        n = len(free)
        mapping = torch.tensor([[a, b] for a, b in zip(ids, free)], dtype=torch.int64, device="cuda")
        dst_k, dst_v, src_k, src_v = k, v, k, v
        moved = 2 * n * block_bytes * 2          # K and V pools, read + write
        bound, peak, peak_kind = "hbm", *measured_peaks()
        peak_kind = f"{peak_kind} copy bandwidth (burst)"
    else:
        host_k = torch.empty((n,) + tuple(k.shape[1:]), dtype=k.dtype).pin_memory()
        host_v = torch.empty_like(host_k).pin_memory()
        if args.op == "swap_out":
            mapping = torch.tensor([[a, j] for j, a in enumerate(ids)], dtype=torch.int64, device="cuda")
            dst_k, dst_v, src_k, src_v = host_k, host_v, k, v
        else:
            mapping = torch.tensor([[j, a] for j, a in enumerate(ids)], dtype=torch.int64, device="cuda")
            dst_k, dst_v, src_k, src_v = k, v, host_k, host_v
        moved = 2 * n * block_bytes              # bytes across PCIe
        bound, peak, peak_kind = "pcie", PCIE_GEN5_X16_GBS, "nominal PCIe Gen5 x16, one direction"

    def one():
        pa.pa_copy_blocks(dst_k, dst_v, src_k, src_v, mapping, stream=stream)

    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize()
    pa.pa_get_device_error()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    barrier(world)
    with ClockSampler(local) as clocks:
        t_busy = time.perf_counter() + 0.3
        while time.perf_counter() < t_busy:
            one()
            torch.cuda.synchronize()
        barrier(world)
        ev[0].record(stream)
        for _ in range(args.steps):
            one()
        ev[1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    if pa.pa_get_device_error() != 0:
        raise RuntimeError("device error word set during the timed steps")
    ms = reduce_max(ev[0].elapsed_time(ev[1]) / args.steps, world)
    total = reduce_sum(moved, world)
    achieved = moved / (ev[0].elapsed_time(ev[1]) / args.steps * 1e-3) / 1e9
    return {
        "metric": {"copy_blocks": "paged KV block copy (copy-on-write duplicate) GB/s",
                   "swap_out": "paged KV block swap-out to host GB/s",
                   "swap_in": "paged KV block swap-in from host GB/s"}[args.op],
        "value": round(total / (ms * 1e-3) / 1e9, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32"}[batch.dtype],
        "data": "synthetic (the decode workload's pools and block tables)",
        "config": {"workload": batch.name, "op": args.op, "blocks": n, "block_bytes_per_pool": block_bytes,
                   "bytes_counted": "K and V read + written" if bound == "hbm" else "K and V moved across PCIe",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "peak_kind": peak_kind,
                     "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": None},
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
    }


def main(argv=None):
    args = parse_args(argv)
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            res = run_reference(args, world, rank)
            if res is not None:
                print(json.dumps(res), flush=True)
            return
        if args.op == "block_step":
            import paged_kv_cache_449_b200 as pa
            from paged_kv_cache_449_b200 import build as pabuild
            pabuild.build()
            pa.load()
            peak, _ = measured_peaks()
            with ClockSampler(local) as clocks:
                res = block_manager_step(args.seed + rank, args.steps, max(3, args.warmup), world, peak)
            res = dict(res, metric="paged decode step through the device block manager, KV GB/s",
                       value=res["gb_per_s"], unit="GB/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
                       higher_is_better=True, clocks=clocks.summary())
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        if args.op != "decode":
            res = (run_prefill if args.op == "prefill" else run_blocks)(args, world, rank, local)
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        res, batch = run_gpu(args, world, rank, local)
        headline = (args.workload == "llama3_8b_decode" and args.mode == "append" and args.kv == "bf16"
                    and args.block_size is None and not args.graph)
        if headline and not args.no_configs:
            res["configs"] = config_lines(args, world, rank)
            res["gpu_launches_configs"] = sum(int(v.get("gpu_launches", 0)) for v in res["configs"].values())
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline and args.kv == "bf16":
                gbs1, desc1, spent, n = oracle_sample(batch, args.cpu_sample_seconds)
                try:
                    gbs, desc, cores = oracle_sample_all_cores(batch, args.cpu_sample_seconds)
                except (OSError, RuntimeError) as err:   # no worker threads on this host: one core only
                    gbs, desc, cores = gbs1, f"{desc1} (threads unavailable: {err})", 1
                res["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                                       "sample": desc, "one_core_value": round(gbs1, 4), "one_core_sample": desc1,
                                       "cpu": cpu_model(), "host_cores": os.cpu_count()}
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
