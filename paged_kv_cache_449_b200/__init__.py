"""Python binding of libpa — B200 paged KV-cache attention (C ABI in include/pa.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libpa.so.  There is no fallback; if the library is missing the
calls raise.  Tensors are torch CUDA tensors; pools are shaped
[num_blocks, num_kv_heads, head_dim // X, block_size, X] (X = 16 bytes /
element size), so block_size, num_blocks and the head counts are read off the
tensor shapes.  Calls run on the current torch CUDA stream unless `stream`
(a torch.cuda.Stream or a raw cudaStream_t int) is given.
"""

from __future__ import annotations

import ctypes
import functools
import os

import torch

__all__ = ["pa_reshape_and_cache", "pa_decode", "pa_decode_append", "pa_decode_splitk",
           "pa_decode_splitk_workspace_size",
           "Counters",
           "pa_decode_splitk_static", "SPLITK_STATIC_SCRATCH_BYTES",
           "pa_get_device_error", "pa_status_string", "PagedAttentionError", "library_path", "load",
           "pool_shape", "DEVERR_BLOCK_ID", "DEVERR_CONTEXT_LEN", "DEVERR_SLOT", "DEVERR_TIMEOUT",
           "DEVERR_SEQ_ORDER", "longest_first", "pa_copy_blocks", "pa_reshape_and_cache_fp8", "pa_decode_fp8",
           "pa_decode_splitk_fp8", "fp8_pool_shape", "pa_prefill", "pa_decode_append_fp8",
           "pa_blocks_init", "pa_blocks_append", "pa_blocks_fork", "pa_blocks_release",
           "DEVERR_NO_FREE_BLOCK", "DEVERR_REF_COUNT", "DEVERR_SHARED_BLOCK", "DEVERR_PREFIX",
           "pa_decode_shared_prefix", "pa_decode_shared_prefix_workspace_size", "prepare_decode_shared_prefix"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_F32, PA_F16, PA_BF16 = 0, 1, 2
_DTYPE = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16}
STATUS = {0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED", 3: "PA_ERR_WORKSPACE", 4: "PA_ERR_CUDA"}
DEVERR_BLOCK_ID, DEVERR_CONTEXT_LEN, DEVERR_SLOT, DEVERR_TIMEOUT, DEVERR_SEQ_ORDER = 1, 2, 4, 8, 16
DEVERR_NO_FREE_BLOCK, DEVERR_REF_COUNT, DEVERR_SHARED_BLOCK, DEVERR_PREFIX = 32, 64, 128, 256


class PagedAttentionError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


_lib = None


def library_path() -> str:
    return _LIB_PATH


def load() -> ctypes.CDLL:
    """Load libpa.so (built in-tree by paged_kv_cache_449_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"libpa.so is not built ({_LIB_PATH}); run paged_kv_cache_449_b200/build.py")
    _lib = load_library(_LIB_PATH)
    return _lib


def load_library(path: str) -> ctypes.CDLL:
    """Open a build of the library at `path` with the argument types of every
    entry point declared in include/pa.h."""
    lib = ctypes.CDLL(path)
    c = ctypes
    P, I, I64, F, SZ = c.c_void_p, c.c_int, c.c_int64, c.c_float, c.c_size_t
    lib.pa_reshape_and_cache.restype = I
    lib.pa_reshape_and_cache.argtypes = [P, P, P, P, P, I64, I, I, I, I64, I, P]
    decode_args = [P, P, P, P, P, P, F, I, I, I, I, I, I, I, I64, I]
    lib.pa_decode.restype = I
    lib.pa_decode.argtypes = decode_args + [P, P]
    lib.pa_decode_append.restype = I
    lib.pa_decode_append.argtypes = [P, P, P, P] + decode_args[2:] + [P, P, P]
    lib.pa_decode_shared_prefix_workspace_size.restype = I
    lib.pa_decode_shared_prefix_workspace_size.argtypes = [I, I, I, I, I, c.POINTER(SZ)]
    lib.pa_decode_shared_prefix.restype = I
    lib.pa_decode_shared_prefix.argtypes = [P, P, P, P] + decode_args[2:] + [I, P, SZ, P, I64, P, P]
    lib.pa_decode_splitk_workspace_size.restype = I
    lib.pa_decode_splitk_workspace_size.argtypes = [I, I, I, I, I, c.POINTER(SZ)]
    lib.pa_decode_splitk.restype = I
    lib.pa_decode_splitk.argtypes = decode_args + [I, P, SZ, P, I64, P, P]
    lib.pa_decode_splitk_static.restype = I
    lib.pa_decode_splitk_static.argtypes = decode_args + [I, P]
    lib.pa_reshape_and_cache_fp8.restype = I
    lib.pa_reshape_and_cache_fp8.argtypes = [P, P, P, P, P, P, P, I64, I, I, I, I64, I, P]
    fp8_args = [P, P, P, P, P, P, P, P, F, I, I, I, I, I, I, I, I64, I]
    lib.pa_decode_fp8.restype = I
    lib.pa_decode_fp8.argtypes = fp8_args + [P, P]
    lib.pa_decode_append_fp8.restype = I
    lib.pa_decode_append_fp8.argtypes = [P, P, P, P] + fp8_args[2:] + [P, P, P]
    lib.pa_decode_splitk_fp8.restype = I
    lib.pa_decode_splitk_fp8.argtypes = fp8_args + [I, P, SZ, P, I64, P, P]
    lib.pa_prefill.restype = I
    lib.pa_prefill.argtypes = [P, P, P, P, P, P, P, F, I, I, I, I, I, I, I, I, I64, I, P]
    lib.pa_copy_blocks.restype = I
    lib.pa_copy_blocks.argtypes = [P, P, P, P, P, I64, I, I, I, I64, I64, I, P]
    lib.pa_blocks_init.restype = I
    lib.pa_blocks_init.argtypes = [P, P, P, I64, P]
    lib.pa_blocks_append.restype = I
    lib.pa_blocks_append.argtypes = [P, P, P, P, P, P, P, I64, P, I, I, I, I64, P]
    lib.pa_blocks_fork.restype = I
    lib.pa_blocks_fork.argtypes = [P, P, P, P, I, I, I, I, I64, P]
    lib.pa_blocks_release.restype = I
    lib.pa_blocks_release.argtypes = [P, P, P, P, P, P, I, I, I, I, I64, P]
    lib.pa_get_device_error.restype = I
    lib.pa_get_device_error.argtypes = [P, c.POINTER(c.c_int32)]
    lib.pa_status_string.restype = c.c_char_p
    lib.pa_status_string.argtypes = [I]
    return lib


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, what: str):
    if status != 0:
        raise PagedAttentionError(status, what)


def pool_shape(num_blocks: int, num_kv_heads: int, head_dim: int, block_size: int, dtype: torch.dtype):
    x = 16 // torch.tensor([], dtype=dtype).element_size()
    return (num_blocks, num_kv_heads, head_dim // x, block_size, x)


def _pool_dims(k_cache: torch.Tensor):
    if k_cache.dim() != 5:
        raise ValueError("pools must be shaped [num_blocks, num_kv_heads, head_dim // X, block_size, X]")
    n, hkv, dv, b, x = k_cache.shape
    return n, hkv, dv * x, b


def _tensor_device(args, kwargs):
    """The one CUDA device that every CUDA tensor argument lives on (None if
    there is none).  The library launches on the current device, so a call
    whose tensors sit on different GPUs is refused: a kernel would otherwise
    dereference another GPU's pointers."""
    found = None
    for a in list(args) + list(kwargs.values()):
        dev = None
        if isinstance(a, torch.Tensor) and a.is_cuda:
            dev = a.device
        elif isinstance(a, torch.cuda.Stream):
            dev = a.device
        if dev is None:
            continue
        if found is None:
            found = dev
        elif dev != found:
            raise ValueError(f"tensors and stream must share one CUDA device (found {found} and {dev})")
    return found


def _on_tensor_device(fn):
    """Runs fn with the device of its CUDA tensor arguments current, so the
    launch, the default stream and any per-device state (shared-memory limits,
    the static split-K array) belong to the GPU that holds the data."""
    @functools.wraps(fn)
    def call(*args, **kwargs):
        dev = _tensor_device(args, kwargs)
        if dev is None or dev.index == torch.cuda.current_device():
            return fn(*args, **kwargs)
        with torch.cuda.device(dev):
            return fn(*args, **kwargs)
    return call


def _dev_ptr(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def pa_status_string(status: int) -> str:
    return load().pa_status_string(int(status)).decode()


@_on_tensor_device
def pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, stream=None):
    """Write key/value [T, Hkv, D] into the pools at slot_mapping (int64 [T])."""
    lib = load()
    n, hkv, d, b = _pool_dims(k_cache)
    T = key.shape[0]
    _check(lib.pa_reshape_and_cache(
        _dev_ptr(key, "key"), _dev_ptr(value, "value"), _dev_ptr(k_cache, "k_cache"),
        _dev_ptr(v_cache, "v_cache"), _dev_ptr(slot_mapping, "slot_mapping"), T, hkv, d, b, n,
        _DTYPE[key.dtype], _stream(stream)), "pa_reshape_and_cache")


def _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, scale, max_context_len):
    n, hkv, d, b = _pool_dims(k_cache)
    S, Hq, D = q.shape
    if max_context_len is None:
        max_context_len = int(block_tables.shape[1]) * b
    return [_dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
            _dev_ptr(block_tables, "block_tables"), _dev_ptr(context_lens, "context_lens"), float(scale), b, S,
            Hq, hkv, D, int(block_tables.shape[1]), int(max_context_len), n, _DTYPE[q.dtype]]


def longest_first(context_lens) -> torch.Tensor:
    """The scheduling hint `seq_order` for a batch whose context lengths the
    host knows: sequence indices by decreasing length (ties by index), as a
    CPU int32 tensor to be copied to the device with the other step inputs."""
    lens = torch.as_tensor(context_lens).detach().to("cpu", torch.int64).reshape(-1)
    return torch.sort(-lens, stable=True).indices.to(torch.int32)


def _order_ptr(seq_order, num_seqs):
    if seq_order is None:
        return None
    if seq_order.dtype != torch.int32 or seq_order.numel() != num_seqs:
        raise ValueError("seq_order must be an int32 permutation of range(num_seqs)")
    return _dev_ptr(seq_order, "seq_order")


@_on_tensor_device
def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, max_context_len=None, stream=None,
              seq_order=None):
    """Paged decode attention, one launch.  out, q: [S, Hq, D]; block_tables
    int32 [S, max_blocks]; context_lens int32 [S]; seq_order: None or an int32
    device permutation of range(S), the order in which sequences are started
    (see longest_first); the result does not depend on it."""
    lib = load()
    args = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, scale, max_context_len)
    _check(lib.pa_decode(*args, _order_ptr(seq_order, q.shape[0]), _stream(stream)), "pa_decode")


def _counts_ptr(ref_counts, num_blocks):
    if ref_counts is None:
        return None
    if ref_counts.dtype != torch.int32 or ref_counts.numel() != num_blocks:
        raise ValueError("ref_counts must be int32 [num_blocks]")
    return _dev_ptr(ref_counts, "ref_counts")


def _append_args(out, q, key, value, k_cache, v_cache, block_tables, context_lens, scale, max_context_len,
                 seq_order, ref_counts):
    args = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, scale, max_context_len)
    return [args[0], args[1], _dev_ptr(key, "key"), _dev_ptr(value, "value"), *args[2:],
            _counts_ptr(ref_counts, k_cache.shape[0]), _order_ptr(seq_order, q.shape[0])]


@_on_tensor_device
def pa_decode_append(out, q, key, value, k_cache, v_cache, block_tables, context_lens, scale, max_context_len=None,
                     stream=None, seq_order=None, ref_counts=None):
    """One decode step: write each sequence's newest token (key/value [S, Hkv,
    D]) at position context_lens[s]-1, then attend over the whole context.
    ref_counts (int32 [num_blocks], optional): a sequence whose newest block
    is held by others is not written (DEVERR_SHARED_BLOCK)."""
    lib = load()
    args = _append_args(out, q, key, value, k_cache, v_cache, block_tables, context_lens, scale, max_context_len,
                        seq_order, ref_counts)
    _check(lib.pa_decode_append(*args, _stream(stream)), "pa_decode_append")


class Prepared:
    """One entry-point call whose arguments were checked and marshalled once:
    calling it (optionally with a stream; the current stream otherwise) makes
    the same C-ABI call again, with the same pointers and sizes, on the device
    that holds its tensors.  For a step repeated over fixed buffers, as a
    serving loop does, it spares the per-call argument work; the buffers'
    contents may change between calls, their storage may not (the object keeps
    a reference to each tensor)."""

    def __init__(self, name, args, device, tensors):
        self._fn = getattr(load(), name)
        self._name = name
        # each argument already of its ctypes type, so a call converts nothing
        # but the stream
        types = self._fn.argtypes[:len(args)]
        self._args = tuple(a if isinstance(a, t) else t(a) for a, t in zip(args, types))
        self._device = device.index
        self._tensors = tensors

    def __call__(self, stream=None):
        if torch.cuda.current_device() != self._device:
            with torch.cuda.device(self._device):
                return self(stream)
        _check(self._fn(*self._args, _stream(stream)), self._name)


def prepare_decode_append(out, q, key, value, k_cache, v_cache, block_tables, context_lens, scale,
                          max_context_len=None, seq_order=None, ref_counts=None) -> Prepared:
    """pa_decode_append's arguments checked and marshalled once (see Prepared)."""
    tensors = (out, q, key, value, k_cache, v_cache, block_tables, context_lens, seq_order, ref_counts)
    dev = _tensor_device(tensors, {})
    if dev is None:
        raise ValueError("pa_decode_append takes CUDA tensors")
    args = _append_args(out, q, key, value, k_cache, v_cache, block_tables, context_lens, scale, max_context_len,
                        seq_order, ref_counts)
    return Prepared("pa_decode_append", args, dev, tensors)


def pa_decode_shared_prefix_workspace_size(num_seqs, num_q_heads, head_dim, prefix_blocks, block_size) -> int:
    lib = load()
    size = ctypes.c_size_t(0)
    _check(lib.pa_decode_shared_prefix_workspace_size(num_seqs, num_q_heads, head_dim, int(prefix_blocks),
                                                      int(block_size), ctypes.byref(size)),
           "pa_decode_shared_prefix_workspace_size")
    return int(size.value)


def _shared_prefix_args(out, q, key, value, k_cache, v_cache, block_tables, context_lens, scale, prefix_blocks,
                        max_context_len, workspace, ref_counts, counters):
    if (key is None) != (value is None):
        raise ValueError("key and value go together (both None: no append)")
    S, Hq, D = q.shape
    b = k_cache.shape[3]
    if workspace is None:
        need = pa_decode_shared_prefix_workspace_size(S, Hq, D, prefix_blocks, b)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    args = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, scale, max_context_len)
    kp = None if key is None else _dev_ptr(key, "key")
    vp = None if value is None else _dev_ptr(value, "value")
    if counters is None:
        counters = _default_counters.setdefault(q.device.index, Counters())
    buf = counters.get(S * k_cache.shape[1], q.device) if isinstance(counters, Counters) else counters
    return [args[0], args[1], kp, vp, *args[2:], int(prefix_blocks), _dev_ptr(workspace, "workspace"),
            workspace.numel() * workspace.element_size(), _dev_ptr(buf, "counters"), buf.numel(),
            _counts_ptr(ref_counts, k_cache.shape[0])], workspace, buf


@_on_tensor_device
def pa_decode_shared_prefix(out, q, key, value, k_cache, v_cache, block_tables, context_lens, scale, prefix_blocks,
                            max_context_len=None, workspace=None, stream=None, ref_counts=None, counters=None):
    """Decode (key = value = None) or decode with append (key/value [S, Hkv,
    D]) for a batch whose rows all begin with the same prefix_blocks physical
    blocks: the prefix is attended once per kv head for every sequence on the
    tensor cores, each sequence's own blocks as in pa_decode, and the two
    merged.  `workspace`: a CUDA uint8 tensor of at least
    pa_decode_shared_prefix_workspace_size(...) bytes (allocated here if None);
    `counters`: a Counters or a zeroed int32 tensor (a per-device default if
    None)."""
    lib = load()
    args, _, _ = _shared_prefix_args(out, q, key, value, k_cache, v_cache, block_tables, context_lens, scale,
                                     prefix_blocks, max_context_len, workspace, ref_counts, counters)
    _check(lib.pa_decode_shared_prefix(*args, _stream(stream)), "pa_decode_shared_prefix")


def prepare_decode_shared_prefix(out, q, key, value, k_cache, v_cache, block_tables, context_lens, scale,
                                 prefix_blocks, max_context_len=None, workspace=None, ref_counts=None,
                                 counters=None) -> Prepared:
    """pa_decode_shared_prefix's arguments checked and marshalled once (see Prepared)."""
    tensors = (out, q, key, value, k_cache, v_cache, block_tables, context_lens, workspace, ref_counts)
    dev = _tensor_device(tensors + ((counters,) if isinstance(counters, torch.Tensor) else ()), {})
    if dev is None:
        raise ValueError("pa_decode_shared_prefix takes CUDA tensors")
    args, workspace, buf = _shared_prefix_args(out, q, key, value, k_cache, v_cache, block_tables, context_lens,
                                               scale, prefix_blocks, max_context_len, workspace, ref_counts,
                                               counters)
    return Prepared("pa_decode_shared_prefix", args, dev, tensors + (workspace, buf))


def pa_decode_splitk_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len, partition_size=512) -> int:
    lib = load()
    size = ctypes.c_size_t(0)
    _check(lib.pa_decode_splitk_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len,
                                               partition_size, ctypes.byref(size)),
           "pa_decode_splitk_workspace_size")
    return int(size.value)


class Counters:
    """Zero-initialised int32 arrival counters for the fused split-K merge
    (pa_decode_splitk with fused=True); the kernels leave
    them at zero, so one array is reused across calls of any shape on a
    stream.  Grows on demand."""

    def __init__(self):
        self.buf = None

    def get(self, n: int, device) -> torch.Tensor:
        device = torch.device(device)
        if self.buf is None or self.buf.numel() < n or self.buf.device != device:
            self.buf = torch.zeros(max(n, 4), dtype=torch.int32, device=device)
        return self.buf


_default_counters: dict = {}
_splitk_ws_cache: dict = {}


@_on_tensor_device
def pa_decode_splitk(out, q, k_cache, v_cache, block_tables, context_lens, scale, max_context_len,
                     partition_size=512, workspace=None, fused=True, counters=None, stream=None, seq_order=None):
    """Split-K paged decode (partitions of partition_size tokens + log-sum-exp
    merge).  `workspace` is a CUDA uint8 tensor of at least
    pa_decode_splitk_workspace_size(...) bytes (allocated here if None).
    fused=True merges inside the partition kernel using `counters` (a
    Counters; a per-device default if None); fused=False launches the
    separate merge kernel."""
    lib = load()
    S, Hq, D = q.shape
    hkv = k_cache.shape[1]
    key = (S, Hq, D, int(max_context_len), partition_size)
    need = _splitk_ws_cache.get(key)
    if need is None:
        need = _splitk_ws_cache[key] = pa_decode_splitk_workspace_size(S, Hq, D, int(max_context_len),
                                                                        partition_size)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    cptr, ncount = None, 0
    if fused:
        if counters is None:
            counters = _default_counters.setdefault(q.device.index, Counters())
        buf = counters.get(S * hkv, q.device) if isinstance(counters, Counters) else counters
        cptr, ncount = _dev_ptr(buf, "counters"), buf.numel()
    args = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, scale, max_context_len)
    _check(lib.pa_decode_splitk(*args, int(partition_size), _dev_ptr(workspace, "workspace"),
                                workspace.numel() * workspace.element_size(), cptr, ncount,
                                _order_ptr(seq_order, S), _stream(stream)),
           "pa_decode_splitk")


SPLITK_STATIC_SCRATCH_BYTES = 16 << 20


@_on_tensor_device
def pa_decode_splitk_static(out, q, k_cache, v_cache, block_tables, context_lens, scale, max_context_len,
                            partition_size=512, stream=None):
    """Split-K paged decode that allocates nothing: for callers that cannot
    allocate device memory when they launch work (runtime plugins handed only
    inputs and outputs, latency-critical loops that must not trigger
    cudaMalloc's implicit synchronisation).  The partials live in a fixed
    SPLITK_STATIC_SCRATCH_BYTES array inside libpa's device image; larger
    requests raise PagedAttentionError (PA_ERR_WORKSPACE).  All calls on a
    device share that array, so calls must not overlap on the GPU.  The first
    call on a device resolves the array's address; make it before any stream
    capture."""
    lib = load()
    args = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, scale, max_context_len)
    _check(lib.pa_decode_splitk_static(*args, int(partition_size), _stream(stream)), "pa_decode_splitk_static")


def _accessible_ptr(t: torch.Tensor, name: str) -> int:
    """A CUDA tensor, or a page-locked CPU tensor (the device reaches it
    through the unified address space)."""
    if not (t.is_cuda or (t.device.type == "cpu" and t.is_pinned())):
        raise ValueError(f"{name} must be a CUDA tensor or a pinned CPU tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


@_on_tensor_device
def pa_copy_blocks(dst_k_cache, dst_v_cache, src_k_cache, src_v_cache, block_mapping, stream=None):
    """Copy whole blocks (src, dst) = block_mapping[i] (int64 [n, 2], on the
    device or pinned) from the source pools to the destination pools.  Same
    pools on both sides: copy-on-write duplicates; a pinned CPU pool on one
    side: swap-out / swap-in.  Pools are [num_blocks, Hkv, D // X, B, X]."""
    lib = load()
    n_src, hkv, d, b = _pool_dims(src_k_cache)
    n_dst, hkv2, d2, b2 = _pool_dims(dst_k_cache)
    if (hkv, d, b) != (hkv2, d2, b2) or src_k_cache.dtype != dst_k_cache.dtype:
        raise ValueError("source and destination pools differ in shape or dtype")
    if block_mapping.dtype != torch.int64 or block_mapping.dim() != 2 or block_mapping.shape[1] != 2:
        raise ValueError("block_mapping must be int64 [n, 2]")
    _check(lib.pa_copy_blocks(
        _accessible_ptr(dst_k_cache, "dst_k_cache"), _accessible_ptr(dst_v_cache, "dst_v_cache"),
        _accessible_ptr(src_k_cache, "src_k_cache"), _accessible_ptr(src_v_cache, "src_v_cache"),
        _accessible_ptr(block_mapping, "block_mapping"), int(block_mapping.shape[0]), hkv, d, b, n_src, n_dst,
        _DTYPE[src_k_cache.dtype], _stream(stream)), "pa_copy_blocks")


# ---- 8-bit (e4m3) pools: uint8 tensors shaped [num_blocks, Hkv, D // 16, B, 16] (one B*D-byte tile per
#      (block, head); inside a tile K and V keep the byte orders of pa.h), fp32 scales [Hkv] per pool

def fp8_pool_shape(num_blocks, num_kv_heads, head_dim, block_size):
    return (num_blocks, num_kv_heads, head_dim // 16, block_size, 16)


def _scale_ptr(t, name):
    if t.dtype != torch.float32:
        raise ValueError(f"{name} must be float32 [num_kv_heads]")
    return _dev_ptr(t, name)


@_on_tensor_device
def pa_reshape_and_cache_fp8(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale, stream=None):
    """Quantise key/value [T, Hkv, D] to e4m3 codes (x / scale of the kv head)
    and write them into the 8-bit pools at slot_mapping (int64 [T])."""
    lib = load()
    if k_cache.dtype != torch.uint8:
        raise ValueError("8-bit pools are uint8 tensors")
    n, hkv, d, b = _pool_dims(k_cache)
    _check(lib.pa_reshape_and_cache_fp8(
        _dev_ptr(key, "key"), _dev_ptr(value, "value"), _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
        _dev_ptr(slot_mapping, "slot_mapping"), _scale_ptr(k_scale, "k_scale"), _scale_ptr(v_scale, "v_scale"),
        key.shape[0], hkv, d, b, n, _DTYPE[key.dtype], _stream(stream)), "pa_reshape_and_cache_fp8")


def _fp8_args(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale, max_context_len):
    if k_cache.dtype != torch.uint8:
        raise ValueError("8-bit pools are uint8 tensors")
    a = _decode_args(out, q, k_cache, v_cache, block_tables, context_lens, scale, max_context_len)
    return a[:4] + [_scale_ptr(k_scale, "k_scale"), _scale_ptr(v_scale, "v_scale")] + a[4:]


@_on_tensor_device
def pa_decode_fp8(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale,
                  max_context_len=None, stream=None, seq_order=None):
    """pa_decode over 8-bit pools; q/out fp16 or bf16."""
    lib = load()
    args = _fp8_args(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale, max_context_len)
    _check(lib.pa_decode_fp8(*args, _order_ptr(seq_order, q.shape[0]), _stream(stream)), "pa_decode_fp8")


def _append_fp8_args(out, q, key, value, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale,
                     max_context_len, seq_order, ref_counts):
    args = _fp8_args(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale, max_context_len)
    return [args[0], args[1], _dev_ptr(key, "key"), _dev_ptr(value, "value"), *args[2:],
            _counts_ptr(ref_counts, k_cache.shape[0]), _order_ptr(seq_order, q.shape[0])]


@_on_tensor_device
def pa_decode_append_fp8(out, q, key, value, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                         scale, max_context_len=None, stream=None, seq_order=None, ref_counts=None):
    """One decode step over 8-bit pools: quantise and write each sequence's
    newest token (key/value [S, Hkv, D]) at position context_lens[s]-1, then
    attend over the whole context (one launch).  ref_counts as in
    pa_decode_append."""
    lib = load()
    args = _append_fp8_args(out, q, key, value, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                            scale, max_context_len, seq_order, ref_counts)
    _check(lib.pa_decode_append_fp8(*args, _stream(stream)), "pa_decode_append_fp8")


def prepare_decode_append_fp8(out, q, key, value, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                              scale, max_context_len=None, seq_order=None, ref_counts=None) -> Prepared:
    """pa_decode_append_fp8's arguments checked and marshalled once (see Prepared)."""
    tensors = (out, q, key, value, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, seq_order,
               ref_counts)
    dev = _tensor_device(tensors, {})
    if dev is None:
        raise ValueError("pa_decode_append_fp8 takes CUDA tensors")
    args = _append_fp8_args(out, q, key, value, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                            scale, max_context_len, seq_order, ref_counts)
    return Prepared("pa_decode_append_fp8", args, dev, tensors)


@_on_tensor_device
def pa_decode_splitk_fp8(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale,
                         max_context_len, partition_size=512, workspace=None, fused=True, counters=None,
                         stream=None, seq_order=None):
    """pa_decode_splitk over 8-bit pools (workspace and counters as there)."""
    lib = load()
    S, Hq, D = q.shape
    hkv = k_cache.shape[1]
    need = pa_decode_splitk_workspace_size(S, Hq, D, int(max_context_len), partition_size)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    cptr, ncount = None, 0
    if fused:
        if counters is None:
            counters = _default_counters.setdefault(q.device.index, Counters())
        buf = counters.get(S * hkv, q.device) if isinstance(counters, Counters) else counters
        cptr, ncount = _dev_ptr(buf, "counters"), buf.numel()
    args = _fp8_args(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale, max_context_len)
    _check(lib.pa_decode_splitk_fp8(*args, int(partition_size), _dev_ptr(workspace, "workspace"),
                                    workspace.numel() * workspace.element_size(), cptr, ncount,
                                    _order_ptr(seq_order, S), _stream(stream)), "pa_decode_splitk_fp8")


@_on_tensor_device
def pa_prefill(out, q, k_cache, v_cache, block_tables, context_lens, query_start, scale, max_context_len=None,
               max_query_len=None, stream=None):
    """Causal chunked prefill: q/out [T, Hq, D] (fp16/bf16); query_start int32
    [S + 1] on the device; sequence s's chunk is its newest Q_s tokens."""
    lib = load()
    n, hkv, d, b = _pool_dims(k_cache)
    T, Hq, D = q.shape
    S = int(context_lens.numel())
    if max_context_len is None:
        max_context_len = int(block_tables.shape[1]) * b
    if max_query_len is None:
        max_query_len = T
    _check(lib.pa_prefill(
        _dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
        _dev_ptr(block_tables, "block_tables"), _dev_ptr(context_lens, "context_lens"),
        _dev_ptr(query_start, "query_start"), float(scale), b, S, Hq, hkv, D, int(block_tables.shape[1]),
        int(max_context_len), int(max_query_len), n, _DTYPE[q.dtype], _stream(stream)), "pa_prefill")


# ---- block management: ref_counts / free_ids int32 [N], free_state int64 [2] (head, tail), block_tables
#      int32 [S, max_blocks], context_lens int32 [S], all on one device

def _typed(t, dtype, name):
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    return _dev_ptr(t, name)


def _state_ptrs(ref_counts, free_ids, free_state):
    if ref_counts.numel() != free_ids.numel() or free_state.numel() != 2:
        raise ValueError("ref_counts and free_ids hold num_blocks entries, free_state two")
    return (_typed(ref_counts, torch.int32, "ref_counts"), _typed(free_ids, torch.int32, "free_ids"),
            _typed(free_state, torch.int64, "free_state"))


def _rows(block_tables, context_lens):
    if block_tables.dim() != 2 or context_lens.numel() != block_tables.shape[0]:
        raise ValueError("block_tables is [num_seqs, max_blocks], context_lens [num_seqs]")
    return (_typed(block_tables, torch.int32, "block_tables"), _typed(context_lens, torch.int32, "context_lens"),
            int(block_tables.shape[0]), int(block_tables.shape[1]))


@_on_tensor_device
def pa_blocks_init(ref_counts, free_ids, free_state, stream=None):
    """Every block free (the ring 0..N-1), every count zero."""
    lib = load()
    r, f, st = _state_ptrs(ref_counts, free_ids, free_state)
    _check(lib.pa_blocks_init(r, f, st, ref_counts.numel(), _stream(stream)), "pa_blocks_init")


@_on_tensor_device
def pa_blocks_append(block_tables, context_lens, num_new_tokens, ref_counts, free_ids, free_state, slot_mapping,
                     copy_pairs, block_size, stream=None):
    """One step: sequence s takes num_new_tokens[s] (int32 [S]) new positions.
    Writes the packed slots (int64, at least sum(num_new_tokens) entries) and
    the copy-on-write pairs (int64 [S, 2]) and updates the tables, lengths,
    counts and free ring in place."""
    lib = load()
    bt, cl, S, mb = _rows(block_tables, context_lens)
    r, f, st = _state_ptrs(ref_counts, free_ids, free_state)
    if num_new_tokens.numel() != S or copy_pairs.shape != (S, 2):
        raise ValueError("num_new_tokens is [num_seqs], copy_pairs [num_seqs, 2]")
    _check(lib.pa_blocks_append(bt, cl, _typed(num_new_tokens, torch.int32, "num_new_tokens"), r, f, st,
                                _typed(slot_mapping, torch.int64, "slot_mapping"), slot_mapping.numel(),
                                _typed(copy_pairs, torch.int64, "copy_pairs"), S, mb, int(block_size),
                                ref_counts.numel(), _stream(stream)), "pa_blocks_append")


@_on_tensor_device
def pa_blocks_fork(block_tables, context_lens, ref_counts, forks, block_size, stream=None):
    """forks: int32 [n, 3] rows (parent, child, length), applied in order."""
    lib = load()
    bt, cl, S, mb = _rows(block_tables, context_lens)
    if forks.dim() != 2 or forks.shape[1] != 3:
        raise ValueError("forks is int32 [n, 3]")
    _check(lib.pa_blocks_fork(bt, cl, _typed(ref_counts, torch.int32, "ref_counts"),
                              _typed(forks, torch.int32, "forks"), int(forks.shape[0]), S, mb, int(block_size),
                              ref_counts.numel(), _stream(stream)), "pa_blocks_fork")


@_on_tensor_device
def pa_blocks_release(block_tables, context_lens, ref_counts, free_ids, free_state, seqs, block_size, stream=None):
    """Free the sequences seqs (int32 [n]) in order."""
    lib = load()
    bt, cl, S, mb = _rows(block_tables, context_lens)
    r, f, st = _state_ptrs(ref_counts, free_ids, free_state)
    _check(lib.pa_blocks_release(bt, cl, r, f, st, _typed(seqs, torch.int32, "seqs"), seqs.numel(), S, mb,
                                 int(block_size), ref_counts.numel(), _stream(stream)), "pa_blocks_release")


def pa_get_device_error(stream=None) -> int:
    """Read and clear the device error word (synchronises the stream)."""
    lib = load()
    code = ctypes.c_int32(0)
    _check(lib.pa_get_device_error(_stream(stream), ctypes.byref(code)), "pa_get_device_error")
    return int(code.value)
