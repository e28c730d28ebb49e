"""Paged-attention oracle — TEST INFRASTRUCTURE ONLY.

A ctypes wrapper around ``pa_oracle.cpp``: a plain, slow, single-threaded fp64
C++ restatement of the KV-cache write and of paged decode attention, written
from the pages' description of PagedAttention (see the header of
``pa_oracle.cpp`` for the page titles and sections it follows).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module.  It does not import the product package, and the
product package does not import it.  Arrays cross as torch CPU tensors (bf16
has no numpy dtype); this module does argument marshalling only.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

# Element type codes of the oracle (its own numbering, same meaning as the
# library's: 0 fp32, 1 fp16, 2 bf16).
DTYPE_CODE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}

ERRORS = {0: "ok", 1: "bad argument", 2: "block id out of range",
          3: "context length out of range", 4: "slot out of range"}


class OracleError(RuntimeError):
    pass


def build(src: str = _SRC, out: str = _LIB, force: bool = False) -> str:
    """Compile the oracle with g++ (-O2, no fast-math: IEEE fp64 throughout)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run(["g++", "-O2", "-std=c++17", "-fno-fast-math", "-ffp-contract=off",
                    "-shared", "-fPIC", "-o", tmp, src], check=True)
    os.replace(tmp, out)
    return out


class Oracle:
    """One loaded copy of the oracle library (tests may load planted-mistake
    variants built from a modified copy of the source)."""

    def __init__(self, path: str | None = None):
        self.path = path or build()
        lib = ctypes.CDLL(self.path)
        c = ctypes
        lib.oracle_reshape_and_cache.restype = c.c_int
        lib.oracle_reshape_and_cache.argtypes = [
            c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_int64,
            c.c_int, c.c_int, c.c_int, c.c_int64, c.c_int]
        decode_args = [c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,
                       c.c_float, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int,
                       c.c_int64, c.c_int, c.c_void_p, c.c_int]
        lib.oracle_decode.restype = c.c_int
        lib.oracle_decode.argtypes = decode_args
        lib.oracle_decode_partitioned.restype = c.c_int
        lib.oracle_decode_partitioned.argtypes = decode_args + [c.c_int]
        lib.oracle_copy_blocks.restype = c.c_int
        lib.oracle_copy_blocks.argtypes = [
            c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_int64,
            c.c_int, c.c_int, c.c_int, c.c_int64, c.c_int64, c.c_int]
        lib.oracle_reshape_and_cache_e4m3.restype = c.c_int
        lib.oracle_reshape_and_cache_e4m3.argtypes = [
            c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_int64,
            c.c_int, c.c_int, c.c_int, c.c_int64, c.c_int]
        lib.oracle_decode_e4m3.restype = c.c_int
        lib.oracle_decode_e4m3.argtypes = [
            c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,
            c.c_float, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int64, c.c_int, c.c_void_p,
            c.c_int, c.c_int]
        for name in ("oracle_e4m3_k_index", "oracle_e4m3_v_index"):
            getattr(lib, name).restype = c.c_int64
            getattr(lib, name).argtypes = [c.c_int64, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int]
        lib.oracle_e4m3_value.restype = c.c_double
        lib.oracle_e4m3_value.argtypes = [c.c_int]
        lib.oracle_e4m3_encode.restype = c.c_int
        lib.oracle_e4m3_encode.argtypes = [c.c_float]
        lib.oracle_prefill.restype = c.c_int
        lib.oracle_prefill.argtypes = [c.c_void_p] * 7 + [c.c_float, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int,
                                                          c.c_int, c.c_int64, c.c_int]
        lib.oracle_pool_index.restype = c.c_int64
        lib.oracle_pool_index.argtypes = [c.c_int64, c.c_int, c.c_int, c.c_int, c.c_int,
                                          c.c_int, c.c_int, c.c_int]
        self.lib = lib

    @staticmethod
    def _check(rc: int):
        if rc != 0:
            raise OracleError(f"oracle returned {rc}: {ERRORS.get(rc, 'unknown')}")

    def reshape_and_cache(self, key, value, k_cache, v_cache, slot_mapping, block_size):
        """In-place write of key/value [T, Hkv, D] into the CPU pools."""
        for t in (key, value, k_cache, v_cache):
            assert t.device.type == "cpu" and t.is_contiguous()
        slots = slot_mapping.to(torch.int64).contiguous()
        T, Hkv, D = key.shape
        num_blocks = k_cache.shape[0]
        self._check(self.lib.oracle_reshape_and_cache(
            key.data_ptr(), value.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
            slots.data_ptr(), T, Hkv, D, block_size, num_blocks, DTYPE_CODE[key.dtype]))

    def decode(self, q, k_cache, v_cache, block_tables, context_lens, scale, block_size,
               num_kv_heads, seqs=None, partition_size=None) -> np.ndarray:
        """fp64 attention output [len(seqs) or S, Hq, D] as a numpy array."""
        for t in (q, k_cache, v_cache):
            assert t.device.type == "cpu" and t.is_contiguous()
        bt = block_tables.to(torch.int32).contiguous()
        cl = context_lens.to(torch.int32).contiguous()
        S, Hq, D = q.shape
        n = S if seqs is None else len(seqs)
        out = np.zeros((n, Hq, D), dtype=np.float64)
        sel = None if seqs is None else np.ascontiguousarray(np.asarray(seqs, dtype=np.int32))
        args = [out.ctypes.data, q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                bt.data_ptr(), cl.data_ptr(), float(scale), block_size, S, Hq, num_kv_heads, D,
                bt.shape[1], k_cache.shape[0], DTYPE_CODE[q.dtype],
                None if sel is None else sel.ctypes.data, n]
        if partition_size is None:
            self._check(self.lib.oracle_decode(*args))
        else:
            self._check(self.lib.oracle_decode_partitioned(*args, int(partition_size)))
        return out

    def copy_blocks(self, dst_k, dst_v, src_k, src_v, block_mapping, block_size):
        """In place: copy whole blocks (src, dst) = block_mapping[i] ([n, 2]
        int64) from the source pools to the destination pools (CPU tensors,
        pool layout; the same tensors on both sides for a copy-on-write)."""
        for t in (dst_k, dst_v, src_k, src_v):
            assert t.device.type == "cpu" and t.is_contiguous()
        m = block_mapping.to(torch.int64).contiguous()
        Hkv = src_k.shape[1]
        D = src_k.shape[2] * src_k.shape[4]
        self._check(self.lib.oracle_copy_blocks(
            dst_k.data_ptr(), dst_v.data_ptr(), src_k.data_ptr(), src_v.data_ptr(), m.data_ptr(),
            m.shape[0], Hkv, D, block_size, src_k.shape[0], dst_k.shape[0], DTYPE_CODE[src_k.dtype]))

    # ---- 8-bit (e4m3) pools: uint8 tensors of B*D bytes per (block, head) tile — K [N, Hkv, D // 16, B, 16],
    #      V [N, Hkv, D, B] (byte orders in pa_oracle.cpp); fp32 scales [Hkv]

    def reshape_and_cache_e4m3(self, key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale, block_size):
        """In-place quantising write of key/value [T, Hkv, D] into e4m3 pools."""
        for t in (key, value, k_cache, v_cache, k_scale, v_scale):
            assert t.device.type == "cpu" and t.is_contiguous()
        assert k_cache.dtype == torch.uint8 and k_scale.dtype == torch.float32
        slots = slot_mapping.to(torch.int64).contiguous()
        T, Hkv, D = key.shape
        self._check(self.lib.oracle_reshape_and_cache_e4m3(
            key.data_ptr(), value.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), slots.data_ptr(),
            k_scale.data_ptr(), v_scale.data_ptr(), T, Hkv, D, block_size, k_cache.shape[0],
            DTYPE_CODE[key.dtype]))

    def decode_e4m3(self, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale, block_size,
                    num_kv_heads, seqs=None, partition_size=None) -> np.ndarray:
        """fp64 attention output over e4m3 pools [len(seqs) or S, Hq, D]."""
        for t in (q, k_cache, v_cache, k_scale, v_scale):
            assert t.device.type == "cpu" and t.is_contiguous()
        bt = block_tables.to(torch.int32).contiguous()
        cl = context_lens.to(torch.int32).contiguous()
        S, Hq, D = q.shape
        n = S if seqs is None else len(seqs)
        out = np.zeros((n, Hq, D), dtype=np.float64)
        sel = None if seqs is None else np.ascontiguousarray(np.asarray(seqs, dtype=np.int32))
        self._check(self.lib.oracle_decode_e4m3(
            out.ctypes.data, q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), k_scale.data_ptr(),
            v_scale.data_ptr(), bt.data_ptr(), cl.data_ptr(), float(scale), block_size, S, Hq, num_kv_heads, D,
            bt.shape[1], k_cache.shape[0], DTYPE_CODE[q.dtype], None if sel is None else sel.ctypes.data, n,
            int(partition_size or 0)))
        return out

    def e4m3_k_index(self, block, head, token, dim, num_kv_heads, block_size, head_dim) -> int:
        return int(self.lib.oracle_e4m3_k_index(block, head, token, dim, num_kv_heads, block_size, head_dim))

    def e4m3_v_index(self, block, head, token, dim, num_kv_heads, block_size, head_dim) -> int:
        return int(self.lib.oracle_e4m3_v_index(block, head, token, dim, num_kv_heads, block_size, head_dim))

    def e4m3_value(self, bits: int) -> float:
        return float(self.lib.oracle_e4m3_value(int(bits)))

    def e4m3_encode(self, v: float) -> int:
        return int(self.lib.oracle_e4m3_encode(float(v)))

    def prefill(self, q, k_cache, v_cache, block_tables, context_lens, query_start, scale, block_size,
                num_kv_heads) -> np.ndarray:
        """fp64 chunked-prefill output [T, Hq, D]: query rows query_start[s] ..
        query_start[s+1]-1 are the newest tokens of sequence s, causal."""
        for t in (q, k_cache, v_cache):
            assert t.device.type == "cpu" and t.is_contiguous()
        bt = block_tables.to(torch.int32).contiguous()
        cl = context_lens.to(torch.int32).contiguous()
        qs = query_start.to(torch.int32).contiguous()
        T, Hq, D = q.shape
        out = np.zeros((T, Hq, D), dtype=np.float64)
        self._check(self.lib.oracle_prefill(
            out.ctypes.data, q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), bt.data_ptr(), cl.data_ptr(),
            qs.data_ptr(), float(scale), block_size, cl.numel(), Hq, num_kv_heads, D, bt.shape[1], k_cache.shape[0],
            DTYPE_CODE[q.dtype]))
        return out

    def pool_index(self, block, head, token, dim, num_kv_heads, block_size, head_dim, dtype):
        return int(self.lib.oracle_pool_index(block, head, token, dim, num_kv_heads,
                                              block_size, head_dim, DTYPE_CODE[dtype]))


_default: Oracle | None = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
