"""Seeded synthetic inputs for paged decode — shared by tests, the smoke check
and the benchmark.

This module builds inputs only: context lengths, block tables (a trivial host
block allocator), slot mappings, and N(0,1) values for the query, the KV pools
and the new tokens.  It holds none of the attention arithmetic and no layout
arithmetic: pool values are drawn i.i.d., so where an element sits inside a
(block, head) tile does not matter here.  It imports neither the CUDA binding
nor the oracle.

The workloads follow the pages' descriptions of PagedAttention serving:
fixed-size blocks of 8/16/32 tokens scattered through one preallocated pool
with a per-sequence block table ("vLLM核心架构总览", §4.1; "从源码剖析 vLLM 的显存
管理与连续批处理", §2.1–2.2), a batch of up to 256 sequences with a short-QA /
long-summary length mix (§4.2 of the first page), and a system-prompt prefix
shared by reference count with copy-on-write for a partial block
("vLLM框架解析：PagedAttention技术如何实现LLM推理20倍加速", §2.3).  Head shapes are
those of Llama-3-8B (32 q / 8 kv heads, head_dim 128) and Llama-3-70B (64 q /
8 kv heads).  No dataset or trained weight is involved.

Conventions of the generated batch:
  * pools are shaped [num_blocks, Hkv, D // x, B, x] with x = 16 bytes / element
    size (the library's pool layout; only the shape is used here);
  * block_tables rows list the physical ids of logical blocks 0..ceil(L/B)-1;
    the remaining entries hold -1 (ignored by the kernels);
  * a slot is physical_block * B + offset (the library's slot format); the
    "decode-consistent" slot of sequence s is the position of its newest token,
    context_lens[s] - 1, so a step writes that token and then attends over it.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def vec_elems(dtype: torch.dtype) -> int:
    """Elements per 16-byte vector."""
    return 16 // torch.tensor([], dtype=dtype).element_size()


@dataclass
class Batch:
    name: str
    dtype: torch.dtype
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float
    context_lens: torch.Tensor      # int32 [S]            (CPU)
    block_tables: torch.Tensor      # int32 [S, max_blocks] (CPU)
    q: torch.Tensor                 # [S, Hq, D]
    k_cache: torch.Tensor           # [N, Hkv, D//x, B, x]
    v_cache: torch.Tensor
    new_key: torch.Tensor           # [T, Hkv, D]
    new_value: torch.Tensor
    slot_mapping: torch.Tensor      # int64 [T]             (CPU)
    meta: dict = field(default_factory=dict)

    @property
    def max_blocks_per_seq(self) -> int:
        return self.block_tables.shape[1]

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max().item()) if self.num_seqs else 0

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def elem_bytes(self) -> int:
        return torch.tensor([], dtype=self.dtype).element_size()

    def kv_bytes(self) -> int:
        """Logical K+V bytes one decode pass reads: sum_s L_s * Hkv * D * 2 * e."""
        return int(self.context_lens.to(torch.int64).sum()) * self.num_kv_heads * self.head_dim * 2 * self.elem_bytes

    def unique_kv_bytes(self) -> int:
        """K+V bytes of the distinct token rows read: tokens of a shared prefix
        block are counted once, however many sequences reference it."""
        return int(self.meta.get("unique_kv_bytes", self.kv_bytes()))

    def algorithmic_bytes(self, unique: bool = False) -> int:
        """K/V + Q + out + the block-table entries read + context_lens."""
        S, Hq, D, e, B = self.num_seqs, self.num_q_heads, self.head_dim, self.elem_bytes, self.block_size
        used_tables = int(((self.context_lens.to(torch.int64) + B - 1) // B).sum()) * 4
        kv = self.unique_kv_bytes() if unique else self.kv_bytes()
        return kv + 2 * S * Hq * D * e + used_tables + S * 4

    def to(self, device) -> "Batch":
        moved = {k: (v.to(device) if isinstance(v, torch.Tensor) and k in
                     ("q", "k_cache", "v_cache", "new_key", "new_value") else v)
                 for k, v in self.__dict__.items()}
        return Batch(**moved)


@dataclass
class Fp8Pools:
    """8-bit KV pools for a batch's block tables: uint8 codes
    [N, Hkv, D // 16, B, 16] and fp32 scales [Hkv] for K and for V."""
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    k_scale: torch.Tensor
    v_scale: torch.Tensor

    def kv_bytes(self, batch: "Batch") -> int:
        return int(batch.context_lens.to(torch.int64).sum()) * batch.num_kv_heads * batch.head_dim * 2

    def algorithmic_bytes(self, batch: "Batch") -> int:
        """K/V codes + the kv heads' scales + Q + out + block-table entries + context_lens."""
        S, Hq, D, e, B = batch.num_seqs, batch.num_q_heads, batch.head_dim, batch.elem_bytes, batch.block_size
        used_tables = int(((batch.context_lens.to(torch.int64) + B - 1) // B).sum()) * 4
        return self.kv_bytes(batch) + 2 * batch.num_kv_heads * 4 + 2 * S * Hq * D * e + used_tables + S * 4


def random_fp8_pools(batch: "Batch", seed=0, device=None) -> Fp8Pools:
    """Uniformly random code bytes (the two NaN patterns 0x7f / 0xff replaced
    by zero) for every block of the pool, and seeded scales in [0.005, 0.05]
    per kv head.  Stands in for a pool written by the quantising write, for
    decode measurements and sampled parity."""
    device = torch.device(device or batch.q.device)
    g = torch.Generator(device=device).manual_seed(seed)   # drawn where the pool lives
    shape = (batch.num_blocks, batch.num_kv_heads, batch.head_dim // 16, batch.block_size, 16)
    pools = []
    for _ in range(2):
        codes = torch.randint(0, 256, shape, generator=g, dtype=torch.uint8, device=device)
        codes[(codes & 0x7f) == 0x7f] = 0
        pools.append(codes)
    scales = [torch.empty(batch.num_kv_heads, device=device).uniform_(0.005, 0.05, generator=g) for _ in range(2)]
    return Fp8Pools(pools[0], pools[1], scales[0], scales[1])


def chunked_prefill(seed=0, device="cpu", dtype=torch.bfloat16, num_seqs=8, num_q_heads=32, num_kv_heads=8,
                    head_dim=128, block_size=16, context_range=(1024, 4096), chunk_range=(256, 1024),
                    num_blocks=None) -> Batch:
    """Chunked prefill: every sequence's K/V (context uniform on
    `context_range`) is already in the pool with shuffled block ids, and its
    newest Q tokens (uniform on `chunk_range`, at most the context) are the
    query chunk.  q is [sum Q, Hq, D]; meta["query_start"] is the int32
    [S + 1] prefix sum of the chunk lengths."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(context_range[0], context_range[1], size=num_seqs, endpoint=True)
    chunks = np.minimum(rng.integers(chunk_range[0], chunk_range[1], size=num_seqs, endpoint=True), lens)
    need = int(sum((int(L) + block_size - 1) // block_size for L in lens))
    N = num_blocks or need + 16
    ids = rng.permutation(N)[:need].astype(np.int32)
    tables, _ = _tables_from_lens(lens, block_size, ids)
    slots = _decode_slots(tables, lens, block_size)
    b = make_batch(f"chunked_prefill_{str(dtype).split('.')[-1]}", dtype=dtype, lens=lens, num_q_heads=num_q_heads,
                   num_kv_heads=num_kv_heads, head_dim=head_dim, block_size=block_size, num_blocks=N, tables=tables,
                   slots=slots, seed=seed, device=device)
    T = int(chunks.sum())
    b.q = _normal((T, num_q_heads, head_dim), dtype, device, seed + 7)
    qs = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    b.meta = dict(b.meta, query_start=torch.from_numpy(qs))
    return b


# --------------------------------------------------------------------------
# value generation

def _normal(shape, dtype, device, seed) -> torch.Tensor:
    """i.i.d. N(0,1) drawn in fp32 by torch's seeded generator on `device`,
    then rounded to `dtype` (round to nearest even)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    chunk = 1 << 27  # bound the fp32 staging buffer to 512 MiB
    for start in range(0, flat.numel(), chunk):
        stop = min(flat.numel(), start + chunk)
        flat[start:stop] = torch.randn(stop - start, generator=gen, device=device,
                                       dtype=torch.float32).to(dtype)
    return out


def pool_shape(num_blocks, num_kv_heads, head_dim, block_size, dtype):
    x = vec_elems(dtype)
    return (num_blocks, num_kv_heads, head_dim // x, block_size, x)


def _tables_from_lens(lens, block_size, ids):
    """Assign physical ids (in the given order) to each sequence's logical
    blocks; unused entries are -1."""
    nblk = [(int(L) + block_size - 1) // block_size for L in lens]
    max_blocks = max(1, max(nblk) if nblk else 1)
    tables = np.full((len(lens), max_blocks), -1, dtype=np.int32)
    cursor = 0
    for s, n in enumerate(nblk):
        tables[s, :n] = ids[cursor:cursor + n]
        cursor += n
    return tables, cursor


def _decode_slots(tables, lens, block_size):
    """Slot of each sequence's newest token (position L-1); -1 if L == 0."""
    slots = np.full(len(lens), -1, dtype=np.int64)
    for s, L in enumerate(lens):
        if L > 0:
            pos = int(L) - 1
            slots[s] = int(tables[s, pos // block_size]) * block_size + pos % block_size
    return slots


def make_batch(name, *, dtype, lens, num_q_heads, num_kv_heads, head_dim, block_size,
               num_blocks, tables, slots, seed, device="cpu", scale=None, meta=None) -> Batch:
    lens = np.asarray(lens, dtype=np.int32)
    S, Hkv, D = len(lens), num_kv_heads, head_dim
    shape = pool_shape(num_blocks, Hkv, D, block_size, dtype)
    q = _normal((S, num_q_heads, D), dtype, device, seed * 1000 + 1)
    k_cache = _normal(shape, dtype, device, seed * 1000 + 2)
    v_cache = _normal(shape, dtype, device, seed * 1000 + 3)
    T = len(slots)
    new_key = _normal((T, Hkv, D), dtype, device, seed * 1000 + 4)
    new_value = _normal((T, Hkv, D), dtype, device, seed * 1000 + 5)
    return Batch(name=name, dtype=dtype, num_seqs=S, num_q_heads=num_q_heads,
                 num_kv_heads=Hkv, head_dim=D, block_size=block_size, num_blocks=num_blocks,
                 scale=scale if scale is not None else 1.0 / math.sqrt(D),
                 context_lens=torch.from_numpy(lens.copy()),
                 block_tables=torch.from_numpy(np.ascontiguousarray(tables)),
                 q=q, k_cache=k_cache, v_cache=v_cache, new_key=new_key, new_value=new_value,
                 slot_mapping=torch.from_numpy(np.asarray(slots, dtype=np.int64)),
                 meta=dict(meta or {}))


# --------------------------------------------------------------------------
# the five workloads

def tiny_mha_f32(seed=0, device="cpu") -> Batch:
    """Tiny MHA, fp32: 4 seqs, 4 q = 4 kv heads, D 64, B 16, lens {1,17,33,100},
    64-block pool, block tables drawn from one random permutation (no reuse);
    one new token per sequence written at its newest position."""
    rng = np.random.default_rng(seed)
    lens = [1, 17, 33, 100]
    B, N = 16, 64
    ids = rng.permutation(N).astype(np.int32)
    tables, _ = _tables_from_lens(lens, B, ids)
    slots = _decode_slots(tables, lens, B)
    return make_batch("tiny_mha_f32", dtype=torch.float32, lens=lens, num_q_heads=4,
                      num_kv_heads=4, head_dim=64, block_size=B, num_blocks=N, tables=tables,
                      slots=slots, seed=seed, device=device, scale=1.0 / 8.0)


def llama3_8b_decode(seed=0, device="cpu", num_seqs=64, num_blocks=16384, block_size=16) -> Batch:
    """Llama-3-8B-shaped single-layer decode, bf16: 64 seqs, 32 q / 8 kv heads,
    D 128, B 16, context lens uniform on [128, 2048], a 16384-block pool whose
    used ids are a shuffled random subset."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(128, 2048, size=num_seqs, endpoint=True)
    need = int(sum((int(L) + block_size - 1) // block_size for L in lens))
    ids = rng.choice(num_blocks, size=need, replace=False).astype(np.int32)
    tables, _ = _tables_from_lens(lens, block_size, ids)
    slots = _decode_slots(tables, lens, block_size)
    return make_batch("llama3_8b_decode_bf16", dtype=torch.bfloat16, lens=lens, num_q_heads=32,
                      num_kv_heads=8, head_dim=128, block_size=block_size, num_blocks=num_blocks,
                      tables=tables, slots=slots, seed=seed, device=device)


def continuous_batching_mix(seed=0, device="cpu", block_size=16, num_seqs=256,
                            short_frac=0.8, utilisation=0.9) -> Batch:
    """Continuous-batching mix, bf16, Llama-3-8B heads: 256 seqs, 80% short
    (context uniform on [16, 64]) and 20% long (uniform on [600, 1000]) in
    shuffled order; the pool is sized so the used blocks fill 90% of it; ids
    shuffled."""
    rng = np.random.default_rng(seed)
    n_short = int(round(short_frac * num_seqs))
    lens = np.concatenate([rng.integers(16, 64, size=n_short, endpoint=True),
                           rng.integers(600, 1000, size=num_seqs - n_short, endpoint=True)])
    lens = lens[rng.permutation(num_seqs)]
    need = int(sum((int(L) + block_size - 1) // block_size for L in lens))
    N = int(math.ceil(need / utilisation))
    ids = rng.permutation(N)[:need].astype(np.int32)
    tables, _ = _tables_from_lens(lens, block_size, ids)
    slots = _decode_slots(tables, lens, block_size)
    return make_batch(f"continuous_batching_mix_bf16_B{block_size}", dtype=torch.bfloat16,
                      lens=lens, num_q_heads=32, num_kv_heads=8, head_dim=128,
                      block_size=block_size, num_blocks=N, tables=tables, slots=slots, seed=seed,
                      device=device, meta={"n_short": n_short})


def prefix_sharing(seed=0, device="cpu", prefix_len=1024, num_seqs=128, block_size=16,
                   materialize_shared=False, suffix_range=(16, 512), dtype=torch.float16, num_q_heads=32,
                   num_kv_heads=8, head_dim=128, suffix_lens=None) -> Batch:
    """Prefix sharing, fp16: 128 seqs, 32 q / 8 kv heads, D 128, B 16.  Every
    sequence references the same physical blocks for the full blocks of a
    shared `prefix_len`-token prefix (ref count = num_seqs), then a private
    suffix of uniform[16, 512] tokens.  When the prefix ends inside a block,
    that block is copy-on-write: each sequence gets its own copy of it (whole
    tile copied) and its suffix continues there.

    materialize_shared=True gives the "copied" twin: every shared block is
    duplicated per sequence instead of referenced, with identical contents, so
    the logical K/V of every sequence are unchanged.  Test cases may change the
    element type, the heads and head dim, and give the suffix lengths
    (`suffix_lens`, one per sequence, 0 allowed) instead of drawing them."""
    rng = np.random.default_rng(seed)
    B = block_size
    if suffix_lens is None:
        suffix = rng.integers(suffix_range[0], suffix_range[1], size=num_seqs, endpoint=True)
    else:
        suffix = np.asarray(suffix_lens, dtype=np.int64)
        assert suffix.shape == (num_seqs,) and (suffix >= 0).all()
    lens = prefix_len + suffix
    n_full = prefix_len // B
    partial = prefix_len % B != 0
    nblk = [(int(L) + B - 1) // B for L in lens]
    private_per_seq = [n - n_full for n in nblk]            # includes the CoW block
    n_shared_unique = n_full + (1 if partial else 0)         # +1: the original partial block
    need = n_shared_unique + sum(private_per_seq)
    if materialize_shared:
        need += n_full * num_seqs
    N = need + 8
    ids = rng.permutation(N).astype(np.int32)
    cursor = 0
    shared = ids[cursor:cursor + n_full]; cursor += n_full
    original_partial = None
    if partial:
        original_partial = int(ids[cursor]); cursor += 1
    tables = np.full((num_seqs, max(nblk)), -1, dtype=np.int32)
    copies = []  # (dst_block, src_block) whole-tile copies
    for s in range(num_seqs):
        if materialize_shared:
            own = ids[cursor:cursor + n_full]; cursor += n_full
            tables[s, :n_full] = own
            copies += [(int(d), int(src)) for d, src in zip(own, shared)]
        else:
            tables[s, :n_full] = shared
        n_priv = private_per_seq[s]
        priv = ids[cursor:cursor + n_priv]; cursor += n_priv
        tables[s, n_full:n_full + n_priv] = priv
        if partial:
            copies.append((int(priv[0]), original_partial))  # copy-on-write of the partial block
    slots = _decode_slots(tables, lens, B)
    tag = {torch.float16: "f16", torch.bfloat16: "bf16", torch.float32: "f32"}[dtype]
    batch = make_batch(f"prefix_sharing_{tag}_p{prefix_len}", dtype=dtype, lens=lens,
                       num_q_heads=num_q_heads, num_kv_heads=num_kv_heads, head_dim=head_dim, block_size=B,
                       num_blocks=N, tables=tables, slots=slots, seed=seed, device=device)
    if copies:
        dst = torch.tensor([d for d, _ in copies], device=batch.k_cache.device)
        src = torch.tensor([s for _, s in copies], device=batch.k_cache.device)
        batch.k_cache[dst] = batch.k_cache[src]
        batch.v_cache[dst] = batch.v_cache[src]
    per_token = batch.num_kv_heads * batch.head_dim * 2 * batch.elem_bytes  # K+V bytes of a token
    shared_tokens = 0 if materialize_shared else n_full * B * (num_seqs - 1)
    batch.meta.update({"prefix_len": prefix_len, "shared_blocks": n_full,
                       "ref_count": 1 if materialize_shared else num_seqs,
                       "unique_kv_bytes": batch.kv_bytes() - shared_tokens * per_token})
    return batch


def llama3_70b_long(seed=0, device="cpu", num_seqs=32, len_range=(4096, 32768), block_size=16,
                    decode_consistent_slots=False, free_frac=0.10) -> Batch:
    """Llama-3-70B-shaped long-context decode, bf16: 32 seqs, 64 q / 8 kv heads
    (GQA 8), D 128, B 16, context uniform on [4096, 32768]; the pool holds the
    used blocks plus 10% free blocks, ids shuffled.  The 32 new tokens go to
    distinct random slots of the free blocks (or, decode-consistent, to each
    sequence's newest position)."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(len_range[0], len_range[1], size=num_seqs, endpoint=True)
    need = int(sum((int(L) + block_size - 1) // block_size for L in lens))
    n_free = max(2, int(math.ceil(free_frac * need)))
    N = need + n_free
    ids = rng.permutation(N).astype(np.int32)
    tables, used = _tables_from_lens(lens, block_size, ids)
    if decode_consistent_slots:
        slots = _decode_slots(tables, lens, block_size)
    else:
        free = ids[used:]
        picks = rng.choice(len(free) * block_size, size=num_seqs, replace=False)
        slots = np.array([int(free[p // block_size]) * block_size + int(p % block_size)
                          for p in picks], dtype=np.int64)
    return make_batch("llama3_70b_long_bf16", dtype=torch.bfloat16, lens=lens, num_q_heads=64,
                      num_kv_heads=8, head_dim=128, block_size=block_size, num_blocks=N,
                      tables=tables, slots=slots, seed=seed, device=device)


def random_small(seed=0, device="cpu", dtype=torch.bfloat16, lens=(5, 40, 1, 16), num_q_heads=8,
                 num_kv_heads=2, head_dim=128, block_size=16, extra_blocks=7, new_tokens=None) -> Batch:
    """A small random case for tests: shuffled ids with spare blocks; the new
    tokens go to the sequences' newest positions unless `new_tokens` asks for
    that many random slots of spare blocks (some marked -1 as padding)."""
    rng = np.random.default_rng(seed)
    need = int(sum((int(L) + block_size - 1) // block_size for L in lens))
    N = need + extra_blocks
    ids = rng.permutation(N).astype(np.int32)
    tables, used = _tables_from_lens(list(lens), block_size, ids)
    if new_tokens is None:
        slots = _decode_slots(tables, lens, block_size)
    else:
        free = ids[used:]
        picks = rng.choice(len(free) * block_size, size=new_tokens, replace=False)
        slots = np.array([int(free[p // block_size]) * block_size + int(p % block_size)
                          for p in picks], dtype=np.int64)
        slots[rng.random(new_tokens) < 0.25] = -1
    return make_batch(f"random_small_seed{seed}", dtype=dtype, lens=list(lens),
                      num_q_heads=num_q_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
                      block_size=block_size, num_blocks=N, tables=tables, slots=slots, seed=seed,
                      device=device)


CONFIGS = {
    "tiny_mha_f32": tiny_mha_f32,
    "llama3_8b_decode": llama3_8b_decode,
    "continuous_batching_mix": continuous_batching_mix,
    "prefix_sharing": prefix_sharing,
    "llama3_70b_long": llama3_70b_long,
}
