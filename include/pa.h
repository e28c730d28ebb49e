/*
 * pa.h — C ABI of the B200 paged KV-cache attention library (libpa.so).
 *
 * What the library computes (page titles and sections):
 *   [P1] "vLLM核心架构总览：PagedAttention、Continuous Batching、分布式推理等核心组件",
 *        §4.1 PagedAttention — the KV cache of every sequence lives in fixed-size
 *        physical blocks of one pool; logically contiguous KV is physically
 *        scattered; a block table maps logical to physical blocks; prefix blocks
 *        can be shared between sequences.
 *   [P3] "从源码剖析 vLLM 的显存管理与连续批处理",
 *        §2.1 BlockTable.append_token — a token's KV is written at the physical
 *             block address plus its offset in the block;
 *        §2.2 one pool, preallocated once and carved into equal blocks;
 *        §2.3 attention takes block tables instead of a (batch, seq, dim) tensor
 *             and gathers K/V through them.
 *   [P4] "vLLM框架解析：PagedAttention技术如何实现LLM推理20倍加速",
 *        §2.3 blocks shared by reference count; copy-on-write for isolation.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Ownership.  Every pointer argument is device memory owned by the caller (for
 *   example allocated by PyTorch).  The library allocates and frees nothing and
 *   keeps no state except one device-side error word per GPU (see
 *   pa_get_device_error).  All calls are asynchronous on `stream` (a
 *   cudaStream_t passed as void*; NULL = the legacy default stream) and return
 *   once the work is enqueued.  Every kernel is launched as a programmatic
 *   dependent launch: its thread blocks may take their places on the SMs
 *   while the work ahead of it on the stream still runs, but each first waits
 *   for that work to complete, so the stream's order and memory visibility
 *   are those of ordinary launches.
 * Alignment.  q, out, key, value, both pools and the workspace must be
 *   16-byte aligned; slot_mapping 8-byte, block_tables and context_lens
 *   4-byte aligned.
 * Element types.  q, out, key, value and both pools share one pa_dtype.
 * Pool layout.  k_cache and v_cache are each an array
 *       [num_blocks][num_kv_heads][head_dim / X][block_size][X],  X = 16 / sizeof(elem)
 *   (X = 8 for fp16/bf16, 4 for fp32): the tile of one (block, kv head) is
 *   contiguous (block_size * head_dim elements) and split along head_dim into
 *   16-byte vectors, vector index outer, token inner.
 * Slots.  slot = physical_block * block_size + offset_in_block; slot < 0 marks
 *   a padding token that is skipped.
 * Block tables.  block_tables is int32 [num_seqs][max_blocks_per_seq]; entry
 *   [s][j] is the physical block holding logical tokens [j*B, (j+1)*B) of
 *   sequence s.  Entries at j >= ceil(context_lens[s] / B) are ignored (a
 *   kernel may load them early and discard them, so the whole
 *   [num_seqs][max_blocks_per_seq] array must be readable device memory).
 *   Several rows may name the same physical block (shared prefix).
 * Context lengths.  context_lens[s] (int32) counts every token of sequence s,
 *   including the one just written by pa_reshape_and_cache; 0 gives an
 *   all-zero output row.
 * GQA.  num_q_heads is a multiple of num_kv_heads; query head h reads kv head
 *   h / (num_q_heads / num_kv_heads).
 * Supported shapes.  head_dim in {64, 128}; block_size in {8, 16, 32};
 *   num_q_heads / num_kv_heads in {1, 2, 4, 8}.
 * Arithmetic.  Scores, softmax and the weighted sum accumulate in fp32 (online
 *   softmax); the output is rounded once (round to nearest even) to the dtype.
 * Errors.  Host-side checks (null pointers, unsupported shapes, misalignment,
 *   a workspace too small) return a non-zero pa_status before anything is
 *   launched.  A launch failure returns PA_ERR_CUDA.  Device data that
 *   violates the conventions (a block id outside [0, num_blocks), a slot past
 *   the pool, a context length above min(max_context_len,
 *   max_blocks_per_seq * block_size)) is never dereferenced: the kernel skips
 *   the offending access and sets a bit in the device error word, readable with
 *   pa_get_device_error.  The library never traps and never waits without a
 *   bound.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer */
    PA_ERR_UNSUPPORTED = 2,   /* head_dim / block_size / group / dtype not supported */
    PA_ERR_WORKSPACE = 3,     /* split-K workspace missing or too small */
    PA_ERR_CUDA = 4           /* a CUDA runtime call or launch failed */
} pa_status;

typedef enum { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2 } pa_dtype;

/* Bits of the device error word. */
#define PA_DEVERR_BLOCK_ID     1  /* a block-table entry outside [0, num_blocks) */
#define PA_DEVERR_CONTEXT_LEN  2  /* a context length < 0 or above the stated maximum */
#define PA_DEVERR_SLOT         4  /* a slot >= num_blocks * block_size */
#define PA_DEVERR_TIMEOUT      8  /* an asynchronous copy did not complete in time; the
                                     outputs of the launches concerned are undefined */
#define PA_DEVERR_SEQ_ORDER   16  /* a seq_order entry outside [0, num_seqs) */
#define PA_DEVERR_NO_FREE_BLOCK 32  /* pa_blocks_append: the free blocks ran out */
#define PA_DEVERR_REF_COUNT   64  /* a reference count would drop below zero, a fork into a
                                     sequence that holds tokens, or a corrupt free ring */
#define PA_DEVERR_SHARED_BLOCK 128 /* pa_decode_append: the newest token's block is held by
                                      more than one sequence; its write was skipped */
#define PA_DEVERR_PREFIX      256 /* pa_decode_shared_prefix: a row's first prefix_blocks
                                      entries differ from row 0's */

/*
 * seq_order (pa_decode, pa_decode_append, pa_decode_splitk) — NULL, or an
 * int32 [num_seqs] device array holding a permutation of 0..num_seqs-1,
 * 4-byte aligned.  The pages fix no processing order; this is a scheduling
 * hint only.  The GPU starts the thread blocks of sequence seq_order[0]
 * first, then seq_order[1], ...; a host scheduler that knows the context
 * lengths passes them longest first, so long sequences do not start last and
 * hold up the end of the launch.  Without it, a one-pass launch of many small
 * thread blocks (more than four per SM) starts the sequences of at least
 * max_context_len / 4 tokens before the others.  The
 * results are bit-identical for every order.  An entry outside [0, num_seqs) sets PA_DEVERR_SEQ_ORDER and the
 * thread blocks it names do nothing; a repeated entry is the caller's error
 * (the sequences it leaves out are then not computed).
 */

/*
 * pa_reshape_and_cache — write the K/V of new tokens into the pools.
 * [P3] §2.1 (append_token: physical address = block address + offset).
 *
 *   key, value     [num_tokens][num_kv_heads][head_dim], contiguous, read only
 *   k_cache,
 *   v_cache        pools of num_blocks blocks (layout above), written in place
 *   slot_mapping   int64 [num_tokens]; token i goes to block slot/B, offset
 *                  slot%B; slot < 0 skips the token
 *   The copy is bit-exact.  Two tokens naming the same slot is the caller's
 *   error (the result then holds one of them).  num_tokens == 0 is a no-op.
 */
pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                               const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads,
                               int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype,
                               void* stream);

/*
 * pa_decode — one query token per sequence attends over its whole paged
 * context, in one launch (one pass over each sequence's KV).
 * [P3] §2.3 (block tables in, gather by index remapping); [P1] §4.1.
 *
 *   out            [num_seqs][num_q_heads][head_dim], written
 *   q              [num_seqs][num_q_heads][head_dim]
 *   k_cache,
 *   v_cache        pools (layout above), read only
 *   block_tables   int32 [num_seqs][max_blocks_per_seq]
 *   context_lens   int32 [num_seqs]
 *   scale          softmax scale applied to q.k (typically 1/sqrt(head_dim))
 *   max_context_len  an upper bound of context_lens (used for validation)
 *   out[s,h,:] = sum_t softmax_t(scale * q[s,h,:].K[s,t,:]) V[s,t,:].
 *   num_seqs == 0 is a no-op.
 */
pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, const int32_t* context_lens, float scale,
                    int block_size, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                    int max_blocks_per_seq, int max_context_len, int64_t num_blocks, pa_dtype dtype,
                    const int32_t* seq_order, void* stream);

/*
 * pa_decode_append — one decode step in one launch: for every sequence s with
 * context_lens[s] = L > 0, write key[s] / value[s] (the newest token) at
 * logical position L-1, i.e. at block block_tables[s][(L-1)/B], offset
 * (L-1)%B ([P3] §2.1 append_token), then attend over all L tokens ([P3] §2.3).
 * The result, and every pool byte, equal pa_reshape_and_cache with that slot
 * per sequence followed by pa_decode.  The CTA that computes a sequence's last
 * block patches the new row into the block it has staged and into the pool.
 *
 *   key, value     [num_seqs][num_kv_heads][head_dim], one new token per
 *                  sequence, 16-byte aligned
 *   k_cache,
 *   v_cache        written at the new tokens' rows, read everywhere else
 *   The block holding position L-1 must belong to sequence s alone (a block
 *   shared with other sequences is copied before it is written, as
 *   copy-on-write requires, [P4] §2.3; pa_blocks_append does that).
 *   ref_counts     NULL, or int32 [num_blocks] reference counts (those of the
 *                  pa_blocks_* entry points), 4-byte aligned: a sequence whose
 *                  newest block's count is not 1 is not written (its output
 *                  attends over the pool as it is) and PA_DEVERR_SHARED_BLOCK
 *                  is set.  With NULL the rule above is trusted.
 *   Other arguments as in pa_decode.
 */
pa_status pa_decode_append(void* out, const void* q, const void* key, const void* value, void* k_cache,
                           void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
                           float scale, int block_size, int num_seqs, int num_q_heads, int num_kv_heads,
                           int head_dim, int max_blocks_per_seq, int max_context_len, int64_t num_blocks,
                           pa_dtype dtype, const int32_t* ref_counts, const int32_t* seq_order, void* stream);

/*
 * pa_decode_splitk_workspace_size — bytes of workspace pa_decode_splitk needs:
 * per (sequence, query head, partition) an fp32 partial output of head_dim
 * values plus its running max and sum, for ceil(max_context_len /
 * partition_size) partitions.
 */
pa_status pa_decode_splitk_workspace_size(int num_seqs, int num_q_heads, int head_dim,
                                          int max_context_len, int partition_size, size_t* bytes);

/*
 * pa_decode_splitk — the same result as pa_decode, computed for long contexts
 * by token partitions: kernel 1 handles each (sequence, kv head, partition of
 * partition_size tokens) on its own and writes fp32 partials (unnormalised
 * output, max, sum) to `workspace`; the partitions of each (sequence, query
 * head) are then merged with log-sum-exp weights exp(m_p - max_p m_p):
 *   counters == NULL   by kernel 2 (two launches on `stream`);
 *   counters != NULL   inside kernel 1 (one launch): the CTA that records the
 *                      last partition of a (sequence, kv head) merges them,
 *                      and a sequence with one partition is finished directly.
 * No thread waits for another CTA in either form.
 *
 *   partition_size  tokens per partition; a positive multiple of 16 and of
 *                   block_size (512 is the usual choice)
 *   workspace       device scratch of at least
 *                   pa_decode_splitk_workspace_size(...) bytes, 16-byte
 *                   aligned; its contents need no initialisation and are
 *                   clobbered
 *   counters        NULL, or an int32 array of num_counters >= num_seqs *
 *                   num_kv_heads arrival counters (entry s*Hkv + kvh), all
 *                   zero before the first call (allocate it zeroed); every
 *                   completed call leaves the entries it used at zero, so one
 *                   array serves successive calls of any shape (a partition
 *                   whose copies timed out still counts as arrived, so this
 *                   holds after PA_DEVERR_TIMEOUT too).
 *   Other arguments as in pa_decode; here max_context_len also sizes the
 *   partition grid, so every context_lens[s] must be <= max_context_len.
 *   Calls that may run concurrently on the GPU need their own workspace and
 *   counters.
 */
pa_status pa_decode_splitk(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens, float scale,
                           int block_size, int num_seqs, int num_q_heads, int num_kv_heads,
                           int head_dim, int max_blocks_per_seq, int max_context_len,
                           int64_t num_blocks, pa_dtype dtype, int partition_size, void* workspace,
                           size_t workspace_bytes, int32_t* counters, int64_t num_counters,
                           const int32_t* seq_order, void* stream);

/*
 * pa_decode_splitk_static — pa_decode_splitk for callers that cannot
 * allocate device memory when they launch work (for example a plugin of an
 * inference runtime that is handed only its inputs and outputs at enqueue
 * time, or a latency-critical loop where cudaMalloc's implicit device
 * synchronisation would stall other streams).  The pages describe no such
 * entry point; it exists for those callers only.
 *
 * The caller passes inputs and outputs exactly as for pa_decode_splitk, but
 * no workspace: the fp32 partials are kept in one fixed array of
 * PA_SPLITK_STATIC_SCRATCH_BYTES bytes inside the library's device image,
 * which every GPU that loads the library holds until the process exits.  The
 * library allocates nothing.  The merge runs as the second kernel (the form
 * of pa_decode_splitk without counters), so nothing in the array has to start
 * at zero and the contents left by an earlier call are never read (a
 * partition whose copies timed out is written as empty; the outputs of such a
 * call are not the attention result, see PA_DEVERR_TIMEOUT).
 *
 *   Requests whose partials need more than PA_SPLITK_STATIC_SCRATCH_BYTES
 *   (num_seqs * num_q_heads * ceil(max_context_len / partition_size) *
 *   (head_dim + 2) * 4 bytes) are refused with PA_ERR_WORKSPACE before any
 *   device work; use a larger partition_size or pa_decode_splitk.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it for the
 *   life of the process; make that first call before any stream capture.
 *   The cached address belongs to the device's primary context: after
 *   cudaDeviceReset (or anything else that destroys that context) it is no
 *   longer valid and this entry point must not be called again.
 *   Every call on a device shares the one array: calls that may overlap on
 *   the GPU (different streams without ordering between them) race on it and
 *   must not be issued.
 *   Other arguments, results and errors as in pa_decode_splitk with
 *   seq_order NULL.
 */
#define PA_SPLITK_STATIC_SCRATCH_BYTES (16u << 20)

pa_status pa_decode_splitk_static(void* out, const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* block_tables, const int32_t* context_lens, float scale,
                                  int block_size, int num_seqs, int num_q_heads, int num_kv_heads,
                                  int head_dim, int max_blocks_per_seq, int max_context_len,
                                  int64_t num_blocks, pa_dtype dtype, int partition_size, void* stream);

/*
 * 8-bit KV pools ([P4] §7 names FP8 attention as the next optimisation).  The
 * pages fix no format; read as e4m3 codes (1 sign, 4 exponent bits with bias
 * 7, 3 mantissa bits, no infinities, S.1111.111 = NaN, largest finite 448),
 * one fp32 scale per kv head for K and one for V:
 *   code = e4m3(x / scale)   (fp32 IEEE division; round to nearest-even;
 *                             saturate to +-448; finite x)
 *   value(code) = e4m3_value(code) * scale.
 * Pools are byte arrays of B*D-byte (block, head) tiles.  K tile:
 * [D/16][B][16], dim j of a 16-dim vector at byte 4*((j%8)/2) + 2*(j/8) + j%2.
 * V tile, transposed: [D][B], the tokens of each dim row in groups of 16
 * with token u of a group at the same byte order (B = 8: natural order).
 * Block sizes 8, 16 and 32.  k_scale and v_scale are device
 * float arrays [Hkv], 4-byte aligned.  Queries and outputs are fp16 or bf16
 * (PA_ERR_UNSUPPORTED for fp32).  The decode widens each staged tile exactly
 * to fp16 and runs the fp16 tensor-core path, so for bf16 queries the query
 * group is scaled by a power of two into fp16 range first (exact except for
 * elements below 2^-24 of the group's largest).  NaN codes in a pool give an
 * unspecified result.  (The byte orders let one 32-bit shared-memory load
 * hold the four codes of a thread's MMA fragment.)
 */

/* pa_reshape_and_cache_fp8 — pa_reshape_and_cache into 8-bit pools: each
 * element of key/value [T][Hkv][D] (dtype: fp32, fp16 or bf16) is quantised
 * with its kv head's scale.  Bit-exact against the definition above. */
pa_status pa_reshape_and_cache_fp8(const void* key, const void* value, void* k_cache, void* v_cache,
                                   const int64_t* slot_mapping, const float* k_scale, const float* v_scale,
                                   int64_t num_tokens, int num_kv_heads, int head_dim, int block_size,
                                   int64_t num_blocks, pa_dtype dtype, void* stream);

/* pa_decode_fp8 — pa_decode over 8-bit pools; dtype is the query/output type. */
pa_status pa_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                        const float* k_scale, const float* v_scale, const int32_t* block_tables,
                        const int32_t* context_lens, float scale, int block_size, int num_seqs,
                        int num_q_heads, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                        int max_context_len, int64_t num_blocks, pa_dtype dtype,
                        const int32_t* seq_order, void* stream);

/* pa_decode_append_fp8 — pa_decode_append over 8-bit pools: every sequence's
 * newest token (key/value [num_seqs][num_kv_heads][head_dim] in dtype, 16-byte
 * aligned) is quantised like pa_reshape_and_cache_fp8, written at position
 * L-1 and attended to, in one launch; the result and every pool byte equal
 * pa_reshape_and_cache_fp8 followed by pa_decode_fp8.  ref_counts as in
 * pa_decode_append. */
pa_status pa_decode_append_fp8(void* out, const void* q, const void* key, const void* value, void* k_cache,
                               void* v_cache, const float* k_scale, const float* v_scale,
                               const int32_t* block_tables, const int32_t* context_lens, float scale,
                               int block_size, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                               int max_blocks_per_seq, int max_context_len, int64_t num_blocks, pa_dtype dtype,
                               const int32_t* ref_counts, const int32_t* seq_order, void* stream);

/* pa_decode_splitk_fp8 — pa_decode_splitk over 8-bit pools (same workspace
 * size, counters and merge forms). */
pa_status pa_decode_splitk_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const float* k_scale, const float* v_scale, const int32_t* block_tables,
                               const int32_t* context_lens, float scale, int block_size, int num_seqs,
                               int num_q_heads, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                               int max_context_len, int64_t num_blocks, pa_dtype dtype,
                               int partition_size, void* workspace, size_t workspace_bytes,
                               int32_t* counters, int64_t num_counters, const int32_t* seq_order,
                               void* stream);

/*
 * pa_prefill — chunked prefill over the paged pool ([P1] §4.3 chunked
 * prefill; attention as in [P3] §2.3).  Sequence s brings Q_s = query_start
 * [s+1] - query_start[s] query tokens: the newest Q_s of its context_lens[s]
 * = L_s tokens, whose K/V are already in the pool (pa_reshape_and_cache).
 * Query i of sequence s sits at position L_s - Q_s + i and attends causally:
 *   out[query_start[s]+i, h, :] = sum_{t <= L_s-Q_s+i} softmax_t(scale *
 *                                 q.K[s,t]) V[s,t].
 *
 *   out, q         [T][num_q_heads][head_dim], T = query_start[num_seqs],
 *                  fp16 or bf16 (PA_ERR_UNSUPPORTED for fp32), 16-byte aligned
 *   query_start    int32 [num_seqs + 1], query_start[0] = 0, non-decreasing,
 *                  with Q_s <= L_s; 4-byte aligned device memory
 *   max_query_len  an upper bound of every Q_s (sizes the grid)
 *   Other arguments as in pa_decode.  A sequence whose length or chunk is out
 *   of range sets PA_DEVERR_CONTEXT_LEN and its rows are not written; block
 *   ids outside [0, num_blocks) set PA_DEVERR_BLOCK_ID, are never read, and
 *   their keys are left out of the softmax.
 *   Every block size runs on the 5th-generation tensor cores (tcgen05, fp32
 *   accumulation in tensor memory).  With blocks of 16 or 32 tokens the K pool
 *   is read through a tensor map built per call, which needs the CUDA driver
 *   and at most 2^31 - 1 rows of (block, kv head, 8 dims); a pool beyond that
 *   runs warp-level mma.sync (fp32 accumulation).  8-token blocks need no
 *   tensor map.  The result is the same attention either way, within the
 *   16-bit tolerance.
 */
pa_status pa_prefill(void* out, const void* q, const void* k_cache, const void* v_cache,
                     const int32_t* block_tables, const int32_t* context_lens, const int32_t* query_start,
                     float scale, int block_size, int num_seqs, int num_q_heads, int num_kv_heads,
                     int head_dim, int max_blocks_per_seq, int max_context_len, int max_query_len,
                     int64_t num_blocks, pa_dtype dtype, void* stream);

/*
 * pa_decode_shared_prefix_workspace_size — bytes of workspace
 * pa_decode_shared_prefix needs at most: per (sequence, query head, partial)
 * an fp32 partial output of head_dim values plus its running max and sum, for
 * up to ceil(prefix_blocks * block_size / 64) key partitions of the prefix
 * and one partial of the sequence's own blocks.
 */
pa_status pa_decode_shared_prefix_workspace_size(int num_seqs, int num_q_heads, int head_dim, int prefix_blocks,
                                                 int block_size, size_t* bytes);

/*
 * pa_decode_shared_prefix — pa_decode_append (key != NULL) or pa_decode (key
 * == value == NULL) for a batch whose sequences all start with the same
 * prefix_blocks physical blocks: a system prompt shared by every request
 * ([P1] §4.1, the comparison table: prefix sharing; blocks shared by
 * reference count, [P4] §2.3).  The result is the same attention over each
 * sequence's whole context (within the 16-bit tolerance), computed in two
 * launches on `stream` that may run at the same time:
 *   1. the prefix, once per kv head for every sequence's query: query rows of
 *      all sequences against the prefix's K/V tiles on the 5th-generation
 *      tensor cores (the prefill kernel's form with every prefix key visible),
 *      key partitions spread over some of the SMs, unnormalised partials
 *      (output, running max, sum) to `workspace`;
 *   2. each sequence's own blocks [prefix_blocks, ceil(L/B)) as in pa_decode
 *      (with the newest token written first when appending), its partial to
 *      `workspace` too; launched as a programmatic dependent launch, so that
 *      it fills the SMs the first pass leaves free.
 * Each (sequence, kv head) counts its partials' arrivals in `counters`; the
 * CTA that brings the last one, in either launch, merges them with
 * log-sum-exp weights into `out` (no CTA waits for another).  Both launches
 * have ended when the second has.  Each prefix K/V byte is read once per kv
 * head instead of once per sequence.
 *
 *   prefix_blocks  the blocks every row of block_tables shares at positions
 *                  [0, prefix_blocks): row 0's ids are the ones read; a row
 *                  that differs sets PA_DEVERR_PREFIX (its output then
 *                  attends over row 0's prefix).  1 <= prefix_blocks <=
 *                  max_blocks_per_seq and prefix_blocks * block_size <=
 *                  max_context_len.
 *   context_lens   every L must cover the prefix: L >= prefix_blocks *
 *                  block_size, and L > that when appending (the newest token
 *                  goes to a block of the sequence's own); a sequence that
 *                  breaks this sets PA_DEVERR_CONTEXT_LEN and gets a zero
 *                  output row.
 *   key, value     as in pa_decode_append, or both NULL (no append)
 *   workspace      device scratch of at least
 *                  pa_decode_shared_prefix_workspace_size(...) bytes, 16-byte
 *                  aligned, clobbered; PA_ERR_WORKSPACE if too small
 *   counters       int32 arrival counters, num_counters >= num_seqs *
 *                  num_kv_heads, all zero before the first call, and left at
 *                  zero by every call (as pa_decode_splitk's; one array may
 *                  serve both entries on one stream); PA_ERR_WORKSPACE if
 *                  NULL or too short.  A call that returns PA_ERR_CUDA may
 *                  have launched the first pass only: zero the counters again
 *                  before the next call.
 *   ref_counts     as in pa_decode_append
 *   fp16 or bf16 only (PA_ERR_UNSUPPORTED for fp32).  Where the prefix pass
 *   would need a tensor map of the K pool that cannot be built (see
 *   pa_prefill) the call runs pa_decode_append / pa_decode instead, with the
 *   same result.  Other arguments as in pa_decode.
 *   Calls that may run concurrently on the GPU need their own workspace and
 *   counters.
 */
pa_status pa_decode_shared_prefix(void* out, const void* q, const void* key, const void* value, void* k_cache,
                                  void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
                                  float scale, int block_size, int num_seqs, int num_q_heads, int num_kv_heads,
                                  int head_dim, int max_blocks_per_seq, int max_context_len, int64_t num_blocks,
                                  pa_dtype dtype, int prefix_blocks, void* workspace, size_t workspace_bytes,
                                  int32_t* counters, int64_t num_counters, const int32_t* ref_counts,
                                  void* stream);

/*
 * pa_copy_blocks — copy whole physical blocks (every kv head, token and
 * dimension, K pool and V pool) from a source pool pair to a destination pool
 * pair.  The same pools on both sides duplicate a shared block before a
 * sequence writes into it (copy-on-write, [P4] §2.3); a page-locked host pool
 * on one side swaps a preempted sequence's blocks out to host memory or back
 * in ([P1] §4.2 preemption by swapping).
 *
 *   dst_k_cache,
 *   dst_v_cache    destination pools of dst_num_blocks blocks (layout above),
 *                  written at the destination blocks only
 *   src_k_cache,
 *   src_v_cache    source pools of src_num_blocks blocks, read only
 *   block_mapping  int64 [num_pairs][2]: (source block, destination block),
 *                  8-byte aligned; a pair with a negative source block is an
 *                  empty entry and copies nothing (the copy_pairs output of
 *                  pa_blocks_append can be passed as it is)
 *   Every pool and block_mapping is device memory or page-locked host memory
 *   that the device can address (cudaHostAlloc / cudaMallocHost, or
 *   cudaHostRegister'd and mapped); anything else is PA_ERR_INVALID_ARG.  The
 *   copy is bit-exact.  A pair naming a block outside its pool sets
 *   PA_DEVERR_BLOCK_ID and is skipped.  Destinations must be distinct, and no
 *   block may be both a source and a destination in one call (the result is
 *   then undefined).  num_pairs == 0 is a no-op.
 */
pa_status pa_copy_blocks(void* dst_k_cache, void* dst_v_cache, const void* src_k_cache,
                         const void* src_v_cache, const int64_t* block_mapping, int64_t num_pairs,
                         int num_kv_heads, int head_dim, int block_size, int64_t src_num_blocks,
                         int64_t dst_num_blocks, pa_dtype dtype, void* stream);

/*
 * Block management on the device ([P3] §2.1 append_token takes a free block
 * when a sequence's next token starts a new logical block; §2.2 one pool of
 * equal blocks; [P4] §2.2-2.3 reference counts, prefix blocks shared by
 * count, copy-on-write, a block whose count reaches zero returns to the free
 * pool; [P3] §3.2 admission while blocks remain, stopping at the first request
 * that does not fit).
 *
 * State, all caller-owned device memory (num_blocks = N <= 2^31 - 1):
 *   ref_counts  int32 [N]  references to each block from block-table rows
 *                          (0 = free)
 *   free_ids    int32 [N]  the free blocks as a ring: positions head ..
 *                          tail-1 (mod N) hold them, oldest first
 *   free_state  int64 [2]  {head, tail}; both only grow; tail - head blocks
 *                          are free (the host may read it: can_allocate)
 * together with block_tables (int32 [num_seqs][max_blocks_per_seq]) and
 * context_lens (int32 [num_seqs]) as the attention entry points read them.
 * Table entries of unused logical blocks hold -1.  Every operation is one
 * launch on `stream`, its result is deterministic and equals the plain
 * sequential bookkeeping: sequences in index (or list) order, blocks in
 * logical order, the free ring first in first out.  Operations on one state
 * must not overlap on the GPU.  Errors found on the device set PA_DEVERR_*
 * bits and skip the offending sequence or pair; nothing faults.
 */

/* pa_blocks_init — every block free (ring = 0, 1, ..., N-1), counts zero. */
pa_status pa_blocks_init(int32_t* ref_counts, int32_t* free_ids, int64_t* free_state, int64_t num_blocks,
                         void* stream);

/*
 * pa_blocks_append — one step of every sequence: sequence s takes
 * num_new_tokens[s] >= 0 new token positions L .. L+n-1 (L = its length).
 *   * A position that starts a logical block gets a block from the ring;
 *     positions in the sequence's last, partly filled block go there.  If that
 *     block's count is above one it is first replaced by a private copy
 *     (copy-on-write): the k-th writer into such a block in this step, in
 *     sequence order, copies it while k < count - 1; the last holder writes in
 *     place.  The copy block is taken before new blocks.
 *   * Sequences are served in index order while free blocks remain; the
 *     first one whose blocks do not fit, and every later one, are not served
 *     (PA_DEVERR_NO_FREE_BLOCK): no block, no length change, slots -1.
 *   * A row that would exceed max_blocks_per_seq * block_size tokens, or a
 *     negative count, is skipped with PA_DEVERR_CONTEXT_LEN.
 * Outputs:
 *   slot_mapping  int64 [num_slots], the step's token slots packed in sequence
 *                 order (offsets = running sum of num_new_tokens), ready for
 *                 pa_reshape_and_cache; num_slots must be at least that sum,
 *                 otherwise nothing is done and PA_DEVERR_SLOT is set
 *   copy_pairs    int64 [num_seqs][2]: (old block, its copy) for a sequence
 *                 that copied, (-1, -1) otherwise; pass it to pa_copy_blocks
 *                 (same pools on both sides) before the new tokens are written
 *                 (negative entries copy nothing)
 *   block_tables, context_lens, ref_counts, free_state updated in place.
 * Also used as scratch while the launch runs: slot_mapping and copy_pairs.
 * For pa_decode_append (which writes the token at position L-1 itself) call
 * this with one token per running sequence, then pa_copy_blocks, then
 * pa_decode_append on the updated tables and lengths.
 */
pa_status pa_blocks_append(int32_t* block_tables, int32_t* context_lens, const int32_t* num_new_tokens,
                           int32_t* ref_counts, const int32_t* free_ids, int64_t* free_state,
                           int64_t* slot_mapping, int64_t num_slots, int64_t* copy_pairs, int num_seqs,
                           int max_blocks_per_seq, int block_size, int64_t num_blocks, void* stream);

/*
 * pa_blocks_fork — for each (parent, child, length) row of forks (int32
 * [num_forks][3]), in order: the child shares the parent's first `length`
 * tokens: its row takes the parent's first ceil(length / B) block ids, each
 * of whose counts goes up by one, and its length becomes `length` (prefix
 * sharing of a common system prompt, or a parallel sample; [P4] §2.3, §3.1).
 * The child must hold no tokens and differ from the parent
 * (PA_DEVERR_REF_COUNT otherwise) and 0 <= length <= the parent's length
 * (PA_DEVERR_CONTEXT_LEN otherwise); a refused row is skipped.
 */
pa_status pa_blocks_fork(int32_t* block_tables, int32_t* context_lens, int32_t* ref_counts, const int32_t* forks,
                         int num_forks, int num_seqs, int max_blocks_per_seq, int block_size, int64_t num_blocks,
                         void* stream);

/*
 * pa_blocks_release — free whole sequences (int32 seqs [num_release], in
 * order): each block of the sequence, in logical order, loses one reference;
 * a block whose count reaches zero joins the ring's tail then.  The row is
 * set to -1 and the length to 0 (a sequence listed twice is freed once).
 * A count already at zero sets PA_DEVERR_REF_COUNT and is left at zero.
 */
pa_status pa_blocks_release(int32_t* block_tables, int32_t* context_lens, int32_t* ref_counts, int32_t* free_ids,
                            int64_t* free_state, const int32_t* seqs, int num_release, int num_seqs,
                            int max_blocks_per_seq, int block_size, int64_t num_blocks, void* stream);

/*
 * pa_get_device_error — read and clear the device error word of the current
 * GPU.  Synchronises `stream` first, so it reports every launch enqueued on it
 * before the call.  *code receives an OR of PA_DEVERR_* bits (0 = no error).
 */
pa_status pa_get_device_error(void* stream, int32_t* code);

/* pa_status_string — a static, human-readable name of a status. */
const char* pa_status_string(pa_status status);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
