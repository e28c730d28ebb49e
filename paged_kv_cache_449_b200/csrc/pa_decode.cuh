// Paged decode attention kernels for sm_100a.
//
// What is computed ("从源码剖析 vLLM 的显存管理与连续批处理" §2.3; "vLLM核心架构总览"
// §4.1): for every sequence s of a continuous batch and every query head h,
//     out[s,h,:] = sum_t softmax_t(scale * q[s,h,:] . K[s,t,:]) V[s,t,:]
// over the sequence's logically ordered tokens t < context_lens[s], where the
// K/V of logical token t live in physical block block_tables[s][t / B] at
// offset t % B of one preallocated pool.
//
// Design (B200):
//  * One CTA per (sequence, kv head[, token partition]).  All query heads of a
//    GQA group are handled by the same CTA, so every K/V byte is read from HBM
//    once per kv head.
//  * Each warp streams its own blocks (logical blocks warp, warp+NW, ...):
//    lane 0 issues one bulk copy for the block's K tile and one for its V tile
//    (each tile is B*D contiguous elements in the pool) into a per-warp ring of
//    STAGES shared-memory slots; completion is tracked by an mbarrier per
//    slot.  No producer/consumer handshake is needed across warps.
//  * 16-bit path: QK^T and PV run on the tensor cores (mma.sync m16n8k16 /
//    m16n8k8, fp32 accumulate) with the g = Hq/Hkv query heads as the M rows
//    (padded to 16) and tokens as N (QK^T) or K (PV).  The pool layout
//    [D/X][B][X] of a tile makes both ldmatrix (K) and ldmatrix.trans (V) read
//    eight consecutive 16-byte rows: bank-conflict free without a swizzle.
//    Scores are kept in base 2 (scale * log2 e folded in).
//  * fp32 path: the same staging, CUDA-core FMA dot products (lanes over
//    tokens for QK^T, lanes over 16-byte D vectors for PV), natural exp.
//  * Online softmax per warp (running max m, running sum l, rescale by
//    exp(m_old - m_new)), then a merge of the NW warp states through shared
//    memory with weights exp(m_w - max_w m_w).
//  * Split mode: the CTA's result for its partition is written unnormalised
//    (acc, m, l) to the workspace and pa_merge_kernel combines partitions.
#pragma once

#include "pa_e4m3.cuh"
#include "pa_warp.cuh"

namespace pa {

struct DecodeParams {
    void* out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* part_acc;    // split: [S][Hq][P][D] fp32 unnormalised outputs
    float* part_ml;     // split: [S][Hq][P][2] running max (score domain) and sum
    float score_scale;  // multiplier from q.k to the score domain
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int group;
    int max_blocks_per_seq;
    int context_cap;       // min(max_context_len, max_blocks_per_seq * B)
    long long num_blocks;
    int partition_blocks;  // split: blocks per partition
    int num_partitions;    // split: P
    int* counters;         // split, fused merge: [S*Hkv] arrival counters (zero between calls); null = merge kernel
    const void* new_key;   // append: [S][Hkv][D] K/V of each sequence's newest token (position L-1), or null
    const void* new_value;
    const int32_t* seq_order;  // optional [S] permutation: CTA z works on sequence seq_order[z]; null = z
    int class_threshold;       // > 0: grid.z = 2S, CTAs z < S take the sequences of at least this many
                               // tokens, CTAs z >= S (sequence z - S) the shorter ones
    const float* k_scale;      // 8-bit pools: [Hkv] scales of the K and V codes
    const float* v_scale;
    const int32_t* ref_counts;  // append: [num_blocks] reference counts, or null (not checked)
    // shared-prefix form: every sequence's blocks [0, first_block) are the
    // prefix that row 0 of block_tables holds, attended by the prefix pass;
    // this pass attends blocks [first_block, nblk) and writes its partial to
    // slot num_partitions - 1 of part_acc / part_ml (the prefix pass's key
    // partitions fill the slots before it); the last of the num_partitions
    // arrivals on counters[s * Hkv + kvh] merges them
    int first_block;
};

// Append: the newest token of sequence s (logical position L-1) is written
// into the block being computed, both in the staged shared-memory tiles and in
// the pool, before the block is used (the same bytes pa_reshape_and_cache
// would write at that token's slot).  Lane v holds 16-byte vector v of the
// new K and V rows (D * sizeof(T) <= 512 bytes), loaded early by load_row.
template <typename T, int D>
struct NewRow {
    static constexpr int kVecs = D * static_cast<int>(sizeof(T)) / 16;
    static_assert(kVecs <= 32, "one 16-byte vector per lane");
    uint4 k, v;
    __device__ __forceinline__ void load_row(const DecodeParams& p, int s, int kvh, int lane) {
        if (lane < kVecs) {
            const long long row = (static_cast<long long>(s) * p.num_kv_heads + kvh) * kVecs;
            k = reinterpret_cast<const uint4*>(p.new_key)[row + lane];
            v = reinterpret_cast<const uint4*>(p.new_value)[row + lane];
        }
    }
};

template <typename T, int D, int B>
__device__ __forceinline__ void append_newest_token(const DecodeParams& p, const NewRow<T, D>& nr, uint8_t* stage,
                                                    int id, int kvh, int t, int lane) {
    constexpr int kTile = B * D * static_cast<int>(sizeof(T));
    char* kpool = reinterpret_cast<char*>(const_cast<void*>(p.k_cache));
    char* vpool = reinterpret_cast<char*>(const_cast<void*>(p.v_cache));
    const long long tile = (static_cast<long long>(id) * p.num_kv_heads + kvh) * kTile;
    if (lane < NewRow<T, D>::kVecs) {
        const uint4 kv = nr.k, vv = nr.v;
        const int off = (lane * B + t) * 16;
        *reinterpret_cast<uint4*>(stage + off) = kv;
        *reinterpret_cast<uint4*>(stage + kTile + off) = vv;
        *reinterpret_cast<uint4*>(kpool + tile + off) = kv;
        *reinterpret_cast<uint4*>(vpool + tile + off) = vv;
    }
    fence_proxy_async_smem();  // the stage is refilled by bulk copies later
    __syncwarp();
}

// The same for 8-bit pools: lane 4j + w owns dims 16j + 2w, +1, +8, +9 of the
// newest row, i.e. word w of K vector j and four bytes of four V dim rows.
// The codes are computed when the row is loaded (the quantising write's
// arithmetic) and stored into the staged tile and the pool like above.
template <typename T, int D>
struct NewRowE4m3 {
    uint32_t kword = 0, vcodes = 0;  // vcodes: bytes of dims d0, d0+1, d0+8, d0+9
    __device__ __forceinline__ void load_row(const DecodeParams& p, int s, int kvh, int lane) {
        if (lane < D / 4) {
            const int d0 = 16 * (lane >> 2) + 2 * (lane & 3);
            const long long row = (static_cast<long long>(s) * p.num_kv_heads + kvh) * D;
            const T* k = reinterpret_cast<const T*>(p.new_key) + row;
            const T* v = reinterpret_cast<const T*>(p.new_value) + row;
            const float ks = __ldg(p.k_scale + kvh), vs = __ldg(p.v_scale + kvh);
            kword = quantise2(to_float<T>(k[d0]), to_float<T>(k[d0 + 1]), ks) |
                    (quantise2(to_float<T>(k[d0 + 8]), to_float<T>(k[d0 + 9]), ks) << 16);
            vcodes = quantise2(to_float<T>(v[d0]), to_float<T>(v[d0 + 1]), vs) |
                     (quantise2(to_float<T>(v[d0 + 8]), to_float<T>(v[d0 + 9]), vs) << 16);
        }
    }
};

template <typename T, int D, int B>
__device__ __forceinline__ void append_newest_token_e4m3(const DecodeParams& p, const NewRowE4m3<T, D>& nr,
                                                         uint8_t* stage, int id, int kvh, int t, int lane) {
    constexpr int kTile = B * D;
    uint8_t* kpool = reinterpret_cast<uint8_t*>(const_cast<void*>(p.k_cache));
    uint8_t* vpool = reinterpret_cast<uint8_t*>(const_cast<void*>(p.v_cache));
    const long long tile = (static_cast<long long>(id) * p.num_kv_heads + kvh) * kTile;
    if (lane < D / 4) {
        const int j = lane >> 2, w = lane & 3;
        const int d0 = 16 * j + 2 * w;
        const int koff = ((j * B + t) * 4 + w) * 4;
        *reinterpret_cast<uint32_t*>(stage + koff) = nr.kword;
        *reinterpret_cast<uint32_t*>(kpool + tile + koff) = nr.kword;
        const int at = v_row_byte(t, B);
        const int dims[4] = {d0, d0 + 1, d0 + 8, d0 + 9};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint8_t code = static_cast<uint8_t>(nr.vcodes >> (8 * e));
            stage[kTile + dims[e] * B + at] = code;
            vpool[tile + dims[e] * B + at] = code;
        }
    }
    fence_proxy_async_smem();  // the stage is refilled by bulk copies later
    __syncwarp();
}

// Fused split-K merge, run by the CTA that completes the last partition of
// (sequence s, kv head kvh): combines the np partial results of each of the
// group's query heads in partition order with a running maximum (the
// log-sum-exp merge) and writes the output rows.  Threads own 16-byte slices.
template <typename T, int D, bool LOG2, int THREADS>
__device__ __forceinline__ void merge_partitions_cta(const DecodeParams& p, int s, int kvh, int np) {
    const int group = p.group;
    const int slices = group * D / 4;
    for (int v = threadIdx.x; v < slices; v += THREADS) {
        const int r = (4 * v) / D;
        const long long row = static_cast<long long>(s) * p.num_q_heads + kvh * group + r;
        const float* ml = p.part_ml + row * p.num_partitions * 2;
        const float4* acc = reinterpret_cast<const float4*>(p.part_acc + row * p.num_partitions * D) + (v % (D / 4));
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        float M = kNegInf, den = 0.f;
#pragma unroll 4
        for (int q = 0; q < np; ++q) {
            const float m = __ldcg(ml + 2 * q), l = __ldcg(ml + 2 * q + 1);
            const float4 x = __ldcg(acc + static_cast<long long>(q) * (D / 4));
            const float mn = fmaxf(M, m);
            if (mn != kNegInf) {
                const float sa = softmax_exp<LOG2>(M - mn), sb = softmax_exp<LOG2>(m - mn);
                a.x = fmaf(a.x, sa, x.x * sb);
                a.y = fmaf(a.y, sa, x.y * sb);
                a.z = fmaf(a.z, sa, x.z * sb);
                a.w = fmaf(a.w, sa, x.w * sb);
                den = fmaf(den, sa, l * sb);
                M = mn;
            }
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
        T* dst = reinterpret_cast<T*>(p.out) + row * D + 4 * (v % (D / 4));
        dst[0] = from_float<T>(a.x * inv);
        dst[1] = from_float<T>(a.y * inv);
        dst[2] = from_float<T>(a.z * inv);
        dst[3] = from_float<T>(a.w * inv);
    }
}


template <typename T, int D, int B, int NW, int STAGES, bool FP8 = false>
struct DecodeSmem {
    static constexpr int kElem = FP8 ? 1 : sizeof(T);
    static constexpr int kTile = B * D * kElem;                 // one (block, head) tile, bytes
    static constexpr int kRing = NW * STAGES * 2 * kTile;       // K and V slots of all warps
    static constexpr int kMerge = NW * kMaxGroup * (kMergeRow<D> + 2) * 4;  // warp states for the CTA merge
    static constexpr int kArea = kRing > kMerge ? kRing : kMerge;
    static constexpr int kBars = (NW * STAGES * 8 + 15) / 16 * 16;  // keeps what follows 16-byte aligned
    static constexpr int kQ = IsF32<T>::value ? kMaxGroup * D * 4 : 0;
    static constexpr int kTotal = kArea + kBars + kQ;
};

// ----------------------------------------------------------------------------
// The decode kernel (SPLIT = false: one pass per (seq, kv head); true: one
// partition of partition_blocks blocks per CTA, partials to the workspace).

// The shared-prefix form's wide CTAs are held to registers that let five
// share an SM (112 registers, four per SM, otherwise: 38.2 against 39.1 us on
// the prefix-sharing workload).
#ifndef PA_PREFIX_MIN_CTAS
#define PA_PREFIX_MIN_CTAS 5
#endif
template <typename T, int D, int B, int NW, int STAGES, bool SPLIT, bool FP8 = false, bool CLASSES = false,
          bool PREFIX = false>
__global__ void __launch_bounds__(NW * 32, (PREFIX && NW <= 4) ? PA_PREFIX_MIN_CTAS : 1)
    pa_decode_kernel(const __grid_constant__ DecodeParams p) {
    using Smem = DecodeSmem<T, D, B, NW, STAGES, FP8>;
    constexpr bool kF32 = IsF32<T>::value;
    static_assert(!(FP8 && kF32), "8-bit pools take 16-bit queries");
    // 8-bit pools run the fp16 tensor-core path on widened tiles.
    using TM = typename std::conditional<FP8, __half, T>::type;
    constexpr int kTile = Smem::kTile;
    static_assert(STAGES >= 1 && STAGES <= 32, "ring depth");
    static_assert(!(PREFIX && (SPLIT || FP8 || kF32)), "the shared-prefix form is one pass over 16-bit pools");
    static_assert((kTile % 16) == 0, "bulk copies move multiples of 16 bytes");

    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* ring = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Smem::kArea);
    float* qs = reinterpret_cast<float*>(smem + Smem::kArea + Smem::kBars);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int part = blockIdx.x, kvh = blockIdx.y;
    int s = blockIdx.z;
    // (the shared-prefix form overlaps the prefix pass instead: see below)
    if constexpr (!PREFIX) wait_for_prior_work();
    // Shared-prefix form: this grid may start while the prefix pass still runs
    // (the two meet only through the arrival counters).  CTA 0 waits for that
    // pass to complete before it leaves, so that this grid, and the work after
    // it on the stream, end after it.
    auto prefix_pass_done = [&]() {
        if constexpr (PREFIX) {
            if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
        }
    };
    if constexpr (CLASSES) {   // the wide one-pass shape: the grid may run two classes
        if (p.class_threshold > 0 && s >= p.num_seqs) s -= p.num_seqs;
    }
    if (p.seq_order != nullptr) {
        // CTAs start roughly in blockIdx order, so a longest-first order
        // starts the long sequences early and leaves the short ones to fill
        // the SMs at the end of the launch.
        s = __ldg(p.seq_order + blockIdx.z);
        if (static_cast<unsigned>(s) >= static_cast<unsigned>(p.num_seqs)) {
            if (threadIdx.x == 0 && part == 0 && kvh == 0) flag_error(16 /* PA_DEVERR_SEQ_ORDER */);
            return;
        }
    }
    const int group = p.group;

    // The warp's ring barriers are set up before any global load is issued.
    uint64_t* wbar = bars + warp * STAGES;
    uint8_t* wring = ring + warp * STAGES * 2 * kTile;
    if (lane == 0) {
        for (int i = 0; i < STAGES; ++i) mbar_init(&wbar[i], 1);
        fence_barrier_init();
    }
    __syncwarp();

    // Issued before the context length arrives, so the three loads overlap:
    // this warp's first 32 block-table entries (any entry of the row is
    // readable; entries past the context are discarded below) and, for the
    // tensor-core path, the query fragments.
    const int b0_first = SPLIT ? part * p.partition_blocks : (PREFIX ? p.first_block : 0);
    const int32_t* bt = p.block_tables + static_cast<long long>(s) * p.max_blocks_per_seq + b0_first + warp;
    int first_ids = -1;
    if (b0_first + warp + lane * NW < p.max_blocks_per_seq) first_ids = __ldg(bt + lane * NW);
    const T* qrows = reinterpret_cast<const T*>(p.q) +
                     (static_cast<long long>(s) * p.num_q_heads + kvh * group) * D;
    typename WarpState<TM, D, B>::type acc;
    acc.reset();
    float score_scale = p.score_scale, out_scale = 1.f;
    if constexpr (FP8) {
        const int q_shift = load_q_half<T, D>(acc.qa, qrows, group, lane);
        score_scale = ldexpf(p.score_scale * __ldg(p.k_scale + kvh) * kE4m3Unit, -q_shift);
        out_scale = __ldg(p.v_scale + kvh) * kE4m3Unit;
    } else if constexpr (!kF32) {
        acc.load_q(qrows, group, lane);
    }

    int L = p.context_lens[s];
    if (L < 0 || L > p.context_cap) {
        if (threadIdx.x == 0 && part == 0 && kvh == 0) flag_error(2 /* PA_DEVERR_CONTEXT_LEN */);
        L = L < 0 ? 0 : p.context_cap;
    }
    // Two classes (no copy is in flight yet): this half of the grid leaves the
    // sequence to the other half.
    if constexpr (CLASSES) {
        if (p.class_threshold > 0 && (L >= p.class_threshold) != (blockIdx.z < static_cast<unsigned>(p.num_seqs))) {
            prefix_pass_done();
            return;
        }
    }
    const int nblk = (L + B - 1) / B;
    int b0 = 0, b1 = nblk;
    if constexpr (SPLIT) {
        b0 = part * p.partition_blocks;
        if (nblk == 0 && part == 0 && p.counters != nullptr) {
            // Fused merge: no partition runs for an empty context, so its
            // output rows are zeroed here.
            T* out = reinterpret_cast<T*>(p.out) + (static_cast<long long>(s) * p.num_q_heads + kvh * group) * D;
            for (int i = threadIdx.x; i < group * D; i += NW * 32) out[i] = from_float<T>(0.f);
        }
        if (b0 >= nblk) return;  // this partition is past the end of the sequence
        b1 = min(nblk, b0 + p.partition_blocks);
    }
    if constexpr (PREFIX) {
        // the sequence's own part starts after the shared prefix; a context
        // that does not reach past it (or, appending, whose newest token would
        // land in it) is refused: no block is attended, the partial is empty
        // and the merge writes a zero output
        b0 = p.first_block;
        if (shared_prefix_refused(L, b0 * B, p.new_key != nullptr)) {
            if (threadIdx.x == 0 && kvh == 0) flag_error(2 /* PA_DEVERR_CONTEXT_LEN */);
            b1 = b0;
        }
    }
    if constexpr (!SPLIT && !PREFIX) {
        if (nblk == 0) {  // empty context: zero output
            T* out = reinterpret_cast<T*>(p.out) + (static_cast<long long>(s) * p.num_q_heads + kvh * group) * D;
            for (int i = threadIdx.x; i < group * D; i += NW * 32) out[i] = from_float<T>(0.f);
            return;
        }
    }

    if constexpr (kF32) {
        for (int i = threadIdx.x; i < group * D; i += NW * 32) qs[i] = reinterpret_cast<const float*>(qrows)[i];
        __syncthreads();
    }

    // ---- per-warp block stream
    const int nb = b1 - b0;
    const int n_w = nb > warp ? (nb - warp + NW - 1) / NW : 0;
    // Append: the warp that will compute the last block loads the new row now.
    const int last_block = nblk - 1;
    bool owns_last = p.new_key != nullptr && last_block >= b0 && last_block < b1 &&
                     (last_block - b0) % NW == warp;
    NewRow<T, D> new_row;
    NewRowE4m3<T, D> new_row8;
    if constexpr (FP8) {
        if (owns_last) new_row8.load_row(p, s, kvh, lane);
    } else {
        if (owns_last) new_row.load_row(p, s, kvh, lane);
    }

    auto load_ids = [&](int round) -> int {
        const int i = round * 32 + lane;
        int id = -1;
        if (i < n_w) {
            id = round == 0 ? first_ids : __ldg(bt + i * NW);
            if (id < 0 || static_cast<long long>(id) >= p.num_blocks) {
                flag_error(1 /* PA_DEVERR_BLOCK_ID */);
                id = -1;
            }
        }
        return id;
    };
    int win0 = load_ids(0);
    int win1 = n_w > 32 ? load_ids(1) : -1;
    int cur_round = 0;
    auto block_id = [&](int i) -> int {  // warp-uniform i
        const int v0 = __shfl_sync(0xffffffffu, win0, i & 31);
        const int v1 = __shfl_sync(0xffffffffu, win1, i & 31);
        return (i >> 5) == cur_round ? v0 : v1;
    };

    const uint64_t policy = l2_evict_first_policy();
    const char* kpool = reinterpret_cast<const char*>(p.k_cache);
    const char* vpool = reinterpret_cast<const char*>(p.v_cache);
    auto issue = [&](int i) {
        const int id = block_id(i);
#ifdef PA_TEST_HOOKS
        if (g_test_skip_first_copy && i == 0 && warp == 0 && s == 0 && kvh == 0 && part == 0) return;
#endif
        if (lane == 0) {
            const int st = i % STAGES;
            uint8_t* dst = wring + st * 2 * kTile;
            if (id >= 0) {
                const long long off = (static_cast<long long>(id) * p.num_kv_heads + kvh) * kTile;
                mbar_arrive_expect_tx(&wbar[st], 2 * kTile);
                bulk_copy_g2s(dst, kpool + off, kTile, &wbar[st], policy);
                bulk_copy_g2s(dst + kTile, vpool + off, kTile, &wbar[st], policy);
            } else {
                mbar_arrive(&wbar[st]);  // nothing to fetch: complete the phase
            }
        }
    };

    if constexpr (kF32) acc.qs = qs;

    int issued = n_w < STAGES ? n_w : STAGES;
    for (int i = 0; i < issued; ++i) issue(i);
    if (owns_last && p.ref_counts != nullptr) {
        // Copy-on-write guard: the block the newest token goes to must be held
        // by this sequence alone.  Checked while the first copies are in flight.
        const int id = __ldg(p.block_tables + static_cast<long long>(s) * p.max_blocks_per_seq + last_block);
        if (id >= 0 && id < p.num_blocks && __ldg(p.ref_counts + id) != 1) {
            if (lane == 0) flag_error(128 /* PA_DEVERR_SHARED_BLOCK */);
            owns_last = false;  // no write; the pool is attended as it is
        }
    }
    if constexpr (PREFIX) {
        // the prefix pass read row 0's prefix: every row must hold the same ids there
        if (kvh == 0 && s != 0) {
            const int32_t* row = p.block_tables + static_cast<long long>(s) * p.max_blocks_per_seq;
            for (int k = threadIdx.x; k < p.first_block; k += NW * 32)
                if (__ldg(row + k) != __ldg(p.block_tables + k)) flag_error(256 /* PA_DEVERR_PREFIX */);
        }
    }
    bool failed = false;
    int i = 0;
    // Tensor-core path with 16-token blocks and rings of three stages or more:
    // a warp takes two of its blocks per online-softmax step (one row maximum
    // and one rescale per 32 tokens) while a third stage stays in flight; a
    // last odd block goes alone.  (With two stages the pair would leave none
    // in flight: slower.)
#ifndef PA_PAIR_MIN_STAGES
#define PA_PAIR_MIN_STAGES 3
#endif
    constexpr bool kPairs = !kF32 && B == 16 && STAGES >= PA_PAIR_MIN_STAGES;
    for (; i < n_w; ++i) {
        if (i > 0 && (i & 31) == 0) {
            win0 = win1;
            ++cur_round;
            win1 = load_ids(cur_round + 1);
        }
        if constexpr (kPairs) {
            if (i + 1 < n_w) {
                // i is even here, so i + 1 lies in the same 32-entry window round
                const int st0 = i % STAGES, st1 = (i + 1) % STAGES;
                if (!mbar_wait_bounded(&wbar[st0], (i / STAGES) & 1, wait_limit_ns()) ||
                    !mbar_wait_bounded(&wbar[st1], ((i + 1) / STAGES) & 1, wait_limit_ns())) {
                    failed = true;
                    break;
                }
                const int id0 = block_id(i), id1 = block_id(i + 1);
                const int j0 = b0 + warp + i * NW, j1 = j0 + NW;
                const int valid0 = id0 < 0 ? 0 : min(B, L - j0 * B);
                const int valid1 = id1 < 0 ? 0 : min(B, L - j1 * B);
                uint8_t* stage0 = wring + st0 * 2 * kTile;
                uint8_t* stage1 = wring + st1 * 2 * kTile;
                if (owns_last) {
                    if constexpr (FP8) {
                        if (j0 == last_block && id0 >= 0)
                            append_newest_token_e4m3<T, D, B>(p, new_row8, stage0, id0, kvh, (L - 1) % B, lane);
                        if (j1 == last_block && id1 >= 0)
                            append_newest_token_e4m3<T, D, B>(p, new_row8, stage1, id1, kvh, (L - 1) % B, lane);
                    } else {
                        if (j0 == last_block && id0 >= 0)
                            append_newest_token<T, D, B>(p, new_row, stage0, id0, kvh, (L - 1) % B, lane);
                        if (j1 == last_block && id1 >= 0)
                            append_newest_token<T, D, B>(p, new_row, stage1, id1, kvh, (L - 1) % B, lane);
                    }
                }
                acc.template block2<FP8>(smem_u32(stage0), smem_u32(stage0 + kTile), valid0, smem_u32(stage1),
                                         smem_u32(stage1 + kTile), valid1, group, score_scale, lane);
                __syncwarp();
                if (i + STAGES < n_w) {
                    issue(i + STAGES);
                    ++issued;
                }
                if (i + 1 + STAGES < n_w) {
                    issue(i + 1 + STAGES);
                    ++issued;
                }
                ++i;   // the loop's increment moves past the pair
                continue;
            }
        }
        const int st = i % STAGES;
        if (!mbar_wait_bounded(&wbar[st], (i / STAGES) & 1, wait_limit_ns())) {
            failed = true;
            break;
        }
        const int id = block_id(i);
        const int j = b0 + warp + i * NW;  // logical block index
        const int valid = id < 0 ? 0 : min(B, L - j * B);
        uint8_t* stage = wring + st * 2 * kTile;
        if constexpr (FP8) {
            if (owns_last && j == last_block && id >= 0)
                append_newest_token_e4m3<T, D, B>(p, new_row8, stage, id, kvh, (L - 1) % B, lane);
            acc.template block<true>(smem_u32(stage), smem_u32(stage + kTile), valid, group, score_scale, lane);
        } else {
            if (owns_last && j == last_block && id >= 0)
                append_newest_token<T, D, B>(p, new_row, stage, id, kvh, (L - 1) % B, lane);
            if constexpr (kF32) {
                acc.block(reinterpret_cast<const float*>(stage), reinterpret_cast<const float*>(stage + kTile),
                          valid, group, score_scale, lane);
            } else {
                acc.block(smem_u32(stage), smem_u32(stage + kTile), valid, group, score_scale, lane);
            }
        }
        __syncwarp();
        if (i + STAGES < n_w) {
            issue(i + STAGES);
            ++issued;
        }
    }
    if (failed) {
        if (lane == 0) flag_error(8 /* PA_DEVERR_TIMEOUT */);
        // Let the copies already in flight land before the CTA may exit.
        for (int k = i; k < issued; ++k) mbar_wait_bounded(&wbar[k % STAGES], (k / STAGES) & 1, wait_limit_ns());
    }
    const int any_failed = __syncthreads_or(failed ? 1 : 0);

    constexpr bool kLog2 = !kF32;
    // Split mode writes fp32 partials, except that with the fused merge a
    // sequence with a single partition is finished here; the shared-prefix
    // form always writes its partial, to the last slot.
    const int num_parts = SPLIT ? (nblk + p.partition_blocks - 1) / p.partition_blocks
                                : (PREFIX ? p.num_partitions : 1);
    const bool to_workspace = (SPLIT && !(p.counters != nullptr && num_parts == 1)) || PREFIX;
    const int slot_part = PREFIX ? p.num_partitions - 1 : part;
    if (any_failed) {
        // A copy timed out (PA_DEVERR_TIMEOUT is set; the outputs are then not
        // the attention result).  A partition is recorded as empty (max -inf,
        // sum 0, zero output) so that no merge reads what an earlier call left
        // in the workspace, and the fused merge below still counts it, which
        // brings the arrival counter back to zero.
        if constexpr (!SPLIT && !PREFIX) {
            return;
        } else {
            if (!to_workspace) return;
            for (int idx = threadIdx.x; idx < group * D; idx += NW * 32) {
                const int r = idx / D, d = idx - r * D;
                const long long slot =
                    (static_cast<long long>(s) * p.num_q_heads + kvh * group + r) * p.num_partitions + slot_part;
                p.part_acc[slot * D + d] = 0.f;
                if (d == 0) {
                    p.part_ml[slot * 2] = kNegInf;
                    p.part_ml[slot * 2 + 1] = 0.f;
                }
            }
        }
    }

    // ---- merge the warps' states (the ring is free now)
    float* mo = reinterpret_cast<float*>(smem);
    float* mml = mo + NW * kMaxGroup * kMergeRow<D>;
    if (!any_failed) {
        acc.store_smem(mo, mml, warp, group, lane);
        __syncthreads();
    }
    for (int idx = threadIdx.x; idx < (any_failed ? 0 : group * D); idx += NW * 32) {
        const int r = idx / D, d = idx - r * D;
        float M = kNegInf;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, mml[(w * kMaxGroup + r) * 2]);
        float num = 0.f, den = 0.f;
        if (M != kNegInf) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float wt = softmax_exp<kLog2>(mml[(w * kMaxGroup + r) * 2] - M);
                num = fmaf(wt, mo[(w * kMaxGroup + r) * kMergeRow<D> + d], num);
                den = fmaf(wt, mml[(w * kMaxGroup + r) * 2 + 1], den);
            }
        }
        num *= out_scale;  // 8-bit pools: the V scale
        const int h = kvh * group + r;
        if (to_workspace) {
            const long long slot = (static_cast<long long>(s) * p.num_q_heads + h) * p.num_partitions + slot_part;
            p.part_acc[slot * D + d] = num;
            if (d == 0) {
                p.part_ml[slot * 2] = M;
                p.part_ml[slot * 2 + 1] = den;
            }
        } else {
            T* out = reinterpret_cast<T*>(p.out) + (static_cast<long long>(s) * p.num_q_heads + h) * D;
            out[d] = from_float<T>(den > 0.f ? num / den : 0.f);
        }
    }
    if constexpr (SPLIT || PREFIX) {
        if (p.counters != nullptr && to_workspace) {
            // Fused merge: the CTA that records the last partition merges them
            // (shared-prefix form: the last of the prefix pass's partitions
            // and this pass, whichever kernel it runs in).
            __shared__ int last_arrival;
            __threadfence();
            __syncthreads();
            if (threadIdx.x == 0) {
                const int old = atomicAdd(p.counters + static_cast<long long>(s) * p.num_kv_heads + kvh, 1);
                last_arrival = old == num_parts - 1;
            }
            __syncthreads();
            if (last_arrival) {
                __threadfence();
                if constexpr (PREFIX) {
                    const bool refused = shared_prefix_refused(L, p.first_block * B, p.new_key != nullptr);
                    for (int v = threadIdx.x; v < group * D / 4; v += NW * 32) {
                        const long long row[1] = {static_cast<long long>(s) * p.num_q_heads + kvh * group + (4 * v) / D};
                        const int c[1] = {v % (D / 4)};
                        const bool use[1] = {true}, zero[1] = {refused};
                        merge_shared_prefix<T, D, 1>(p.out, p.part_acc, p.part_ml, num_parts, row, c, use, zero);
                    }
                } else {
                    merge_partitions_cta<T, D, kLog2, NW * 32>(p, s, kvh, num_parts);
                }
                if (threadIdx.x == 0) p.counters[static_cast<long long>(s) * p.num_kv_heads + kvh] = 0;
            }
        }
    }
    prefix_pass_done();
}

// ----------------------------------------------------------------------------
// Log-sum-exp merge of the partitions: one warp per (sequence, query head).

struct MergeParams {
    void* out;
    const float* part_acc;
    const float* part_ml;
    const int32_t* context_lens;
    int num_seqs;
    int num_q_heads;
    int context_cap;
    int block_size;
    int partition_blocks;
    int num_partitions;
};

template <typename T, int D, bool LOG2>
__global__ void __launch_bounds__(128) pa_merge_kernel(const __grid_constant__ MergeParams p) {
    wait_for_prior_work();
    constexpr int kPer = D / 32;
    const int lane = threadIdx.x & 31;
    const long long gw = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
    if (gw >= static_cast<long long>(p.num_seqs) * p.num_q_heads) return;
    const int s = static_cast<int>(gw / p.num_q_heads);
    int L = p.context_lens[s];
    L = L < 0 ? 0 : (L > p.context_cap ? p.context_cap : L);
    const int nblk = (L + p.block_size - 1) / p.block_size;
    const int np = (nblk + p.partition_blocks - 1) / p.partition_blocks;
    T* out = reinterpret_cast<T*>(p.out) + gw * D + lane * kPer;
    const float* ml = p.part_ml + gw * p.num_partitions * 2;
    const float* acc = p.part_acc + gw * p.num_partitions * D + lane * kPer;

    float M = kNegInf;
    for (int q = lane; q < np; q += 32) M = fmaxf(M, ml[2 * q]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));

    float num[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) num[e] = 0.f;
    float den = 0.f;
    if (M != kNegInf) {
        for (int base = 0; base < np; base += 32) {
            // lane q holds the weight of partition base+q
            float wq = 0.f, lq = 0.f;
            if (base + lane < np) {
                wq = softmax_exp<LOG2>(ml[2 * (base + lane)] - M);
                lq = ml[2 * (base + lane) + 1];
            }
            const int cnt = min(32, np - base);
            for (int q = 0; q < cnt; ++q) {
                const float w = __shfl_sync(0xffffffffu, wq, q);
                const float l = __shfl_sync(0xffffffffu, lq, q);
                den = fmaf(w, l, den);
                const float* a = acc + static_cast<long long>(base + q) * D;
                if constexpr (kPer == 4) {
                    const float4 v = *reinterpret_cast<const float4*>(a);
                    num[0] = fmaf(w, v.x, num[0]);
                    num[1] = fmaf(w, v.y, num[1]);
                    num[2] = fmaf(w, v.z, num[2]);
                    num[3] = fmaf(w, v.w, num[3]);
                } else {
                    const float2 v = *reinterpret_cast<const float2*>(a);
                    num[0] = fmaf(w, v.x, num[0]);
                    num[1] = fmaf(w, v.y, num[1]);
                }
            }
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int e = 0; e < kPer; ++e) out[e] = from_float<T>(den > 0.f ? num[e] * inv : 0.f);
}

}  // namespace pa
