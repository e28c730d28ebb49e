// Chunked prefill on the 5th-generation tensor cores (tcgen05): the same
// computation as pa_prefill_kernel ("vLLM核心架构总览" §4.3 chunked prefill,
// causal attention of each sequence's newest Q tokens over its paged context).
//
//  * One CTA (448 threads, one per SM) per (sequence, kv head, pair of query
//    tiles), or with QT = 1 two CTAs per SM (256 threads) of one query tile
//    each.  A query tile is 128 MMA rows, (query token, head of the GQA group)
//    pairs, 128 / g tokens; in a softmax warpgroup thread t owns row t, which
//    is tensor-memory lane t.  The tiles of a CTA share every K/V tile.
//  * Key tiles of 64 keys (8, 4 or 2 pool blocks of 8, 16 or 32 tokens), so
//    that S = Q K^T is one N = 64 MMA per 16-dim step.  With 16- and 32-token
//    blocks K arrives chunk-major, [D/8][64][8], by tile::gather4 loads (one
//    8-dim chunk of four pool blocks per load, two chunks of two blocks for
//    32-token blocks); an 8-token block's (block, head) tile [D/8][8][8] is
//    already one column of the operand's core matrices, so those tiles arrive
//    whole by 1-D bulk copies and the MMA steps from block to block with a
//    stride of one tile.  V arrives as whole (block, head) tiles [D/8][B][8]
//    by 1-D bulk copies, the MN-major B operand of O += P V as stored (with
//    8-token blocks one 16-key step reads two adjacent tiles).  K and V have
//    three-stage rings of their own.
//  * Warp roles: 0-3 and 4-7 softmax of query tile 0 and 1; 8 and 9 issue
//    S = Q K^T for query tile 0 and 1 (Q and K in shared memory); 10 and 11
//    issue O += P V for query tile 0 and 1 (P in tensor memory, V in shared
//    memory); 12 and 13 fetch K and V.  One issuer per query tile keeps each
//    tile's chain of MMAs from waiting on the other tile's.  tcgen05.commit
//    arrives on the mbarriers the other roles wait on, every wait bounded; a K
//    or V stage is free once both tiles' issuers committed it.
//  * Per query tile, S (64 fp32 columns), O (D columns) and two P buffers (32
//    columns of 16-bit pairs each) live in tensor memory.  The softmax warps
//    read their S row with tcgen05.ld, mask (causal, refused blocks), run the
//    online softmax in base 2, write the P row with one tcgen05.st and rescale
//    their O row in tensor memory when the reference maximum moves.
//  * Tokens past the context in the last block are zeroed in the staged V tile
//    (P is 0 there, but 0 times a stale non-finite value would not be); blocks
//    with a refused id are never fetched and their keys are masked.
//  * Tensor memory is allocated after every early exit and released on every
//    path.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "pa_device.cuh"

namespace pa {

namespace tc {

__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    // no swizzle; start, leading and stride byte offsets in 16-byte units; version 1
    return static_cast<uint64_t>((addr >> 4) & 0x3fffu) | (static_cast<uint64_t>((lbo >> 4) & 0x3fffu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3fffu) << 32) | (1ull << 46);
}

// kind::f16 instruction descriptor: fp32 accumulator, A/B 16-bit (bf16 = 1,
// fp16 = 0), A K-major, B K-major (b_mn = 0) or MN-major (1), M = 128, N.
template <typename T>
__device__ __forceinline__ uint32_t instr_desc(int n, bool b_mn) {
    constexpr uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((b_mn ? 1u : 0u) << 16) |
           (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

__device__ __forceinline__ void mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

// Same, with A (128 x 16) read from tensor memory: lane = row, 32-bit column c
// = elements (2c, 2c+1) of the K step, low half first.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

__device__ __forceinline__ void commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 columns of this warp's 32 lanes, without waiting (tcgen05.wait::ld follows).
__device__ __forceinline__ void ld32_nowait(uint32_t taddr, float* v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void st32u(uint32_t taddr, const uint32_t (&w)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),
          "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15]),
          "r"(w[16]), "r"(w[17]), "r"(w[18]), "r"(w[19]), "r"(w[20]), "r"(w[21]), "r"(w[22]), "r"(w[23]),
          "r"(w[24]), "r"(w[25]), "r"(w[26]), "r"(w[27]), "r"(w[28]), "r"(w[29]), "r"(w[30]), "r"(w[31])
        : "memory");
}

__device__ __forceinline__ void st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
          "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
          "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
          "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
          "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
          "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
          "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
          "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
          "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
          "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
          "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

// Four rows of a 2-D tensor (row coordinates r0..r3, columns from `col`, one
// box wide) into consecutive shared memory; completion counted on `bar`.
__device__ __forceinline__ void gather4(void* dst, const CUtensorMap* map, int col, int r0, int r1, int r2, int r3,
                                        uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(col), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(smem_u32(bar))
        : "memory");
}

// Global -> shared bulk copy with the default L2 policy (prefill rereads a
// sequence's tiles once per query tile, so they should stay in L2).
__device__ __forceinline__ void bulk_copy(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Packed pairs of fp32 (one 64-bit register pair): fused multiply-add and add
// on both halves in one instruction.
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

}  // namespace tc

// One CTA per SM holds two tiles of 128 query rows (two consecutive tiles of
// the same sequence and kv head) that share every K and V tile it fetches.
// One key tile per MMA round: 64 keys (4 blocks of 16 tokens or 2 of 32).
// K and V tiles have rings of their own: a K stage is free once the S MMAs
// of both query tiles finish, a V stage once both O += P V finish.  A K stage
// holds the tile chunk-major, [D/8][64 keys][8], gathered from the pool's
// (block, head) tiles by tile::gather4 loads (one 8-dim chunk of four blocks
// per load), so that one N = 64 MMA covers all of the tile's keys.
template <typename T, int D, int B, int QT = 2>
struct PrefillTcSmem {
    static constexpr int kKeys = 64;
    static constexpr int kBlocks = kKeys / B;             // blocks per key tile
    static constexpr int kTile = B * D * 2;               // one (block, head) K or V tile
    static constexpr int kStage = kBlocks * kTile;        // the K (or V) tiles of one key tile
#ifndef PA_PF_STAGES
#define PA_PF_STAGES 3
#endif
    // (one query tile per CTA: two CTAs share an SM, so two stages each)
    static constexpr int kKStages = QT == 2 ? (D == 128 ? PA_PF_STAGES : PA_PF_STAGES + 2) : (D == 128 ? 2 : 4);
    static constexpr int kVStages = kKStages;
    static constexpr int kQ = 128 * D * 2;                // one query tile, core-matrix layout
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kKStages * kStage;
    static constexpr int kQOff = kVOff + kVStages * kStage;   // [query tile]
    static constexpr int kBarOff = kQOff + QT * kQ;
    static constexpr int kMiscOff = kBarOff + 48 * 8;     // tmem base, abort
    static constexpr int kTotal = kMiscOff + 16;
    static_assert(kTotal <= (QT == 2 ? 232448 : 115712), "shared memory per CTA");
    static_assert(kKStages <= 6, "barrier slots");
    // the barrier set-up and both producers index the K and V rings with one
    // stage count
    static_assert(kVStages == kKStages, "K and V rings of one depth");
};

// Bounded mbarrier wait that also gives up when another role of the CTA has
// raised `abort` (a timed-out wait raises it and flags PA_DEVERR_TIMEOUT).
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t start = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort) return false;
        if (global_timer_ns() - start > kWaitLimitNs) {
            *abort = 1u;
            flag_error(8 /* PA_DEVERR_TIMEOUT */);
            return false;
        }
    }
    return true;
}

// Warps 0-3 and 4-7: softmax of query tile 0 and 1 (thread = row = tensor-memory
// lane); warps 8 / 9 issue S = Q K^T and 10 / 11 O += P V for query tile 0 / 1;
// warps 12 and 13 fetch K and V (QT = 1: warps 0-3, 4, 5, 6 and 7).
template <typename T, int D, int B, bool PREFIX = false, int QT = 2>
__global__ void __launch_bounds__((6 * QT + 2) * 32, QT == 2 ? 1 : 2) pa_prefill_tc_kernel(const __grid_constant__ PrefillParams p,
                                                                const __grid_constant__ CUtensorMap k_rows) {
    using Sm = PrefillTcSmem<T, D, B, QT>;
    constexpr int kKeys = Sm::kKeys, kBlocks = Sm::kBlocks, kTile = Sm::kTile;
    constexpr int KS = Sm::kKStages, VS = Sm::kVStages;
    // tensor memory, per query tile q (256 columns at q * 256): S [0, 64),
    // O [64, 64 + D), P (16-bit pairs per column, two buffers of 32 columns)
    constexpr uint32_t kTmemCols = QT * 256;
    // warp roles: softmax [0, 4 QT), S issuers [4 QT, 5 QT), O += P V issuers
    // [5 QT, 6 QT), K producer 6 QT, V producer 6 QT + 1
    constexpr int kThreads = (6 * QT + 2) * 32;
    constexpr int kSoftWarps = 4 * QT, kSIss = 4 * QT, kPVIss = 5 * QT, kProdK = 6 * QT, kProdV = 6 * QT + 1;
    constexpr uint32_t kOCol = kKeys, kPCol = kKeys + D;
    static_assert(kPCol + kKeys <= 256, "tensor memory budget");
    static_assert(B == 8 || B == 16 || B == 32, "8-, 16- or 32-token blocks");
    static_assert(D == 64 || D == 128, "head dims");
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sm::kBarOff);
    uint64_t* k_full = bars;         // [KS] K tiles of a key tile landed
    uint64_t* k_empty = bars + 6;    // [KS] the S MMAs reading them finished
    uint64_t* v_full = bars + 12;    // [VS] V tiles landed
    uint64_t* v_empty = bars + 18;   // [VS] the O += P V reading them finished
    uint64_t* s_full = bars + 24;    // [q] S = Q K^T finished
    uint64_t* s_free = bars + 26;    // [q] the softmax warps have read S
    uint64_t* p_full = bars + 28;    // [q * 2 + buffer] P written (and O rescaled)
    uint64_t* p_free = bars + 32;    // [q * 2 + buffer] the O += P V reading that P finished
    uint64_t* drain = bars + 36;     // [4] each issuer's MMAs finished
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Sm::kMiscOff);
    volatile uint32_t* abort = misc + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    wait_for_prior_work();   // (the shared-prefix form's decode pass may then start: it overlaps this grid)
    // PREFIX: the table of row 0 holds the shared prefix; blockIdx.z is the key partition
    const int kvh = blockIdx.y, s = PREFIX ? 0 : static_cast<int>(blockIdx.z);
    const int group = p.group;

    int q0, Q, L, tb = 0;   // tb: the first key tile of this CTA
    if constexpr (PREFIX) {
        // (the decode pass of the sequences' own blocks shares nothing with
        // this grid but the arrival counters)
        // every sequence's decode query is one "token" of the chunk, and all of
        // the prefix is visible to it
        q0 = 0;
        Q = p.num_seqs;
        L = p.prefix_len;
        tb = static_cast<int>(blockIdx.z) * p.prefix_tiles;
        if (L <= 0 || L > p.context_cap) {   // (the host never launches such a pass)
            if (tid == 0 && blockIdx.x == 0 && kvh == 0 && blockIdx.z == 0) flag_error(2 /* PA_DEVERR_CONTEXT_LEN */);
            return;
        }
    } else {
        q0 = p.query_start[s];
        Q = p.query_start[s + 1] - q0;
        L = p.context_lens[s];
        if (L < 0 || L > p.context_cap || Q < 0 || Q > L) {
            if (tid == 0 && blockIdx.x == 0 && kvh == 0) flag_error(2 /* PA_DEVERR_CONTEXT_LEN */);
            return;
        }
    }
    // query tile q covers tokens [tok0[q], tok1[q]) of the chunk; nt[q] key tiles
    int tok0[2], tok1[2], nt[2];
#ifndef PA_PF_HEAVY_FIRST
#define PA_PF_HEAVY_FIRST 1
#endif
    // the latest query tiles of a sequence see the most keys: launch them first
    const int tile = PA_PF_HEAVY_FIRST ? static_cast<int>(gridDim.x - 1 - blockIdx.x) : static_cast<int>(blockIdx.x);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        tok0[q] = q < QT ? (QT * tile + q) * p.tile_tokens : Q;
        tok1[q] = min(Q, tok0[q] + p.tile_tokens);
        if constexpr (PREFIX) {
            nt[q] = tok0[q] < Q ? min(p.prefix_tiles, (L + kKeys - 1) / kKeys - tb) : 0;
        } else {
            nt[q] = tok0[q] < Q ? ((L - Q + tok1[q] - 1) / B + kBlocks) / kBlocks : 0;
        }
    }
    // Shared-prefix form, the CTA's last step: its sequences [tok0[0], seq_end)
    // arrive on their (sequence, kv head) counters once its partials are
    // written (`empty`: empty partials written here first); the last of the
    // num_partitions arrivals of a sequence merges its partials into `out`.
    // The K ring holds the list of sequences this CTA merges.
    auto prefix_finish = [&](bool empty) {
        if constexpr (PREFIX) {
            const int seq_end = min(Q, tok0[0] + QT * p.tile_tokens);
            const int rows = (seq_end - tok0[0]) * group;
            if (empty) {
                for (int i = tid; i < rows * (D + 2); i += kThreads) {
                    const int r = i / (D + 2), e = i % (D + 2);
                    const long long slot = (static_cast<long long>(tok0[0] + r / group) * p.num_q_heads +
                                            kvh * group + r % group) * p.num_partitions + blockIdx.z;
                    if (e < D) p.part_acc[slot * D + e] = 0.f;
                    else p.part_ml[slot * 2 + (e - D)] = e == D ? kNegInf : 0.f;
                }
            }
            int* merge_list = reinterpret_cast<int*>(smem + Sm::kKOff);
            volatile uint32_t* n_merge = misc + 2;
            if (tid == 0) *n_merge = 0u;
            __threadfence();   // this CTA's partials before its arrivals
            __syncthreads();
            for (int t = tok0[0] + tid; t < seq_end; t += kThreads) {
                const int old = atomicAdd(p.counters + static_cast<long long>(t) * p.num_kv_heads + kvh, 1);
                if (old == p.num_partitions - 1) merge_list[atomicAdd(const_cast<uint32_t*>(n_merge), 1u)] = t;
            }
            __syncthreads();
            const int n = static_cast<int>(*n_merge);
            if (n > 0) {
                __threadfence();
                // two outputs per thread and step (eight loads in flight)
                constexpr int kU = 2;
                const int slices = group * D / 4;
                for (int w0 = tid; w0 < n * slices; w0 += kU * kThreads) {
                    long long row[kU];
                    int c[kU];
                    bool use[kU], zero[kU];
#pragma unroll
                    for (int u = 0; u < kU; ++u) {
                        const int w = w0 + u * kThreads;
                        use[u] = w < n * slices;
                        const int t = use[u] ? merge_list[w / slices] : 0, v = w % slices;
                        int Lt = use[u] ? p.context_lens[t] : 0;
                        Lt = Lt < 0 ? 0 : (Lt > p.context_cap ? p.context_cap : Lt);   // as the decode pass reads it
                        zero[u] = shared_prefix_refused(Lt, L, p.prefix_append != 0);
                        row[u] = static_cast<long long>(t) * p.num_q_heads + kvh * group + (4 * v) / D;
                        c[u] = v % (D / 4);
                    }
                    merge_shared_prefix<T, D, kU>(p.out, p.part_acc, p.part_ml, p.num_partitions, row, c, use, zero);
                }
                for (int i = tid; i < n; i += kThreads)
                    p.counters[static_cast<long long>(merge_list[i]) * p.num_kv_heads + kvh] = 0;
            }
        }
    };
    if (nt[0] <= 0) return;   // (no sequence: tok0[0] >= Q; the host gives every key partition a tile)
    const int ntiles = max(nt[0], nt[1]);                           // key tiles fetched (>= 1)
    // blocks needed (absolute: block index from the start of the table row)
    const int nblk = PREFIX ? (L + B - 1) / B : (L - Q + (nt[1] ? tok1[1] : tok1[0]) - 1) / B + 1;
    // tensor copies land on 128-byte boundaries (the dynamic window starts on one)
    if (smem_u32(smem) & 127u) {
        if (tid == 0) flag_error(8 /* PA_DEVERR_TIMEOUT: nothing fetched */);
        prefix_finish(true);
        return;
    }

    if (tid == kSIss * 32) {
        for (int i = 0; i < KS; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], QT);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], QT);
        }
        for (int q = 0; q < QT; ++q) {
            mbar_init(&s_full[q], 1);
            mbar_init(&s_free[q], 4);
            for (int b = 0; b < 2; ++b) {
                mbar_init(&p_full[q * 2 + b], 128);
                mbar_init(&p_free[q * 2 + b], 1);
            }
        }
        for (int d = 0; d < 2 * QT; ++d) mbar_init(&drain[d], 1);
        *abort = 0u;
        fence_barrier_init();
    }
    if (warp == kSIss) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(misc)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = misc[0];

    // ---- block ids of key tile j, and which of them may be fetched (every role
    //      derives the same mask from the table)
    const int32_t* table = p.block_tables + static_cast<long long>(s) * p.max_blocks_per_seq;
    auto load_ids = [&](int j, int (&ids)[kBlocks]) {
#pragma unroll
        for (int b = 0; b < kBlocks; ++b) {
            const int jb = (tb + j) * kBlocks + b;
            ids[b] = (j < ntiles && jb < nblk) ? __ldg(table + jb) : -1;
        }
    };
    // The same mask computed by a whole warp: lane b loads block b's id (the
    // id of lane `lane` for tile j; -1 past the need), a ballot gathers them.
    auto lane_id = [&](int j) -> int {
        const int jb = (tb + j) * kBlocks + lane;
        return (lane < kBlocks && j < ntiles && jb < nblk) ? __ldg(table + jb) : -1;
    };
    auto ok_ballot = [&](int id) -> uint32_t {
        return __ballot_sync(0xffffffffu, id >= 0 && static_cast<long long>(id) < p.num_blocks);
    };
    auto ok_of = [&](const int (&ids)[kBlocks]) {
        uint32_t ok = 0;
#pragma unroll
        for (int b = 0; b < kBlocks; ++b)
            if (ids[b] >= 0 && static_cast<long long>(ids[b]) < p.num_blocks) ok |= 1u << b;
        return ok;
    };

    // ---- producers: warp 12 lane 0 fetches K tiles, warp 13 lane 0 V tiles
    const bool is_producer = (warp == kProdK || warp == kProdV) && lane == 0;
    const bool v_side = warp == kProdV;
    const char* vpool = reinterpret_cast<const char*>(p.v_cache);
    uint64_t* full = v_side ? v_full : k_full;
    uint64_t* empty = v_side ? v_empty : k_empty;
    constexpr int nst = KS;
    uint8_t* ring = smem + (v_side ? Sm::kVOff : Sm::kKOff);
    int ids[kBlocks], nxt[kBlocks];
    int issued = 0;
    auto produce = [&](int j) {   // copies of key tile j (ids in `ids`) into stage j % nst
        const int st = j % nst;
        const uint32_t ok = ok_of(ids);
        uint8_t* dst = ring + st * Sm::kStage;
        if (!v_side) {
#pragma unroll
            for (int b = 0; b < kBlocks; ++b)
                if ((tb + j) * kBlocks + b < nblk && !((ok >> b) & 1u)) flag_error(1 /* PA_DEVERR_BLOCK_ID */);
            if constexpr (B == 8) {
                // 8-token blocks: a (block, head) tile, [D/8][8][8], is already a
                // column of core matrices of the S MMA's K-major operand, so the
                // stage holds whole tiles (block-major) by 1-D bulk copies and the
                // MMA steps over blocks with a stride of one tile.  A refused or
                // unneeded block is not fetched: its scores are masked.
                mbar_arrive_expect_tx(&full[st], __popc(ok) * kTile);
#pragma unroll
                for (int b = 0; b < kBlocks; ++b) {
                    if (!((ok >> b) & 1u)) continue;
                    const long long off = (static_cast<long long>(ids[b]) * p.num_kv_heads + kvh) * kTile;
                    tc::bulk_copy(dst + b * kTile, reinterpret_cast<const char*>(p.k_cache) + off, kTile, &full[st]);
                }
            } else if (ok == 0u) {
                mbar_arrive_expect_tx(&full[st], 0);   // nothing to fetch: every key is masked
            } else {
                // refused ids and blocks past the need read a fetched block instead
                // (their scores are masked); row (id, head, chunk c) of the 2-D view
                int rid[kBlocks];
                int sub = ids[kBlocks - 1];
#pragma unroll
                for (int b = kBlocks - 1; b >= 0; --b)
                    if ((ok >> b) & 1u) sub = ids[b];   // the first fetched block
#pragma unroll
                for (int b = 0; b < kBlocks; ++b)
                    rid[b] = ((((ok >> b) & 1u) ? ids[b] : sub) * p.num_kv_heads + kvh) * (D / 8);
                mbar_arrive_expect_tx(&full[st], Sm::kStage);
                if constexpr (B <= 16) {   // four blocks' rows of chunk c per load
#pragma unroll
                    for (int c = 0; c < D / 8; ++c)
#pragma unroll
                        for (int g = 0; g < kBlocks / 4; ++g)
                            tc::gather4(dst + c * 1024 + g * (4 * B * 16), &k_rows, 0, rid[4 * g] + c,
                                        rid[4 * g + 1] + c, rid[4 * g + 2] + c, rid[4 * g + 3] + c, &full[st]);
                } else {
#pragma unroll
                    for (int c = 0; c < D / 8; c += 2)
                        tc::gather4(dst + c * 1024, &k_rows, 0, rid[0] + c, rid[1] + c, rid[0] + c + 1,
                                    rid[1] + c + 1, &full[st]);
                }
            }
        } else if constexpr (B == 8) {
            // One 16-key MMA step spans two 8-token blocks, so every block of a
            // tile with any fetchable one is fetched: a refused or unneeded one
            // as the tile's first fetchable block (P is 0 on its keys), so that
            // no step reads stale shared memory.
            int sub = ids[kBlocks - 1];
#pragma unroll
            for (int b = kBlocks - 1; b >= 0; --b)
                if ((ok >> b) & 1u) sub = ids[b];
            mbar_arrive_expect_tx(&full[st], ok != 0u ? kBlocks * kTile : 0);
            if (ok != 0u) {
#pragma unroll
                for (int b = 0; b < kBlocks; ++b) {
                    const int id = ((ok >> b) & 1u) ? ids[b] : sub;
                    const long long off = (static_cast<long long>(id) * p.num_kv_heads + kvh) * kTile;
                    tc::bulk_copy(dst + b * kTile, vpool + off, kTile, &full[st]);
                }
            }
        } else {
            mbar_arrive_expect_tx(&full[st], __popc(ok) * kTile);
#pragma unroll
            for (int b = 0; b < kBlocks; ++b) {
                if (!((ok >> b) & 1u)) continue;
                const long long off = (static_cast<long long>(ids[b]) * p.num_kv_heads + kvh) * kTile;
                tc::bulk_copy(dst + b * kTile, vpool + off, kTile, &full[st]);
            }
        }
        issued = j + 1;
    };
    if (is_producer) {
        load_ids(0, ids);
        for (int j = 0; j < nst && j < ntiles; ++j) {
            load_ids(j + 1, nxt);
            produce(j);
#pragma unroll
            for (int b = 0; b < kBlocks; ++b) ids[b] = nxt[b];
        }
    }

    // ---- softmax warps: Q row into tensor memory (pairs packed per 32-bit column), O = 0
    const int qt = warp >> 2;                          // query tile of a softmax warp
    const int my_tok0 = qt == 1 ? tok0[1] : tok0[0];
    const int my_tok1 = qt == 1 ? tok1[1] : tok1[0];
    const int my_nt = qt == 1 ? nt[1] : nt[0];
    const int row = tid & 127;
    const bool softmax_warp = warp < kSoftWarps && my_nt > 0;
    const int row_tok = my_tok0 + row / group;
    const int row_head = kvh * group + row % group;
    const bool row_ok = warp < kSoftWarps && row_tok < my_tok1;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t qbase = tmem + static_cast<uint32_t>(qt & 1) * 256u;
    const uint32_t s_tmem = qbase, o_tmem = qbase + kOCol, p_tmem = qbase + kPCol;
    if (softmax_warp) {
        // Q row into shared memory, K-major core-matrix layout: (8-row group g,
        // 8-dim chunk c) at c * 2048 + g * 128
        const T* qrow = reinterpret_cast<const T*>(p.q) +
                        (static_cast<long long>(q0 + (row_ok ? row_tok : my_tok0)) * p.num_q_heads + row_head) * D;
        uint8_t* qs = smem + Sm::kQOff + (qt & 1) * Sm::kQ;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
            const uint4 v = row_ok ? *reinterpret_cast<const uint4*>(qrow + 8 * c) : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(qs + c * 2048 + (row >> 3) * 128 + (row & 7) * 16) = v;
        }
        fence_proxy_async_smem();   // Q (generic stores) visible to the tensor cores
        float z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) tc::st32(o_tmem + lane_base + c0, z);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();

    bool failed = false;
    if (warp == kProdK || warp == kProdV) {
        // ---------------- producers
        if (is_producer) {
            for (int j = nst; j < ntiles; ++j) {
                load_ids(j + 1, nxt);   // the next tile's ids load while this one waits for its stage
                if (!tc_wait(&empty[j % nst], ((j / nst) - 1) & 1, abort)) break;
                produce(j);
#pragma unroll
                for (int b = 0; b < kBlocks; ++b) ids[b] = nxt[b];
            }
            // no copy may still be landing when the CTA leaves
            for (int k = issued > nst ? issued - nst : 0; k < issued; ++k)
                mbar_wait_bounded(&full[k % nst], (k / nst) & 1, kWaitLimitNs);
        }
    } else if (warp >= kSIss && warp < kSIss + QT) {
        // ---------------- S = Q K^T issue (lane 0), one warp per query tile
        const int q = warp - kSIss;
        if (lane == 0) {
            const uint32_t idesc_s = tc::instr_desc<T>(kKeys, false);
            const uint32_t k_ring = smem_u32(smem + Sm::kKOff);
            int id_n[kBlocks];
            load_ids(0, id_n);
            for (int j = 0; j < ntiles; ++j) {
                const uint32_t ok = ok_of(id_n);
                load_ids(j + 1, id_n);
                if (!tc_wait(&k_full[j % KS], (j / KS) & 1, abort)) break;
                if (j < nt[q]) {
                    // S(j) overwrites S(j - 1): the softmax warps must have read it
                    if (j > 0 && !tc_wait(&s_free[q], (j - 1) & 1, abort)) break;
                    tc::fence_after();
                    const uint32_t kbase = k_ring + (j % KS) * Sm::kStage;
                    const uint32_t qb = tmem + static_cast<uint32_t>(q) * 256u;
                    const uint32_t qs = smem_u32(smem + Sm::kQOff + q * Sm::kQ);
                    if (ok != 0u) {
#pragma unroll
                        for (int kc = 0; kc < D / 16; ++kc)
                            tc::mma(qb, tc::smem_desc(qs + 2 * kc * 2048, 2048, 128),
                                    B == 8 ? tc::smem_desc(kbase + 2 * kc * 128, 128, kTile)    // block-major
                                           : tc::smem_desc(kbase + 2 * kc * 1024, 1024, 128),  // chunk-major
                                    idesc_s, kc > 0);
                    }
                    tc::commit(&s_full[q]);
                }
                tc::commit(&k_empty[j % KS]);
            }
            tc::commit(&drain[q]);
            mbar_wait_bounded(&drain[q], 0, kWaitLimitNs);
        }
    } else if (warp >= kPVIss && warp < kPVIss + QT) {
        // ---------------- O += P V issue (lane 0), one warp per query tile; each warp
        //                  zeroes V rows past the context (the same zeros: harmless twice)
        const int q = warp - kPVIss;
        const uint32_t idesc_o = tc::instr_desc<T>(D, true);
        const uint32_t v_ring = smem_u32(smem + Sm::kVOff);
        int id_n = lane_id(0);
        for (int j = 0; j < ntiles; ++j) {
            const uint32_t ok = ok_ballot(id_n);
            id_n = lane_id(j + 1);
            const int vst = j % VS;
            if (!__all_sync(0xffffffffu, tc_wait(&v_full[vst], (j / VS) & 1, abort))) break;
            if constexpr (!PREFIX) {   // (a shared prefix ends on a block boundary: no tail)
                const int lb = (L - 1) / B - j * kBlocks;
                if (lb >= 0 && lb < kBlocks && ((ok >> lb) & 1u)) {
                    uint8_t* vt = smem + Sm::kVOff + vst * Sm::kStage + lb * kTile;
                    const int t_from = (L - 1) % B + 1;
                    for (int i = lane; i < (B - t_from) * (D / 8); i += 32) {
                        const int t = t_from + i / (D / 8), c = i % (D / 8);
                        *reinterpret_cast<uint4*>(vt + (c * B + t) * 16) = make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
            }
            if (j < nt[q]) {
                const uint32_t vbase = v_ring + vst * Sm::kStage;
                const int pb = q * 2 + (j & 1);
                if (!__all_sync(0xffffffffu, tc_wait(&p_full[pb], (j >> 1) & 1, abort))) break;
                if (lane == 0) {
                    tc::fence_after();
                    const uint32_t qb = tmem + static_cast<uint32_t>(q) * 256u;
                    const uint32_t pt = qb + kPCol + static_cast<uint32_t>(j & 1) * (kKeys / 2);
                    if constexpr (B == 8) {
                        // keys 16 pr .. 16 pr + 15: blocks 2 pr and 2 pr + 1, adjacent
                        // tiles (the next 8 keys one tile further on)
                        for (int pr = 0; pr < kBlocks / 2; ++pr) {
                            if (!((ok >> (2 * pr)) & 3u)) continue;
                            tc::mma_ts(qb + kOCol, pt + 8 * pr, tc::smem_desc(vbase + 2 * pr * kTile, kTile, 128),
                                       idesc_o, true);
                        }
                    } else {
                        for (int b = 0; b < kBlocks; ++b) {
                            if (!((ok >> b) & 1u)) continue;
#pragma unroll
                            for (int ks = 0; ks < B / 16; ++ks)
                                tc::mma_ts(qb + kOCol, pt + (b * B) / 2 + 8 * ks,
                                           tc::smem_desc(vbase + b * kTile + ks * 256, 128, B * 16), idesc_o, true);
                        }
                    }
                    tc::commit(&p_free[pb]);
                }
            }
            if (lane == 0) tc::commit(&v_empty[vst]);
        }
        if (lane == 0) {
            tc::commit(&drain[QT + q]);
            mbar_wait_bounded(&drain[QT + q], 0, kWaitLimitNs);
        }
        __syncwarp();
    } else if (softmax_warp) {
        // ---------------- softmax of query tile qt (thread = row = tensor-memory lane)
        const float scale = p.score_scale;
        const int row_pos = row_ok ? (PREFIX ? INT_MAX : L - Q + row_tok) : -1;
        const uint32_t all_blocks = (1u << kBlocks) - 1u;
        const int n = my_nt;
        uint64_t* sfull = &s_full[qt];
        uint64_t* sfree = &s_free[qt];
        int id_n = lane_id(0);
        uint32_t ok = ok_ballot(id_n);
        float m_run = kNegInf, l_run = 0.f;
        for (int j = 0; j < n; ++j) {
            const int pb = qt * 2 + (j & 1);
            id_n = lane_id(j + 1);
            if (!__all_sync(0xffffffffu, tc_wait(sfull, j & 1, abort))) {
                failed = true;
                break;
            }
            tc::fence_after();
            float sv[kKeys];
#pragma unroll
            for (int c0 = 0; c0 < kKeys; c0 += 32) tc::ld32_nowait(s_tmem + lane_base + c0, sv + c0);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            tc::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sfree);
            const int key0 = (tb + j) * kKeys;
            // row maximum over eight independent partial maxima (no 64-long chain)
            float m8[8];
            if (ok == all_blocks && key0 + kKeys - 1 <= row_pos) {
#pragma unroll
                for (int c = 0; c < 8; ++c) m8[c] = sv[c];
#pragma unroll
                for (int c = 8; c < kKeys; ++c) m8[c & 7] = fmaxf(m8[c & 7], sv[c]);
            } else {
#pragma unroll
                for (int c = 0; c < kKeys; ++c) {
                    const bool vis = ((ok >> (c / B)) & 1u) && key0 + c <= row_pos;
                    sv[c] = vis ? sv[c] : kNegInf;
                    m8[c & 7] = c < 8 ? sv[c] : fmaxf(m8[c & 7], sv[c]);
                }
            }
            float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
            mx *= scale;   // base-2 domain (scale > 0)
            // The reference maximum moves only when a score exceeds it by more
            // than 2^8: P stays <= 256 and O is rescaled far less often (l and
            // O share the reference, so the result is the same softmax).
            const float m_old = m_run;
            m_run = (m_old == kNegInf || mx > m_old + 8.f) ? fmaxf(m_old, mx) : m_old;
            const float mu = m_run == kNegInf ? 0.f : m_run;
            const float alpha = exp2_approx(m_old - mu);
            // P buffer j % 2 was last read by the O += P V of tile j - 2
            if (j >= 2 && !__all_sync(0xffffffffu, tc_wait(&p_free[pb], ((j >> 1) - 1) & 1, abort))) {
                failed = true;
                break;
            }
            // P = 2^(s * scale - mu): arguments and row sums two at a time, the
            // sums in four independent pairs
            const uint64_t scale2 = tc::f2(scale, scale), nmu2 = tc::f2(-mu, -mu);
            uint64_t acc[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[e] = tc::f2(0.f, 0.f);
            uint32_t pw[kKeys / 2];   // P row, 16-bit pairs: the A-operand columns of O += P V
#pragma unroll
            for (int k8 = 0; k8 < kKeys / 8; ++k8) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float x0, x1;
                    tc::f2_split(tc::fma2(tc::f2(sv[8 * k8 + 2 * e], sv[8 * k8 + 2 * e + 1]), scale2, nmu2), x0, x1);
                    const float a0 = exp2_approx(x0), a1 = exp2_approx(x1);
                    acc[e] = tc::add2(acc[e], tc::f2(a0, a1));
                    pw[4 * k8 + e] = Mma<T>::pack(a0, a1);
                }
            }
            static_assert(kKeys / 2 == 32, "one 32-column store");
            tc::st32u(p_tmem + lane_base + static_cast<uint32_t>(j & 1) * (kKeys / 2), pw);
            float rs;
            {
                float r[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) tc::f2_split(acc[e], r[2 * e], r[2 * e + 1]);
                rs = ((r[0] + r[1]) + (r[2] + r[3])) + ((r[4] + r[5]) + (r[6] + r[7]));
            }
            l_run = l_run * alpha + rs;
            // rescale this row of O (after the previous O += P V), unless no
            // row of the warp moved its reference
            if (!__all_sync(0xffffffffu, m_old == kNegInf || alpha == 1.f)) {
                const int pp = qt * 2 + ((j - 1) & 1);
                if (!__all_sync(0xffffffffu, tc_wait(&p_free[pp], ((j - 1) >> 1) & 1, abort))) {
                    failed = true;
                    break;
                }
                tc::fence_after();
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    float v[32];
                    tc::ld32(o_tmem + lane_base + c0, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= alpha;
                    tc::st32(o_tmem + lane_base + c0, v);
                }
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            }
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            tc::fence_before();
            mbar_arrive(&p_full[pb]);
            ok = ok_ballot(id_n);
        }
        // ---- the last O += P V, then this row of the output
        if (!failed && !__all_sync(0xffffffffu, tc_wait(&p_free[qt * 2 + ((n - 1) & 1)], ((n - 1) >> 1) & 1, abort)))
            failed = true;
        if constexpr (PREFIX) {
            // this key partition's unnormalised partial of the row: O, the
            // running reference (base 2) and the sum, in the split-K layout;
            // an empty partial if the pass failed (the error flag is set).
            // O leaves through shared memory, 32 columns at a time, so that
            // each store of the warp writes four whole 128-byte row segments:
            // the warp's 4 KiB slice of its query tile's Q area (no MMA reads
            // Q any more), 16-byte chunk c of row r at chunk c ^ (r % 8)
            // (conflict-free both ways).
            const bool good = __all_sync(0xffffffffu, !failed && !*abort);   // warp-uniform: ld32 is collective
            const long long slot =
                (static_cast<long long>(row_ok ? row_tok : 0) * p.num_q_heads + row_head) * p.num_partitions +
                blockIdx.z;
            if (good) tc::fence_after();
            float* stage = reinterpret_cast<float*>(smem + Sm::kQOff + (qt & 1) * Sm::kQ + (warp & 3) * 4096);
            static_assert(4 * 4096 <= Sm::kQ, "four warps' staging slices fit one query tile's Q area");
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
                float v[32];
                if (good) {
                    tc::ld32(o_tmem + lane_base + c0, v);   // collective per warp: every row takes part
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0.f;
                }
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<float4*>(stage + lane * 32 + ((c ^ (lane & 7)) * 4)) =
                        make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int rr = 4 * i + (lane >> 3), c = lane & 7;   // row of the warp, chunk
                    const int trow = (warp & 3) * 32 + rr;               // row of the query tile
                    const int tok = my_tok0 + trow / group;
                    if (tok < my_tok1) {
                        const long long rs = (static_cast<long long>(tok) * p.num_q_heads + kvh * group + trow % group) *
                                                 p.num_partitions + blockIdx.z;
                        *reinterpret_cast<float4*>(p.part_acc + rs * D + c0 + 4 * c) =
                            *reinterpret_cast<const float4*>(stage + rr * 32 + ((c ^ (rr & 7)) * 4));
                    }
                }
                __syncwarp();
            }
            if (row_ok)
                *reinterpret_cast<float2*>(p.part_ml + slot * 2) =
                    good ? make_float2(m_run, l_run) : make_float2(kNegInf, 0.f);
        } else if (!failed && !*abort) {
            tc::fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            T* dst = reinterpret_cast<T*>(p.out) +
                     (static_cast<long long>(q0 + (row_ok ? row_tok : my_tok0)) * p.num_q_heads + row_head) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                float v[32];
                tc::ld32(o_tmem + lane_base + c0, v);   // collective per warp: every row takes part
                if (row_ok) {
#pragma unroll
                    for (int k8 = 0; k8 < 4; ++k8) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            w[e] = Mma<T>::pack(v[8 * k8 + 2 * e] * inv, v[8 * k8 + 2 * e + 1] * inv);
                        *reinterpret_cast<uint4*>(dst + c0 + 8 * k8) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == kSIss) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
    prefix_finish(false);
}

}  // namespace pa
