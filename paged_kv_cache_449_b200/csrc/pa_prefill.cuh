// Paged chunked prefill ("vLLM核心架构总览" §4.3 chunked prefill): every
// sequence s brings Q_s new query tokens, the newest of its L_s tokens (their
// K/V are already in the pool); query i sits at position L_s - Q_s + i and
// attends causally to the tokens at positions 0 .. L_s - Q_s + i, gathered
// through the block table like decode.
//
// Design:
//  * One CTA per (sequence, kv head, tile of query tokens).  Its NW warps own
//    16 MMA rows each; a row is a (query token, query head of the GQA group)
//    pair (row m -> token m / g, head m % g), so the K/V tiles of the kv head
//    are shared by the whole group.
//  * K/V arrive block by block (one bulk copy of the K tile and one of the V
//    tile) into a CTA-wide ring of STAGES stages.  One thread produces; every
//    warp consumes each stage and then arrives on the stage's "empty"
//    barrier; the producer refills a stage once all warps released it.  All
//    waits are bounded.
//  * Tensor cores (mma.sync m16n8k16, fp32 accumulate), FlashAttention-style
//    register reuse: S = Q K^T with Q as the A operand (registers, loaded
//    once) and K as the B operand (ldmatrix of the [D/8][B][8] tile: rows are
//    tokens); the S accumulators of two 8-token n-tiles are exactly the A
//    fragments of P for O += P V; V is the B operand via ldmatrix.trans.
//  * Online softmax per row in base 2 (scale * log2 e folded in); each thread
//    holds rows r and r + 8 of its warp; row statistics are reduced over the
//    four threads of a quad.
#pragma once

#include "pa_device.cuh"

namespace pa {

struct PrefillParams {
    void* out;                      // [T][Hq][D]
    const void* q;                  // [T][Hq][D]
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;    // [S][max_blocks_per_seq]
    const int32_t* context_lens;    // [S]
    const int32_t* query_start;     // [S + 1]
    float score_scale;              // scale * log2(e)
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int group;
    int max_blocks_per_seq;
    int context_cap;
    long long num_blocks;
    int tile_tokens;                // query tokens per CTA: NW * 16 / group
    // shared-prefix pass (the tensor-core kernel's PREFIX form): the query rows
    // are every sequence's decode query, the keys the prefix_len tokens of the
    // prefix that row 0 of block_tables holds, prefix_tiles 64-key tiles per
    // CTA (key partition = blockIdx.z); unnormalised partials go to slot
    // blockIdx.z of part_acc / part_ml ([S][Hq][num_partitions][D], [..][2]),
    // whose last slot holds the decode pass's partial of the sequence's own
    // blocks.  Each CTA then arrives on counters[s * Hkv + kvh] for its
    // sequences; the last of the num_partitions arrivals merges into `out`
    // (a zero row where context_lens[s] does not reach past the prefix, or,
    // with prefix_append, its newest token would land in it).
    float* part_acc;
    float* part_ml;
    int32_t* counters;
    int num_partitions;
    int prefix_len;
    int prefix_tiles;
    int prefix_append;
};

template <typename T, int D, int B, int NW, int STAGES>
struct PrefillSmem {
    static constexpr int kTile = B * D * static_cast<int>(sizeof(T));
    static constexpr int kRing = STAGES * 2 * kTile;
    static constexpr int kBars = STAGES * 2 * 8;
    static constexpr int kTotal = kRing + kBars;
};

template <typename T, int D, int B, int NW, int STAGES>
__global__ void __launch_bounds__(NW * 32) pa_prefill_kernel(const __grid_constant__ PrefillParams p) {
    wait_for_prior_work();
    using Smem = PrefillSmem<T, D, B, NW, STAGES>;
    constexpr int kTile = Smem::kTile;
    constexpr int kNt = B / 8;          // 8-token n-tiles per block
    constexpr int kDt = D / 8;          // 8-dim n-tiles of the output
    static_assert(B % 8 == 0 && D % 32 == 0, "tile shapes");
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Smem::kRing);
    uint64_t* empty = full + STAGES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 2, c = lane & 3;
    const int tile = blockIdx.x, kvh = blockIdx.y, s = blockIdx.z;
    const int group = p.group;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], NW);
        }
        fence_barrier_init();
    }

    const int q0 = p.query_start[s];
    const int Q = p.query_start[s + 1] - q0;
    int L = p.context_lens[s];
    if (L < 0 || L > p.context_cap || Q < 0 || Q > L) {
        if (threadIdx.x == 0 && tile == 0 && kvh == 0) flag_error(2 /* PA_DEVERR_CONTEXT_LEN */);
        return;
    }
    const int tok0 = tile * p.tile_tokens;
    if (tok0 >= Q) return;
    const int tok1 = min(Q, tok0 + p.tile_tokens);
    // blocks that the tile's last query can see
    const int last_pos = L - Q + tok1 - 1;
    const int nblk = last_pos / B + 1;
    __syncthreads();  // barrier initialisation visible to every thread

    // ---- this thread's two rows: (token, head) and their query positions
    int row_tok[2], row_head[2], row_pos[2];
    bool row_ok[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int m = warp * 16 + r + 8 * e;
        row_tok[e] = tok0 + m / group;
        row_head[e] = kvh * group + m % group;
        row_ok[e] = row_tok[e] < tok1;
        row_pos[e] = row_ok[e] ? L - Q + row_tok[e] : -1;
    }

    // ---- Q as A fragments: qa[ks] = rows r / r+8, dims 16ks + 2c.. and 16ks + 8 + 2c..
    uint32_t qa[D / 16][4];
    {
        const T* qbase = reinterpret_cast<const T*>(p.q);
        const T* row0 = qbase + (static_cast<long long>(q0 + row_tok[0]) * p.num_q_heads + row_head[0]) * D;
        const T* row1 = qbase + (static_cast<long long>(q0 + row_tok[1]) * p.num_q_heads + row_head[1]) * D;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const int d = 16 * ks + 2 * c;
            qa[ks][0] = row_ok[0] ? *reinterpret_cast<const uint32_t*>(row0 + d) : 0u;
            qa[ks][1] = row_ok[1] ? *reinterpret_cast<const uint32_t*>(row1 + d) : 0u;
            qa[ks][2] = row_ok[0] ? *reinterpret_cast<const uint32_t*>(row0 + d + 8) : 0u;
            qa[ks][3] = row_ok[1] ? *reinterpret_cast<const uint32_t*>(row1 + d + 8) : 0u;
        }
    }

    float o[kDt][4];
#pragma unroll
    for (int dt = 0; dt < kDt; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
    float m_run[2] = {kNegInf, kNegInf}, l_run[2] = {0.f, 0.f};

    // ---- producer (thread 0): one stage per block
    const int32_t* table = p.block_tables + static_cast<long long>(s) * p.max_blocks_per_seq;
    const char* kpool = reinterpret_cast<const char*>(p.k_cache);
    const char* vpool = reinterpret_cast<const char*>(p.v_cache);
    const uint64_t policy = l2_evict_first_policy();
    // bit j of `bad` marks blocks of the current window whose id was refused
    auto issue = [&](int j) -> bool {  // thread 0 only; returns whether the id was valid
        const int st = j % STAGES;
        const int id = __ldg(table + j);
        uint8_t* dst = smem + st * 2 * kTile;
        if (id >= 0 && static_cast<long long>(id) < p.num_blocks) {
            const long long off = (static_cast<long long>(id) * p.num_kv_heads + kvh) * kTile;
            mbar_arrive_expect_tx(&full[st], 2 * kTile);
            bulk_copy_g2s(dst, kpool + off, kTile, &full[st], policy);
            bulk_copy_g2s(dst + kTile, vpool + off, kTile, &full[st], policy);
            return true;
        }
        flag_error(1 /* PA_DEVERR_BLOCK_ID */);
        mbar_arrive(&full[st]);
        return false;
    };
    __shared__ int block_ok[STAGES];
    bool failed = false;
    if (threadIdx.x == 0) {
        for (int j = 0; j < STAGES && j < nblk; ++j) block_ok[j % STAGES] = issue(j);
    }

    const float scale = p.score_scale;
    int j = 0;
    for (; j < nblk; ++j) {
        const int st = j % STAGES;
        const uint32_t phase = (j / STAGES) & 1;
        if (!mbar_wait_bounded(&full[st], phase, kWaitLimitNs)) {
            failed = true;
            break;
        }
        const bool ok = block_ok[st] != 0;
        const uint32_t kbase = smem_u32(smem + st * 2 * kTile);
        const uint32_t vbase = kbase + kTile;
        const int t0 = j * B;

        // S = Q K^T for the block's n-tiles
        float sc[kNt][4];
#pragma unroll
        for (int nt = 0; nt < kNt; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
        const int mi = lane >> 3, row = lane & 7;
#pragma unroll
        for (int kq = 0; kq < D / 32; ++kq) {
#pragma unroll
            for (int nt = 0; nt < kNt; ++nt) {
                uint32_t b0, b1, b2, b3;  // dims chunks 4kq .. 4kq+3 of tokens 8nt..8nt+7
                ldsm_x4(kbase + ((4 * kq + mi) * B + 8 * nt + row) * 16, b0, b1, b2, b3);
                Mma<T>::k16(sc[nt], qa[2 * kq][0], qa[2 * kq][1], qa[2 * kq][2], qa[2 * kq][3], b0, b1);
                Mma<T>::k16(sc[nt], qa[2 * kq + 1][0], qa[2 * kq + 1][1], qa[2 * kq + 1][2], qa[2 * kq + 1][3],
                            b2, b3);
            }
        }

        // causal mask + online softmax (rows r: e = 0, r + 8: e = 1)
        float mx[2] = {kNegInf, kNegInf};
#pragma unroll
        for (int nt = 0; nt < kNt; ++nt) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int e = k >> 1;
                const int t = t0 + 8 * nt + 2 * c + (k & 1);
                const float x = (ok && t <= row_pos[e]) ? sc[nt][k] * scale : kNegInf;
                sc[nt][k] = x;
                mx[e] = fmaxf(mx[e], x);
            }
        }
        float alpha[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 1));
            mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 2));
            const float mn = fmaxf(m_run[e], mx[e]);
            const float mu = mn == kNegInf ? 0.f : mn;
            alpha[e] = exp2_approx(m_run[e] - mu);
            m_run[e] = mn;
            float rs = 0.f;
#pragma unroll
            for (int nt = 0; nt < kNt; ++nt) {
                sc[nt][2 * e] = exp2_approx(sc[nt][2 * e] - mu);
                sc[nt][2 * e + 1] = exp2_approx(sc[nt][2 * e + 1] - mu);
                rs += sc[nt][2 * e] + sc[nt][2 * e + 1];
            }
            l_run[e] = l_run[e] * alpha[e] + rs;
        }
#pragma unroll
        for (int dt = 0; dt < kDt; ++dt) {
            o[dt][0] *= alpha[0];
            o[dt][1] *= alpha[0];
            o[dt][2] *= alpha[1];
            o[dt][3] *= alpha[1];
        }

        // O += P V
        if constexpr (B >= 16) {
#pragma unroll
            for (int kk = 0; kk < B / 16; ++kk) {
                const uint32_t a0 = Mma<T>::pack(sc[2 * kk][0], sc[2 * kk][1]);
                const uint32_t a1 = Mma<T>::pack(sc[2 * kk][2], sc[2 * kk][3]);
                const uint32_t a2 = Mma<T>::pack(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
                const uint32_t a3 = Mma<T>::pack(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
                for (int dp = 0; dp < kDt / 2; ++dp) {
                    uint32_t b0, b1, b2, b3;  // dims chunks 2dp, 2dp+1 x tokens 16kk..+7, +8..+15
                    ldsm_x4_trans(vbase + ((2 * dp + (mi >> 1)) * B + 16 * kk + 8 * (mi & 1) + row) * 16, b0, b1,
                                  b2, b3);
                    Mma<T>::k16(o[2 * dp], a0, a1, a2, a3, b0, b1);
                    Mma<T>::k16(o[2 * dp + 1], a0, a1, a2, a3, b2, b3);
                }
            }
        } else {  // 8-token blocks: m16n8k8
            const uint32_t a0 = Mma<T>::pack(sc[0][0], sc[0][1]);
            const uint32_t a1 = Mma<T>::pack(sc[0][2], sc[0][3]);
#pragma unroll
            for (int dq = 0; dq < kDt / 4; ++dq) {
                uint32_t b0, b1, b2, b3;  // dims chunks 4dq .. 4dq+3 x tokens 0..7
                ldsm_x4_trans(vbase + ((4 * dq + mi) * B + row) * 16, b0, b1, b2, b3);
                Mma<T>::k8(o[4 * dq], a0, a1, b0);
                Mma<T>::k8(o[4 * dq + 1], a0, a1, b1);
                Mma<T>::k8(o[4 * dq + 2], a0, a1, b2);
                Mma<T>::k8(o[4 * dq + 3], a0, a1, b3);
            }
        }

        // release the stage; thread 0 refills it once every warp has
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
        if (threadIdx.x == 0 && j + STAGES < nblk) {
            if (!mbar_wait_bounded(&empty[st], phase, kWaitLimitNs)) {
                failed = true;
            } else {
                block_ok[st] = issue(j + STAGES);
            }
        }
        if (__shfl_sync(0xffffffffu, failed ? 1 : 0, 0)) break;
    }
    if (failed) {
        if (lane == 0) flag_error(8 /* PA_DEVERR_TIMEOUT */);
        // let the copies already issued land before the CTA may exit
        if (threadIdx.x == 0)
            for (int k = j; k < nblk && k < j + STAGES; ++k)
                mbar_wait_bounded(&full[k % STAGES], (k / STAGES) & 1, kWaitLimitNs);
    }
    const int any_failed = __syncthreads_or(failed ? 1 : 0);
    if (any_failed) return;

    // ---- normalise and write the valid rows
    T* out = reinterpret_cast<T*>(p.out);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        float l = l_run[e];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        if (!row_ok[e]) continue;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        T* dst = out + (static_cast<long long>(q0 + row_tok[e]) * p.num_q_heads + row_head[e]) * D;
#pragma unroll
        for (int dt = 0; dt < kDt; ++dt) {
            const int d = 8 * dt + 2 * c;
            dst[d] = from_float<T>(o[dt][2 * e] * inv);
            dst[d + 1] = from_float<T>(o[dt][2 * e + 1] * inv);
        }
    }
}

}  // namespace pa
