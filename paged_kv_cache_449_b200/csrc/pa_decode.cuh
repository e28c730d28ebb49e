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

#include "pa_device.cuh"

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
};

constexpr int kMaxGroup = 8;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait, far above any copy time

template <typename T>
struct IsF32 {
    static constexpr bool value = false;
};
template <>
struct IsF32<float> {
    static constexpr bool value = true;
};

template <typename T, int D, int B, int NW, int STAGES>
struct DecodeSmem {
    static constexpr int kElem = sizeof(T);
    static constexpr int kTile = B * D * kElem;                 // one (block, head) tile, bytes
    static constexpr int kRing = NW * STAGES * 2 * kTile;       // K and V slots of all warps
    static constexpr int kMerge = NW * kMaxGroup * (D + 2) * 4;  // warp states for the CTA merge
    static constexpr int kArea = kRing > kMerge ? kRing : kMerge;
    static constexpr int kBars = (NW * STAGES * 8 + 15) / 16 * 16;  // keeps what follows 16-byte aligned
    static constexpr int kQ = IsF32<T>::value ? kMaxGroup * D * 4 : 0;
    static constexpr int kTotal = kArea + kBars + kQ;
};

// ----------------------------------------------------------------------------
// Per-warp accumulator state and block computation, 16-bit inputs (tensor cores)

template <typename T, int D, int B>
struct WarpMma {
    static constexpr int kNt = B / 8;  // 8-token n-tiles per block
    float o[D / 8][4];                 // out^ rows (r, r+8) x d-tile
    uint32_t qa[D / 16][2];            // Q A-fragments: row r, k = 2c.., 8+2c..
    float m_run = kNegInf;             // row r, score domain (base 2)
    float l_run = 0.f;                 // this thread's share of row r's sum

    __device__ __forceinline__ void init(const T* q_rows, int group, int lane) {
        const int r = lane >> 2, c = lane & 3;
#pragma unroll
        for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            if (r < group) {
                const T* row = q_rows + r * D + ks * 16 + 2 * c;
                qa[ks][0] = *reinterpret_cast<const uint32_t*>(row);
                qa[ks][1] = *reinterpret_cast<const uint32_t*>(row + 8);
            } else {
                qa[ks][0] = qa[ks][1] = 0u;
            }
        }
    }

    // Zero the 16-bit halves of a V fragment register that belong to tokens
    // >= valid (token `tok` in the low half, tok+1 in the high half).
    static __device__ __forceinline__ uint32_t mask_pair(uint32_t v, int tok, int valid) {
        const uint32_t keep = (tok < valid ? 0x0000ffffu : 0u) | (tok + 1 < valid ? 0xffff0000u : 0u);
        return v & keep;
    }

    __device__ __forceinline__ void block(uint32_t kbase, uint32_t vbase, int valid, int group, float scale_log2,
                                          int lane) {
        const int r = lane >> 2, c = lane & 3;
        const int mtx = lane >> 3, row = lane & 7;
        float sc[kNt][4];
#pragma unroll
        for (int nt = 0; nt < kNt; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;

        // S = Q K^T: M = query rows, N = tokens, K = head dim.
        if constexpr (B >= 16) {
#pragma unroll
            for (int np = 0; np < kNt / 2; ++np) {
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const int tok = np * 16 + (mtx >> 1) * 8 + row;
                    const int chunk = 2 * ks + (mtx & 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kbase + (chunk * B + tok) * 16, b0, b1, b2, b3);
                    Mma<T>::k16(sc[2 * np], qa[ks][0], 0u, qa[ks][1], 0u, b0, b1);
                    Mma<T>::k16(sc[2 * np + 1], qa[ks][0], 0u, qa[ks][1], 0u, b2, b3);
                }
            }
        } else {
#pragma unroll
            for (int kq = 0; kq < D / 32; ++kq) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kbase + ((4 * kq + mtx) * 8 + row) * 16, b0, b1, b2, b3);
                Mma<T>::k16(sc[0], qa[2 * kq][0], 0u, qa[2 * kq][1], 0u, b0, b1);
                Mma<T>::k16(sc[0], qa[2 * kq + 1][0], 0u, qa[2 * kq + 1][1], 0u, b2, b3);
            }
        }

        // Online softmax on row r (rows r+8 are padding and stay zero).
        const bool row_ok = r < group;
        float mx = kNegInf;
#pragma unroll
        for (int nt = 0; nt < kNt; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int tok = nt * 8 + 2 * c + e;
                const float x = (row_ok && tok < valid) ? sc[nt][e] * scale_log2 : kNegInf;
                sc[nt][e] = x;
                mx = fmaxf(mx, x);
            }
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(m_run, mx);
        const float m_use = (m_new == kNegInf) ? 0.f : m_new;
        const float alpha = exp2_approx(m_run - m_use);
        float rs = 0.f;
#pragma unroll
        for (int nt = 0; nt < kNt; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float pv = exp2_approx(sc[nt][e] - m_use);
                sc[nt][e] = pv;
                rs += pv;
            }
        }
        l_run = l_run * alpha + rs;
        m_run = m_new;
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
            o[j][0] *= alpha;
            o[j][1] *= alpha;
        }

        // O += P V: M = query rows, N = head dim, K = tokens.
        const bool partial = valid < B;
        if constexpr (B >= 16) {
#pragma unroll
            for (int kp = 0; kp < kNt / 2; ++kp) {
                const uint32_t a0 = Mma<T>::pack(sc[2 * kp][0], sc[2 * kp][1]);
                const uint32_t a2 = Mma<T>::pack(sc[2 * kp + 1][0], sc[2 * kp + 1][1]);
                const int tlo = kp * 16 + 2 * c, thi = kp * 16 + 8 + 2 * c;
#pragma unroll
                for (int dj = 0; dj < D / 16; ++dj) {
                    const int tok = kp * 16 + (mtx & 1) * 8 + row;
                    const int chunk = 2 * dj + (mtx >> 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_trans(vbase + (chunk * B + tok) * 16, b0, b1, b2, b3);
                    if (partial) {
                        b0 = mask_pair(b0, tlo, valid);
                        b1 = mask_pair(b1, thi, valid);
                        b2 = mask_pair(b2, tlo, valid);
                        b3 = mask_pair(b3, thi, valid);
                    }
                    Mma<T>::k16(o[2 * dj], a0, 0u, a2, 0u, b0, b1);
                    Mma<T>::k16(o[2 * dj + 1], a0, 0u, a2, 0u, b2, b3);
                }
            }
        } else {
            const uint32_t a0 = Mma<T>::pack(sc[0][0], sc[0][1]);
#pragma unroll
            for (int dq = 0; dq < D / 32; ++dq) {
                uint32_t b[4];
                ldsm_x4_trans(vbase + ((4 * dq + mtx) * 8 + row) * 16, b[0], b[1], b[2], b[3]);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    if (partial) b[m] = mask_pair(b[m], 2 * c, valid);
                    Mma<T>::k8(o[4 * dq + m], a0, 0u, b[m]);
                }
            }
        }
    }

    // Writes this warp's (m, l, o) for its valid rows into the merge area.
    __device__ __forceinline__ void store(float* mo, float* mml, int warp, int group, int lane) {
        const int r = lane >> 2, c = lane & 3;
        float l = l_run;
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        if (r < group) {
            float* dst = mo + (warp * kMaxGroup + r) * D;
#pragma unroll
            for (int j = 0; j < D / 8; ++j) {
                dst[8 * j + 2 * c] = o[j][0];
                dst[8 * j + 2 * c + 1] = o[j][1];
            }
            if (c == 0) {
                mml[(warp * kMaxGroup + r) * 2] = m_run;
                mml[(warp * kMaxGroup + r) * 2 + 1] = l;
            }
        }
    }
};

// ----------------------------------------------------------------------------
// fp32 inputs (CUDA cores)

template <int D, int B>
struct WarpF32 {
    static constexpr int kC = D / 4;          // 16-byte vectors per token row
    static constexpr int kTg = 32 / B;        // lanes sharing one token in QK^T
    static constexpr int kCpp = kC / kTg;     // vectors per lane in QK^T
    static constexpr int kGrp = 32 / kC;      // token groups in PV (1 for D=128, 2 for D=64)
    float o[kMaxGroup][4];
    float m_run[kMaxGroup];
    float l_run[kMaxGroup];

    __device__ __forceinline__ void init() {
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            o[h][0] = o[h][1] = o[h][2] = o[h][3] = 0.f;
            m_run[h] = kNegInf;
            l_run[h] = 0.f;
        }
    }

    __device__ __forceinline__ void block(const float* ktile, const float* vtile, const float* qs, int valid,
                                          int group, float scale, int lane) {
        const int t = lane % B, part = lane / B;
        float s[kMaxGroup];
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) s[h] = 0.f;
#pragma unroll 4
        for (int cc = 0; cc < kCpp; ++cc) {
            const int chunk = part * kCpp + cc;
            const float4 kv = *reinterpret_cast<const float4*>(ktile + (chunk * B + t) * 4);
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h) {
                if (h < group) {
                    const float4 qv = *reinterpret_cast<const float4*>(qs + h * D + chunk * 4);
                    s[h] = fmaf(qv.x, kv.x, s[h]);
                    s[h] = fmaf(qv.y, kv.y, s[h]);
                    s[h] = fmaf(qv.z, kv.z, s[h]);
                    s[h] = fmaf(qv.w, kv.w, s[h]);
                }
            }
        }
        float p[kMaxGroup];
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            if (h >= group) {
                p[h] = 0.f;
                continue;
            }
#pragma unroll
            for (int off = B; off < 32; off <<= 1) s[h] += __shfl_xor_sync(0xffffffffu, s[h], off);
            const float x = (t < valid) ? s[h] * scale : kNegInf;
            float mx = x;
#pragma unroll
            for (int off = 1; off < B; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float m_new = fmaxf(m_run[h], mx);
            const float m_use = (m_new == kNegInf) ? 0.f : m_new;
            const float alpha = expf(m_run[h] - m_use);
            const float pv = expf(x - m_use);
            float sum = (part == 0) ? pv : 0.f;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            l_run[h] = l_run[h] * alpha + sum;
            m_run[h] = m_new;
            o[h][0] *= alpha;
            o[h][1] *= alpha;
            o[h][2] *= alpha;
            o[h][3] *= alpha;
            p[h] = pv;
        }
        // PV: lane owns vector cj of D for the tokens of group tg.
        const int cj = lane % kC, tg = lane / kC;
        constexpr int kPer = B / kGrp;
#pragma unroll 4
        for (int ii = 0; ii < kPer; ++ii) {
            const int tt = ((ii + cj) % kPer) * kGrp + tg;  // rotated so a quarter-warp hits 8 banks
            float4 vv = *reinterpret_cast<const float4*>(vtile + (cj * B + tt) * 4);
            if (tt >= valid) vv = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h) {
                const float ph = __shfl_sync(0xffffffffu, p[h], tt);
                if (h < group) {
                    o[h][0] = fmaf(ph, vv.x, o[h][0]);
                    o[h][1] = fmaf(ph, vv.y, o[h][1]);
                    o[h][2] = fmaf(ph, vv.z, o[h][2]);
                    o[h][3] = fmaf(ph, vv.w, o[h][3]);
                }
            }
        }
    }

    __device__ __forceinline__ void store(float* mo, float* mml, int warp, int group, int lane) {
        const int cj = lane % kC, tg = lane / kC;
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            if constexpr (kGrp == 2) {
#pragma unroll
                for (int e = 0; e < 4; ++e) o[h][e] += __shfl_xor_sync(0xffffffffu, o[h][e], 16);
            }
            if (h < group && tg == 0) {
                float* dst = mo + (warp * kMaxGroup + h) * D + cj * 4;
                dst[0] = o[h][0];
                dst[1] = o[h][1];
                dst[2] = o[h][2];
                dst[3] = o[h][3];
            }
            if (h < group && lane == 0) {
                mml[(warp * kMaxGroup + h) * 2] = m_run[h];
                mml[(warp * kMaxGroup + h) * 2 + 1] = l_run[h];
            }
        }
    }
};

template <typename T, int D, int B>
struct WarpState {
    using type = WarpMma<T, D, B>;
};
template <int D, int B>
struct WarpState<float, D, B> {
    using type = WarpF32<D, B>;
};

// ----------------------------------------------------------------------------
// The decode kernel (SPLIT = false: one pass per (seq, kv head); true: one
// partition of partition_blocks blocks per CTA, partials to the workspace).

template <typename T, int D, int B, int NW, int STAGES, bool SPLIT>
__global__ void __launch_bounds__(NW * 32) pa_decode_kernel(const __grid_constant__ DecodeParams p) {
    using Smem = DecodeSmem<T, D, B, NW, STAGES>;
    constexpr bool kF32 = IsF32<T>::value;
    constexpr int kTile = Smem::kTile;
    static_assert(STAGES >= 1 && STAGES <= 32, "ring depth");
    static_assert((kTile % 16) == 0, "bulk copies move multiples of 16 bytes");

    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* ring = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Smem::kArea);
    float* qs = reinterpret_cast<float*>(smem + Smem::kArea + Smem::kBars);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int part = blockIdx.x, kvh = blockIdx.y, s = blockIdx.z;
    const int group = p.group;

    int L = p.context_lens[s];
    if (L < 0 || L > p.context_cap) {
        if (threadIdx.x == 0 && part == 0 && kvh == 0) flag_error(2 /* PA_DEVERR_CONTEXT_LEN */);
        L = L < 0 ? 0 : p.context_cap;
    }
    const int nblk = (L + B - 1) / B;
    int b0 = 0, b1 = nblk;
    if constexpr (SPLIT) {
        b0 = part * p.partition_blocks;
        if (b0 >= nblk) return;  // this partition is past the end of the sequence
        b1 = min(nblk, b0 + p.partition_blocks);
    }
    const T* qrows = reinterpret_cast<const T*>(p.q) +
                     (static_cast<long long>(s) * p.num_q_heads + kvh * group) * D;
    if constexpr (!SPLIT) {
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
    uint64_t* wbar = bars + warp * STAGES;
    uint8_t* wring = ring + warp * STAGES * 2 * kTile;
    if (lane == 0) {
        for (int i = 0; i < STAGES; ++i) mbar_init(&wbar[i], 1);
        fence_barrier_init();
    }
    __syncwarp();

    const int32_t* bt = p.block_tables + static_cast<long long>(s) * p.max_blocks_per_seq + b0 + warp;
    auto load_ids = [&](int round) -> int {
        const int i = round * 32 + lane;
        int id = -1;
        if (i < n_w) {
            id = __ldg(bt + i * NW);
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

    typename WarpState<T, D, B>::type acc;
    if constexpr (kF32) {
        acc.init();
    } else {
        acc.init(qrows, group, lane);
    }

    int issued = n_w < STAGES ? n_w : STAGES;
    for (int i = 0; i < issued; ++i) issue(i);
    bool failed = false;
    int i = 0;
    for (; i < n_w; ++i) {
        if (i > 0 && (i & 31) == 0) {
            win0 = win1;
            ++cur_round;
            win1 = load_ids(cur_round + 1);
        }
        const int st = i % STAGES;
        if (!mbar_wait_bounded(&wbar[st], (i / STAGES) & 1, kWaitLimitNs)) {
            failed = true;
            break;
        }
        const int id = block_id(i);
        const int j = b0 + warp + i * NW;  // logical block index
        const int valid = id < 0 ? 0 : min(B, L - j * B);
        uint8_t* stage = wring + st * 2 * kTile;
        if constexpr (kF32) {
            acc.block(reinterpret_cast<const float*>(stage), reinterpret_cast<const float*>(stage + kTile), qs,
                      valid, group, p.score_scale, lane);
        } else {
            acc.block(smem_u32(stage), smem_u32(stage + kTile), valid, group, p.score_scale, lane);
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
        for (int k = i; k < issued; ++k) mbar_wait_bounded(&wbar[k % STAGES], (k / STAGES) & 1, kWaitLimitNs);
    }
    const int any_failed = __syncthreads_or(failed ? 1 : 0);
    if (any_failed) return;

    // ---- merge the warps' states (the ring is free now)
    float* mo = reinterpret_cast<float*>(smem);
    float* mml = mo + NW * kMaxGroup * D;
    acc.store(mo, mml, warp, group, lane);
    __syncthreads();

    constexpr bool kLog2 = !kF32;
    for (int idx = threadIdx.x; idx < group * D; idx += NW * 32) {
        const int r = idx / D, d = idx - r * D;
        float M = kNegInf;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, mml[(w * kMaxGroup + r) * 2]);
        float num = 0.f, den = 0.f;
        if (M != kNegInf) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float wt = softmax_exp<kLog2>(mml[(w * kMaxGroup + r) * 2] - M);
                num = fmaf(wt, mo[(w * kMaxGroup + r) * D + d], num);
                den = fmaf(wt, mml[(w * kMaxGroup + r) * 2 + 1], den);
            }
        }
        const int h = kvh * group + r;
        if constexpr (SPLIT) {
            const long long slot = (static_cast<long long>(s) * p.num_q_heads + h) * p.num_partitions + part;
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
