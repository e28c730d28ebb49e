// Work-balanced ("stream-K") paged decode for sm_100a.
//
// Same result as the one-pass and split-K kernels (attention of one query
// token per sequence over its paged context, "从源码剖析 vLLM 的显存管理与连续批处理"
// §2.3), scheduled for a continuous batch whose context lengths differ widely
// ("vLLM核心架构总览" §4.2: sequences of every length run in one batch):
//
//  * The work is the flat list of items (sequence s, kv head, logical block
//    j), ordered by pair p = s*Hkv + kvh, then j.  A persistent grid (one wave)
//    of CTAs with NW warps gives every warp ("worker") one equal contiguous
//    range of that list, so every warp streams the same number of KV tiles
//    whatever the length mix, and its copy pipeline never drains between
//    sequences.
//  * A pair lying inside one worker's range is finished there and written
//    normalised.  A pair cut by range boundaries leaves one partial record
//    (unnormalised acc, running max m, sum l) per piece in the workspace; the
//    piece that arrives last (an atomic counter per pair) merges all pieces in
//    worker order with log-sum-exp weights exp(m_k - max m) and resets the
//    counter to zero.  The merge order is fixed, so results are bitwise
//    reproducible and do not depend on which warp merges.
//  * No thread ever waits for another CTA.
#pragma once

#include "pa_warp.cuh"

namespace pa {

// Floats per partial record: [g][D] acc, [g] m, [g] l, padded so that every
// record starts on a 16-byte boundary (records are accessed as float4/float2).
__host__ __device__ constexpr int record_floats(int group, int head_dim) {
    return (group * (head_dim + 2) + 3) / 4 * 4;
}

struct StreamParams {
    void* out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* records;    // [workers][2][record_floats(g, D)] partial records
    int* counters;     // [num_seqs * Hkv] arrival counters, zero between calls
    float score_scale;
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int group;
    int max_blocks_per_seq;
    int context_cap;
    long long num_blocks;
    int workers;       // grid size * NW
};

template <typename T, int D, int B, int NW, int STAGES>
struct StreamSmem {
    static constexpr int kTile = B * D * static_cast<int>(sizeof(T));
    static constexpr int kRing = NW * STAGES * 2 * kTile;
    static constexpr int kBars = (NW * STAGES * 8 + 15) / 16 * 16;
    static constexpr int kQ = IsF32<T>::value ? NW * kMaxGroup * D * 4 : 0;  // per-warp query rows (fp32)
    static constexpr int kFixed = kRing + kBars + kQ;
    // + block-count prefix [S+1] and clamped lengths [S+1]
    static int total(int num_seqs) { return kFixed + ((2 * (num_seqs + 1) * 4 + 15) / 16) * 16; }
};

// Log-sum-exp merge of the partial records of one pair: pieces k0 (its record
// in slot 1: the pair starts in k0's range) and k0+1..k1 (slot 0: their
// ranges start inside the pair), folded in that order with a running maximum:
//   M' = max(M, m_k);  acc = acc e^(M-M') + a_k e^(m_k-M');  den likewise with l_k.
// Each lane owns whole 16-byte slices of the [g][D] output, so a piece costs one
// batch of independent loads.
template <typename T, int D, bool LOG2>
__device__ __forceinline__ void merge_records(const float* records, int k0, int k1, int group, T* rows, int lane) {
    constexpr int kVecPerHead = D / 4;                      // float4 slices per head row
    constexpr int kSlots = kMaxGroup * kVecPerHead / 32;    // slices per lane at g = 8
    const int R = record_floats(group, D);
    const int np = k1 - k0 + 1;
    float4 acc[kSlots];
    float M[kSlots], den[kSlots];
#pragma unroll
    for (int i = 0; i < kSlots; ++i) {
        acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        M[i] = kNegInf;
        den[i] = 0.f;
    }
#pragma unroll 2
    for (int q = 0; q < np; ++q) {
        const float* rq = records + (static_cast<long long>(k0 + q) * 2 + (q == 0 ? 1 : 0)) * R;
#pragma unroll
        for (int i = 0; i < kSlots; ++i) {
            const int v = lane + 32 * i;
            const int h = v / kVecPerHead;
            if (h < group) {
                const float m = __ldcg(rq + group * D + h);
                const float l = __ldcg(rq + group * D + group + h);
                const float4 x = __ldcg(reinterpret_cast<const float4*>(rq) + v);
                const float mn = fmaxf(M[i], m);
                if (mn != kNegInf) {
                    const float sa = softmax_exp<LOG2>(M[i] - mn), sb = softmax_exp<LOG2>(m - mn);
                    acc[i].x = fmaf(acc[i].x, sa, x.x * sb);
                    acc[i].y = fmaf(acc[i].y, sa, x.y * sb);
                    acc[i].z = fmaf(acc[i].z, sa, x.z * sb);
                    acc[i].w = fmaf(acc[i].w, sa, x.w * sb);
                    den[i] = fmaf(den[i], sa, l * sb);
                    M[i] = mn;
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kSlots; ++i) {
        const int v = lane + 32 * i;
        if (v / kVecPerHead < group) {
            const float inv = den[i] > 0.f ? 1.f / den[i] : 0.f;
            T* dst = rows + 4 * v;
            dst[0] = from_float<T>(acc[i].x * inv);
            dst[1] = from_float<T>(acc[i].y * inv);
            dst[2] = from_float<T>(acc[i].z * inv);
            dst[3] = from_float<T>(acc[i].w * inv);
        }
    }
}

template <typename T, int D, int B, int NW, int STAGES>
__global__ void __launch_bounds__(NW * 32) pa_decode_streamk_kernel(const __grid_constant__ StreamParams p) {
    using Smem = StreamSmem<T, D, B, NW, STAGES>;
    constexpr bool kF32 = IsF32<T>::value;
    constexpr int kTile = Smem::kTile;
    constexpr int kThreads = NW * 32;
    static_assert(STAGES >= 1 && STAGES <= 32, "ring depth");

    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int warp_total[NW];
    const int S = p.num_seqs, Hkv = p.num_kv_heads, Hq = p.num_q_heads, G = p.group;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* wring = smem + warp * STAGES * 2 * kTile;
    uint64_t* wbar = reinterpret_cast<uint64_t*>(smem + Smem::kRing) + warp * STAGES;
    float* qslot = reinterpret_cast<float*>(smem + Smem::kRing + Smem::kBars) + warp * kMaxGroup * D;
    int* pref = reinterpret_cast<int*>(smem + Smem::kFixed);
    int* lens = pref + (S + 1);

    // ---- clamped lengths and the exclusive prefix of block counts over sequences
    {
        const int per = (S + kThreads - 1) / kThreads;
        const int s0 = min(S, threadIdx.x * per), s1 = min(S, s0 + per);
        int sum = 0;
        for (int s = s0; s < s1; ++s) {
            int L = p.context_lens[s];
            if (L < 0 || L > p.context_cap) {
                if (blockIdx.x == 0) flag_error(2 /* PA_DEVERR_CONTEXT_LEN */);
                L = L < 0 ? 0 : p.context_cap;
            }
            lens[s] = L;
            sum += (L + B - 1) / B;
        }
        int incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        if (lane == 31) warp_total[warp] = incl;
        __syncthreads();
        int run = 0;
        for (int w = 0; w < warp; ++w) run += warp_total[w];
        if (threadIdx.x == kThreads - 1) pref[S] = run + incl;
        run += incl - sum;
        for (int s = s0; s < s1; ++s) {
            pref[s] = run;
            run += (lens[s] + B - 1) / B;
        }
        __syncthreads();
    }

    // ---- sequences without tokens get an all-zero output
    for (int s = blockIdx.x; s < S; s += gridDim.x) {
        if (lens[s] == 0) {
            T* rows = reinterpret_cast<T*>(p.out) + static_cast<long long>(s) * Hq * D;
            for (int i = threadIdx.x; i < Hq * D; i += kThreads) rows[i] = from_float<T>(0.f);
        }
    }

    const long long total = static_cast<long long>(Hkv) * pref[S];
    const long long W = total < p.workers ? total : p.workers;
    const long long k = static_cast<long long>(blockIdx.x) * NW + warp;
    if (k >= W) return;  // this warp has no range (no CTA-wide barrier follows)
    const long long i0 = k * total / W, i1 = (k + 1) * total / W;
    const int cnt = static_cast<int>(i1 - i0);
    auto worker_of = [&](long long item) -> int { return static_cast<int>(((item + 1) * W - 1) / total); };

    if (lane == 0) {
        for (int i = 0; i < STAGES; ++i) mbar_init(&wbar[i], 1);
        fence_barrier_init();
    }
    __syncwarp();

    // Item i -> (physical block id, pair, logical block j); id -1 = nothing to read.
    auto item_info = [&](long long i, int& id, int& pair, int& j) {
        id = -1;
        pair = -1;
        j = 0;
        if (i >= i1) return;
        int lo = 0, hi = S - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (static_cast<long long>(Hkv) * pref[mid] <= i) lo = mid; else hi = mid - 1;
        }
        const int s = lo;
        const int nb = pref[s + 1] - pref[s];
        const int rem = static_cast<int>(i - static_cast<long long>(Hkv) * pref[s]);
        const int kvh = rem / nb;
        j = rem - kvh * nb;
        pair = s * Hkv + kvh;
        const int blk = __ldg(p.block_tables + static_cast<long long>(s) * p.max_blocks_per_seq + j);
        if (blk < 0 || static_cast<long long>(blk) >= p.num_blocks) {
            flag_error(1 /* PA_DEVERR_BLOCK_ID */);
        } else {
            id = blk;
        }
    };
    int wid0, wpair0, wj0, wid1 = -1, wpair1 = -1, wj1 = 0;
    item_info(i0 + lane, wid0, wpair0, wj0);
    if (cnt > 32) item_info(i0 + 32 + lane, wid1, wpair1, wj1);
    int cur_round = 0;
    auto get = [&](int n, int& id, int& pair, int& j) {  // warp-uniform n
        const bool in0 = (n >> 5) == cur_round;
        id = __shfl_sync(0xffffffffu, in0 ? wid0 : wid1, n & 31);
        pair = __shfl_sync(0xffffffffu, in0 ? wpair0 : wpair1, n & 31);
        j = __shfl_sync(0xffffffffu, in0 ? wj0 : wj1, n & 31);
    };

    const uint64_t policy = l2_evict_first_policy();
    const char* kpool = reinterpret_cast<const char*>(p.k_cache);
    const char* vpool = reinterpret_cast<const char*>(p.v_cache);
    auto issue = [&](int n) {
        int id, pair, j;
        get(n, id, pair, j);
        if (lane == 0) {
            const int st = n % STAGES;
            uint8_t* dst = wring + st * 2 * kTile;
            if (id >= 0) {
                const int kvh = pair % Hkv;
                const long long off = (static_cast<long long>(id) * Hkv + kvh) * kTile;
                mbar_arrive_expect_tx(&wbar[st], 2 * kTile);
                bulk_copy_g2s(dst, kpool + off, kTile, &wbar[st], policy);
                bulk_copy_g2s(dst + kTile, vpool + off, kTile, &wbar[st], policy);
            } else {
                mbar_arrive(&wbar[st]);
            }
        }
    };

    typename WarpState<T, D, B>::type acc;
    acc.reset();
    const T* qbase = reinterpret_cast<const T*>(p.q);
    T* obase = reinterpret_cast<T*>(p.out);
    const int R = record_floats(G, D);
    auto q_rows = [&](int pair) {
        const int s = pair / Hkv, kvh = pair - s * Hkv;
        return qbase + (static_cast<long long>(s) * Hq + kvh * G) * D;
    };

    // Emits the state of `pair` (first/last logical block this worker saw).
    auto finalize = [&](int pair, int first_j, int last_j) {
        const int s = pair / Hkv, kvh = pair - s * Hkv;
        const int nb = pref[s + 1] - pref[s];
        T* rows = obase + (static_cast<long long>(s) * Hq + kvh * G) * D;
        const bool first = first_j == 0, last = last_j == nb - 1;
        if (first && last) {
            acc.write_out(rows, G, lane);
        } else {
            float* rec = p.records + (k * 2 + (first ? 1 : 0)) * R;
            acc.write_record(rec, G, lane);
            __threadfence();
            __syncwarp();
            int old = 0;
            if (lane == 0) old = atomicAdd(p.counters + pair, 1);
            old = __shfl_sync(0xffffffffu, old, 0);
            const long long start = static_cast<long long>(Hkv) * pref[s] + static_cast<long long>(kvh) * nb;
            const int k0 = worker_of(start), k1 = worker_of(start + nb - 1);
            if (old == k1 - k0) {  // every other piece is already recorded
                __threadfence();
                merge_records<T, D, !kF32>(p.records, k0, k1, G, rows, lane);
                if (lane == 0) p.counters[pair] = 0;  // ready for the next call
            }
        }
        acc.reset();
    };

    const int issued0 = cnt < STAGES ? cnt : STAGES;
    for (int n = 0; n < issued0; ++n) issue(n);
    int issued = issued0;
    int cur_pair = -1, first_j = 0, last_j = 0, prefetched = -1;
    bool failed = false;
    int n = 0;
    for (; n < cnt; ++n) {
        if (n > 0 && (n & 31) == 0) {
            wid0 = wid1;
            wpair0 = wpair1;
            wj0 = wj1;
            ++cur_round;
            item_info(i0 + static_cast<long long>(cur_round + 1) * 32 + lane, wid1, wpair1, wj1);
        }
        const int st = n % STAGES;
        if (!mbar_wait_bounded(&wbar[st], (n / STAGES) & 1, kWaitLimitNs)) {
            failed = true;
            break;
        }
        int id, pair, j;
        get(n, id, pair, j);
        if (pair != cur_pair) {
            if (cur_pair >= 0) finalize(cur_pair, first_j, last_j);
            cur_pair = pair;
            first_j = j;
            if constexpr (kF32) {
                acc.load_q(qslot, q_rows(pair), G, lane);
            } else {
                if (prefetched == pair) {
                    acc.use_prefetched_q();
                } else {
                    acc.load_q(q_rows(pair), G, lane);
                }
                if (pair + 1 < S * Hkv) {
                    acc.prefetch_q(q_rows(pair + 1), G, lane);
                    prefetched = pair + 1;
                }
            }
        }
        last_j = j;
        const int valid = id < 0 ? 0 : min(B, lens[pair / Hkv] - j * B);
        uint8_t* stage = wring + st * 2 * kTile;
        if constexpr (kF32) {
            acc.block(reinterpret_cast<const float*>(stage), reinterpret_cast<const float*>(stage + kTile), valid, G,
                      p.score_scale, lane);
        } else {
            acc.block(smem_u32(stage), smem_u32(stage + kTile), valid, G, p.score_scale, lane);
        }
        __syncwarp();
        if (n + STAGES < cnt) {
            issue(n + STAGES);
            ++issued;
        }
    }
    if (failed) {
        if (lane == 0) flag_error(8 /* PA_DEVERR_TIMEOUT */);
        for (int m = n; m < issued; ++m) mbar_wait_bounded(&wbar[m % STAGES], (m / STAGES) & 1, kWaitLimitNs);
        return;
    }
    if (cur_pair >= 0) finalize(cur_pair, first_j, last_j);
}

}  // namespace pa
