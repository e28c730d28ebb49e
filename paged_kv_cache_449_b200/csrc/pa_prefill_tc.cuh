// Chunked prefill on the 5th-generation tensor cores (tcgen05): the same
// computation as pa_prefill_kernel ("vLLM核心架构总览" §4.3 chunked prefill,
// causal attention of each sequence's newest Q tokens over its paged context).
//
//  * One CTA of 128 threads per (sequence, kv head, tile of 128 / g query
//    tokens).  The 128 MMA rows are (query token, head of the GQA group)
//    pairs; thread t owns row t, which is TMEM lane t.
//  * Tiles of 128 keys (8 blocks of 16 tokens, or 4 of 32) arrive by bulk
//    copies into a 2-stage ring.  The paged (block, head) tile layout
//    [D/8][B][8] is used as the MMA operand directly: K-major B operand of
//    S = Q K^T (8-token groups 128 bytes apart, the next 8 dims B*16 bytes
//    apart) and MN-major B operand of O += P V (the same numbers with the
//    roles of the two offsets exchanged); no copy into another layout.
//  * S (128 x 128 fp32) and O (128 x D fp32) live in tensor memory.  One
//    thread issues every MMA; tcgen05.commit arrives on mbarriers that the
//    other threads wait on (bounded).  Each thread reads its S row with
//    tcgen05.ld, masks (causal, past the context), runs the online softmax in
//    base 2, writes its P row (16-bit) into shared memory in the MMA core
//    matrix layout and rescales its O row in tensor memory before the next
//    O += P V.
//  * Tokens past the context in the tile's last block are zeroed in the
//    staged V tile (P is 0 there, but 0 times a stale non-finite value would
//    not be); blocks beyond the context or with a refused id get no MMA.
//  * Tensor memory is allocated after every early exit and released on every
//    path.
#pragma once

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

}  // namespace tc

#ifndef PA_PREFILL_TC_KEYS
#define PA_PREFILL_TC_KEYS 64
#endif

template <typename T, int D, int B>
struct PrefillTcSmem {
    static constexpr int kKeys = PA_PREFILL_TC_KEYS;      // keys per tile
    static constexpr int kBlocks = kKeys / B;             // blocks per tile
    static constexpr int kTile = B * D * 2;               // one (block, head) K or V tile
    static constexpr int kStage = kBlocks * 2 * kTile;    // K and V of a key tile
    static constexpr int kStages = 2;
    static constexpr int kQ = 128 * D * 2;
    static constexpr int kP = 128 * kKeys * 2;
    static constexpr int kRingOff = 0;
    static constexpr int kQOff = kStages * kStage;
    static constexpr int kPOff = kQOff + kQ;
    static constexpr int kBarOff = kPOff + kP;
    static constexpr int kTotal = kBarOff + 8 * 8 + 16;
};

template <typename T, int D, int B>
__global__ void __launch_bounds__(128) pa_prefill_tc_kernel(const __grid_constant__ PrefillParams p) {
    using Sm = PrefillTcSmem<T, D, B>;
    constexpr int kKeys = Sm::kKeys, kBlocks = Sm::kBlocks, kTile = Sm::kTile;
    // S: kKeys columns, then O: D columns (allocations are powers of two)
    constexpr uint32_t kTmemCols = kKeys + D <= 128 ? 128 : (kKeys + D <= 256 ? 256 : 512);
    static_assert(B == 16 || B == 32, "16- or 32-token blocks");
    static_assert(D == 64 || D == 128, "head dims");
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Sm::kBarOff);   // [2]
    uint64_t* empty = full + 2;                                         // [2]
    uint64_t* s_done = full + 4;
    uint64_t* o_done = full + 5;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(full + 8);
    uint8_t* qs = smem + Sm::kQOff;
    uint8_t* ps = smem + Sm::kPOff;

    const int tid = threadIdx.x, warp = tid >> 5;
    const int tile = blockIdx.x, kvh = blockIdx.y, s = blockIdx.z;
    const int group = p.group;

    const int q0 = p.query_start[s];
    const int Q = p.query_start[s + 1] - q0;
    const int L = p.context_lens[s];
    if (L < 0 || L > p.context_cap || Q < 0 || Q > L) {
        if (tid == 0 && tile == 0 && kvh == 0) flag_error(2 /* PA_DEVERR_CONTEXT_LEN */);
        return;
    }
    const int tok0 = tile * p.tile_tokens;
    if (tok0 >= Q) return;
    const int tok1 = min(Q, tok0 + p.tile_tokens);
    const int last_pos = L - Q + tok1 - 1;
    const int nblk = last_pos / B + 1;                   // blocks the tile needs
    const int ntiles = (nblk + kBlocks - 1) / kBlocks;  // key tiles

    // ---- this thread's row
    const int row_tok = tok0 + tid / group;
    const int row_head = kvh * group + tid % group;
    const bool row_ok = row_tok < tok1;
    const int row_pos = row_ok ? L - Q + row_tok : -1;

    // ---- Q row into the K-major core-matrix layout: (8-row group g, 8-dim chunk c) at c*2048 + g*128
    {
        const T* qrow = reinterpret_cast<const T*>(p.q) +
                        (static_cast<long long>(q0 + (row_ok ? row_tok : tok0)) * p.num_q_heads + row_head) * D;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
            const uint4 v = row_ok ? *reinterpret_cast<const uint4*>(qrow + 8 * c) : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(qs + c * 2048 + (tid >> 3) * 128 + (tid & 7) * 16) = v;
        }
    }
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(s_done, 1);
        mbar_init(o_done, 1);
        fence_barrier_init();
    }
    fence_proxy_async_smem();  // Q (generic stores) visible to the tensor cores
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t s_tmem = tmem;            // columns 0 .. kKeys-1
    const uint32_t o_tmem = tmem + kKeys;    // columns kKeys .. kKeys+D-1
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    {   // O starts at zero, so every O += P V accumulates
        float z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) tc::st32(o_tmem + lane_base + c0, z);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }

    // ---- producer: key tile j (its blocks) into stage j % 2
    const int32_t* table = p.block_tables + static_cast<long long>(s) * p.max_blocks_per_seq;
    const char* kpool = reinterpret_cast<const char*>(p.k_cache);
    const char* vpool = reinterpret_cast<const char*>(p.v_cache);
    const uint64_t policy = l2_evict_first_policy();
    __shared__ uint32_t blk_ok[2];  // bit b: block b of the staged tile was fetched
    auto issue = [&](int j) {       // thread 0
        const int st = j & 1;
        uint8_t* base = smem + st * Sm::kStage;
        uint32_t ok = 0;
        int bytes = 0;
        for (int b = 0; b < kBlocks; ++b) {
            const int jb = j * kBlocks + b;
            if (jb >= nblk) break;
            const int id = __ldg(table + jb);
            if (id >= 0 && static_cast<long long>(id) < p.num_blocks) {
                ok |= 1u << b;
                bytes += 2 * kTile;
            } else {
                flag_error(1 /* PA_DEVERR_BLOCK_ID */);
            }
        }
        blk_ok[st] = ok;
        mbar_arrive_expect_tx(&full[st], bytes);
        for (int b = 0; b < kBlocks; ++b) {
            if (!(ok >> b & 1u)) continue;
            const int id = __ldg(table + j * kBlocks + b);
            const long long off = (static_cast<long long>(id) * p.num_kv_heads + kvh) * kTile;
            bulk_copy_g2s(base + b * kTile, kpool + off, kTile, &full[st], policy);
            bulk_copy_g2s(base + (kBlocks + b) * kTile, vpool + off, kTile, &full[st], policy);
        }
    };
    if (tid == 0) {
        issue(0);
        if (ntiles > 1) issue(1);
    }

    const float scale = p.score_scale;
    float m_run = kNegInf, l_run = 0.f;
    bool failed = false;
    int j = 0;
    for (; j < ntiles; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait_bounded(&full[st], ph, kWaitLimitNs)) failed = true;
        if (__syncthreads_or(failed ? 1 : 0)) {
            failed = true;
            break;
        }
        const uint32_t ok = blk_ok[st];
        uint8_t* kbase = smem + st * Sm::kStage;
        uint8_t* vbase = kbase + kBlocks * kTile;
        const int key0 = j * kKeys;

        // zero V rows of tokens at or past the context in the tile's last needed block
        {
            const int lb = (L - 1) / B - j * kBlocks;   // block of the last context token, in this tile
            if (lb >= 0 && lb < kBlocks && ((ok >> lb) & 1u)) {
                const int t_from = (L - 1) % B + 1;     // first token past the context in that block
                for (int i = tid; i < (B - t_from) * (D / 8); i += 128) {
                    const int t = t_from + i / (D / 8), c = i % (D / 8);
                    *reinterpret_cast<uint4*>(vbase + lb * kTile + (c * B + t) * 16) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
        }
        tc::fence_before();
        __syncthreads();

        // S = Q K^T (one MMA per block and 16-dim step)
        if (tid == 0) {
            tc::fence_after();
            const uint32_t idesc_s = tc::instr_desc<T>(B, false);
            for (int b = 0; b < kBlocks; ++b) {
                if (!((ok >> b) & 1u)) continue;
                const uint32_t kb = smem_u32(kbase + b * kTile);
#pragma unroll
                for (int kc = 0; kc < D / 16; ++kc) {
                    const uint64_t a = tc::smem_desc(smem_u32(qs) + 2 * kc * 2048, 2048, 128);
                    const uint64_t bd = tc::smem_desc(kb + 2 * kc * B * 16, B * 16, 128);
                    tc::mma(s_tmem + b * B, a, bd, idesc_s, kc > 0);
                }
            }
            tc::commit(s_done);
        }
        if (!mbar_wait_bounded(s_done, j & 1, kWaitLimitNs)) failed = true;
        tc::fence_after();

        // online softmax over this thread's row of S (held in registers)
        float sv[kKeys];
        float mx = kNegInf;
#pragma unroll
        for (int c0 = 0; c0 < kKeys; c0 += 32) {
            float v[32];
            tc::ld32(s_tmem + lane_base + c0, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int col = c0 + i;
                const bool vis = ((ok >> (col / B)) & 1u) && key0 + col <= row_pos;
                sv[col] = vis ? v[i] * scale : kNegInf;
                mx = fmaxf(mx, sv[col]);
            }
        }
        // The reference maximum moves only when a score exceeds it by more than
        // 2^8 (base 2): P stays <= 256, exact for the sums, and O is rescaled
        // far less often (l and O share the reference, so the result is the
        // same softmax).
#ifndef PA_PREFILL_TC_SLACK
#define PA_PREFILL_TC_SLACK 8.f
#endif
        const float mn = (m_run == kNegInf || mx > m_run + PA_PREFILL_TC_SLACK) ? fmaxf(m_run, mx) : m_run;
        const float mu = mn == kNegInf ? 0.f : mn;
        const float alpha = exp2_approx(m_run - mu);
        m_run = mn;
        // the previous O += P V must be done before P is rewritten and O rescaled
        if (j > 0 && !mbar_wait_bounded(o_done, (j - 1) & 1, kWaitLimitNs)) failed = true;
        tc::fence_after();
        float rs = 0.f;
#pragma unroll
        for (int k8 = 0; k8 < kKeys / 8; ++k8) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a0 = exp2_approx(sv[8 * k8 + 2 * e] - mu);
                const float a1 = exp2_approx(sv[8 * k8 + 2 * e + 1] - mu);
                rs += a0 + a1;
                w[e] = Mma<T>::pack(a0, a1);
            }
            // P row, 8 keys per 16-byte core-matrix row: (8-row group, 8-key chunk k8) at k8*2048 + g*128
            *reinterpret_cast<uint4*>(ps + k8 * 2048 + (tid >> 3) * 128 + (tid & 7) * 16) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
        l_run = l_run * alpha + rs;
        // rescale this row of O, unless no row of the warp changed its maximum
        if (!__all_sync(0xffffffffu, alpha == 1.f)) {
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
        fence_proxy_async_smem();  // P (generic stores) visible to the tensor cores
        tc::fence_before();
        if (__syncthreads_or(failed ? 1 : 0)) {
            failed = true;
            break;
        }

        // O += P V (one MMA per block and 16-key step); then the stage is free
        if (tid == 0) {
            tc::fence_after();
            const uint32_t idesc_o = tc::instr_desc<T>(D, true);
            for (int b = 0; b < kBlocks; ++b) {
                if (!((ok >> b) & 1u)) continue;
                const uint32_t vb = smem_u32(vbase + b * kTile);
#pragma unroll
                for (int ks = 0; ks < B / 16; ++ks) {
                    const int kc = (b * B) / 8 + 2 * ks;   // first 8-key chunk of this step
                    const uint64_t a = tc::smem_desc(smem_u32(ps) + kc * 2048, 2048, 128);
                    const uint64_t bd = tc::smem_desc(vb + ks * 2 * 128, 128, B * 16);
                    tc::mma(o_tmem, a, bd, idesc_o, true);
                }
            }
            tc::commit(o_done);
            tc::commit(&empty[st]);
            if (j + 2 < ntiles) {
                if (mbar_wait_bounded(&empty[st], (j >> 1) & 1, kWaitLimitNs)) {
                    issue(j + 2);
                } else {
                    failed = true;
                }
            }
        }
    }

    // ---- drain, write the rows, release tensor memory
    if (!failed && ntiles > 0 && !mbar_wait_bounded(o_done, (ntiles - 1) & 1, kWaitLimitNs)) failed = true;
    if (__syncthreads_or(failed ? 1 : 0)) {
        if (tid == 0) {
            flag_error(8 /* PA_DEVERR_TIMEOUT */);
            // let the tensor-core work and copies already issued finish before the CTA exits
            mbar_wait_bounded(o_done, (j > 0 ? j - 1 : 0) & 1, kWaitLimitNs);
            for (int k = j; k < ntiles && k < j + 2; ++k) mbar_wait_bounded(&full[k & 1], (k >> 1) & 1, kWaitLimitNs);
        }
    } else {
        tc::fence_after();
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        T* dst = reinterpret_cast<T*>(p.out) +
                 (static_cast<long long>(q0 + (row_ok ? row_tok : tok0)) * p.num_q_heads + row_head) * D;
        float v[32];
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
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
    tc::fence_before();
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

}  // namespace pa
