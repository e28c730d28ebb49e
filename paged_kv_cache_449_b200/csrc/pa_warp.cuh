// Per-warp decode state: the running softmax statistics and output
// accumulator of the g = Hq/Hkv query heads of one (sequence, kv head), and
// the computation of one KV block staged in shared memory.
//
// Online softmax ("从源码剖析 vLLM 的显存管理与连续批处理" §2.3 computes attention
// over the gathered K/V; the streaming form is a reordering of that sum): for
// each block, m_new = max(m, max_t s_t); the accumulator and the running sum
// are rescaled by exp(m - m_new) and the block's exp(s_t - m_new) terms added.
//
// Emitting the state:
//   write_out     out = acc / l rounded once to the output type (complete);
//   write_record  (acc, m, l) for a later log-sum-exp merge:  record layout
//                 [g][D] acc, then [g] m, then [g] l (fp32);
//   store_smem    the same, into the CTA-merge area of shared memory.
#pragma once

#include "pa_device.cuh"
#include "pa_e4m3.cuh"

namespace pa {

constexpr int kMaxGroup = 8;

// Row stride (floats) of the accumulator rows in the CTA-merge area of shared
// memory: four floats of padding put the rows that one store instruction
// writes (the heads of a thread, two rows apart) in different banks.
template <int D>
constexpr int kMergeRow = D + 4;

template <typename T>
struct IsF32 {
    static constexpr bool value = false;
};
template <>
struct IsF32<float> {
    static constexpr bool value = true;
};

// ----------------------------------------------------------------------------
// 16-bit inputs: tensor-core MMA with tokens as the M dimension.
//   S^T = K Q^T     (M = 16 tokens, N = 8 query heads of the group, K = head dim)
//   O^T += V^T P^T  (M = 16 head-dim rows, N = 8 query heads, K = 16 tokens)
// Thread (r = lane/4, c = lane%4) holds S^T rows (tokens) r and r+8 for heads
// 2c and 2c+1, so it keeps the softmax statistics of those two heads; P^T goes
// from the accumulator layout to the B-operand layout with one movmatrix
// (8x8 transpose) per 8 tokens.  The query heads of a GQA group fill the N
// dimension (g <= 8), so no MMA row is padding.

template <typename T, int D, int B>
struct WarpMma {
    static constexpr int kMt = D / 16;  // 16-row tiles of head_dim in O^T
    float o[kMt][4];                    // O^T: (d=16mt+r, h=2c), (d, 2c+1), (d+8, 2c), (d+8, 2c+1)
    uint32_t qa[D / 16][2];             // Q as the B operand: head r, d = 16ks+2c.., 16ks+8+2c..
    float m_run[2];                     // heads 2c, 2c+1 (score domain, base 2)
    float l_run[2];                     // this thread's share of the sums of heads 2c, 2c+1

    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int mt = 0; mt < kMt; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
        m_run[0] = m_run[1] = kNegInf;
        l_run[0] = l_run[1] = 0.f;
    }

    static __device__ __forceinline__ void fetch_q(uint32_t (&dst)[D / 16][2], const T* q_rows, int group,
                                                   int lane) {
        const int r = lane >> 2, c = lane & 3;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            if (r < group) {
                const T* row = q_rows + r * D + ks * 16 + 2 * c;
                dst[ks][0] = *reinterpret_cast<const uint32_t*>(row);
                dst[ks][1] = *reinterpret_cast<const uint32_t*>(row + 8);
            } else {
                dst[ks][0] = dst[ks][1] = 0u;
            }
        }
    }
    __device__ __forceinline__ void load_q(const T* q_rows, int group, int lane) { fetch_q(qa, q_rows, group, lane); }

    // Zero the 16-bit halves of a V fragment register that belong to tokens
    // >= valid (token `tok` in the low half, tok+1 in the high half).
    static __device__ __forceinline__ uint32_t mask_pair(uint32_t v, int tok, int valid) {
        const uint32_t keep = (tok < valid ? 0x0000ffffu : 0u) | (tok + 1 < valid ? 0xffff0000u : 0u);
        return v & keep;
    }

    // One block of B tokens: K tile at kbase, V tile at vbase (shared memory,
    // layout [D/8][B][8]; E4M3: the 8-bit pools' K and V tile layouts, codes
    // widened to fp16 in registers); tokens >= valid are masked out.
    template <bool E4M3 = false>
    __device__ __forceinline__ void block(uint32_t kbase, uint32_t vbase, int valid, int group, float scale_log2,
                                          int lane) {
        const int r = lane >> 2, c = lane & 3;
        const int mtx = lane >> 3, row = lane & 7;
        const bool h0ok = 2 * c < group, h1ok = 2 * c + 1 < group;
        constexpr int kGroups = B >= 16 ? B / 16 : 1;  // 16-token groups in the block
#pragma unroll
        for (int tg = 0; tg < kGroups; ++tg) {
            // S^T = K Q^T
            float sc[4] = {0.f, 0.f, 0.f, 0.f};
            if constexpr (B >= 16) {
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    uint32_t a0, a1, a2, a3;
                    if constexpr (E4M3) {  // tokens r, r+8 of the group; dims 2c.., 2c+8.. of vector ks
                        const uint32_t at = kbase + ((ks * B + tg * 16 + r) * 16 + 4 * c);
                        e4m3x4_to_frags(lds32(at), a0, a2);
                        e4m3x4_to_frags(lds32(at + 8 * 16), a1, a3);
                    } else {
                        const int tok = tg * 16 + (mtx & 1) * 8 + row;
                        const int chunk = 2 * ks + (mtx >> 1);
                        ldsm_x4(kbase + (chunk * B + tok) * 16, a0, a1, a2, a3);
                    }
                    Mma<T>::k16(sc, a0, a1, a2, a3, qa[ks][0], qa[ks][1]);
                }
            } else if constexpr (E4M3) {  // 8-token blocks: rows 8..15 of the tile are zero
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    uint32_t a0, a2;
                    e4m3x4_to_frags(lds32(kbase + ((ks * 8 + r) * 16 + 4 * c)), a0, a2);
                    Mma<T>::k16(sc, a0, 0u, a2, 0u, qa[ks][0], qa[ks][1]);
                }
            } else {  // 8-token blocks: rows 8..15 of the tile are zero
#pragma unroll
                for (int kq = 0; kq < D / 32; ++kq) {
                    uint32_t x0, x1, x2, x3;
                    ldsm_x4(kbase + ((4 * kq + mtx) * 8 + row) * 16, x0, x1, x2, x3);
                    Mma<T>::k16(sc, x0, 0u, x1, 0u, qa[2 * kq][0], qa[2 * kq][1]);
                    Mma<T>::k16(sc, x2, 0u, x3, 0u, qa[2 * kq + 1][0], qa[2 * kq + 1][1]);
                }
            }

            // Online softmax per head (column) over the 16 tokens (rows).
            const int t_lo = tg * 16 + r, t_hi = t_lo + 8;
            float x0 = (h0ok && t_lo < valid) ? sc[0] * scale_log2 : kNegInf;
            float x1 = (h1ok && t_lo < valid) ? sc[1] * scale_log2 : kNegInf;
            float x2 = (h0ok && t_hi < valid) ? sc[2] * scale_log2 : kNegInf;
            float x3 = (h1ok && t_hi < valid) ? sc[3] * scale_log2 : kNegInf;
            float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
            }
            const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
            const float mu0 = mn0 == kNegInf ? 0.f : mn0, mu1 = mn1 == kNegInf ? 0.f : mn1;
            const float al0 = exp2_approx(m_run[0] - mu0), al1 = exp2_approx(m_run[1] - mu1);
            const float p0 = exp2_approx(x0 - mu0), p1 = exp2_approx(x1 - mu1);
            const float p2 = exp2_approx(x2 - mu0), p3 = exp2_approx(x3 - mu1);
            l_run[0] = l_run[0] * al0 + (p0 + p2);
            l_run[1] = l_run[1] * al1 + (p1 + p3);
            m_run[0] = mn0;
            m_run[1] = mn1;
#pragma unroll
            for (int mt = 0; mt < kMt; ++mt) {
                o[mt][0] *= al0;
                o[mt][1] *= al1;
                o[mt][2] *= al0;
                o[mt][3] *= al1;
            }

            // P^T from the accumulator layout to the B operand of O^T += V^T P^T.
            const uint32_t b0 = movmatrix_trans(Mma<T>::pack(p0, p1));  // tokens 0..7 of the group
            const uint32_t b1 = movmatrix_trans(Mma<T>::pack(p2, p3));  // tokens 8..15
            const bool partial = valid < tg * 16 + 16;
            if constexpr (B >= 16) {
                const int tlo = tg * 16 + 2 * c, thi = tlo + 8;
#pragma unroll
                for (int mt = 0; mt < kMt; ++mt) {
                    uint32_t a0, a1, a2, a3;
                    if constexpr (E4M3) {  // dim rows r, r+8 of tile mt; tokens 2c.., 2c+8.. of the group
                        const uint32_t at = vbase + ((16 * mt + r) * B + 16 * tg + 4 * c);
                        e4m3x4_to_frags(lds32(at), a0, a2);
                        e4m3x4_to_frags(lds32(at + 8 * B), a1, a3);
                    } else {
                        const int tok = tg * 16 + (mtx >> 1) * 8 + row;
                        const int chunk = 2 * mt + (mtx & 1);
                        ldsm_x4_trans(vbase + (chunk * B + tok) * 16, a0, a1, a2, a3);
                    }
                    if (partial) {
                        a0 = mask_pair(a0, tlo, valid);
                        a1 = mask_pair(a1, tlo, valid);
                        a2 = mask_pair(a2, thi, valid);
                        a3 = mask_pair(a3, thi, valid);
                    }
                    Mma<T>::k16(o[mt], a0, a1, a2, a3, b0, b1);
                }
            } else if constexpr (E4M3) {
#pragma unroll
                for (int mt = 0; mt < kMt; ++mt) {
                    uint32_t y0 = e4m3x2_to_frag(lds16(vbase + ((16 * mt + r) * 8 + 2 * c)));
                    uint32_t y1 = e4m3x2_to_frag(lds16(vbase + ((16 * mt + r + 8) * 8 + 2 * c)));
                    if (partial) {
                        y0 = mask_pair(y0, 2 * c, valid);
                        y1 = mask_pair(y1, 2 * c, valid);
                    }
                    Mma<T>::k8(o[mt], y0, y1, b0);
                }
            } else {
#pragma unroll
                for (int mq = 0; mq < D / 32; ++mq) {
                    uint32_t y0, y1, y2, y3;
                    ldsm_x4_trans(vbase + ((4 * mq + mtx) * 8 + row) * 16, y0, y1, y2, y3);
                    if (partial) {
                        y0 = mask_pair(y0, 2 * c, valid);
                        y1 = mask_pair(y1, 2 * c, valid);
                        y2 = mask_pair(y2, 2 * c, valid);
                        y3 = mask_pair(y3, 2 * c, valid);
                    }
                    Mma<T>::k8(o[2 * mq], y0, y1, b0);
                    Mma<T>::k8(o[2 * mq + 1], y2, y3, b0);
                }
            }
        }
    }

    // Two 16-token blocks (a and b) in one online-softmax step: one row
    // maximum, one rescale of O^T and the running sums for the 32 tokens.
    // Scores S^T of block a in sa, of block b in sb; returns the P^T operands
    // of both blocks.
    __device__ __forceinline__ void softmax_step2(const float (&sa)[4], const float (&sb)[4], int valid_a,
                                                  int valid_b, int group, float scale_log2, int lane,
                                                  uint32_t (&pa)[2], uint32_t (&pb)[2]) {
        const int r = lane >> 2, c = lane & 3;
        const bool h0ok = 2 * c < group, h1ok = 2 * c + 1 < group;
        const int t_lo = r, t_hi = r + 8;
        const float xa0 = (h0ok && t_lo < valid_a) ? sa[0] * scale_log2 : kNegInf;
        const float xa1 = (h1ok && t_lo < valid_a) ? sa[1] * scale_log2 : kNegInf;
        const float xa2 = (h0ok && t_hi < valid_a) ? sa[2] * scale_log2 : kNegInf;
        const float xa3 = (h1ok && t_hi < valid_a) ? sa[3] * scale_log2 : kNegInf;
        const float xb0 = (h0ok && t_lo < valid_b) ? sb[0] * scale_log2 : kNegInf;
        const float xb1 = (h1ok && t_lo < valid_b) ? sb[1] * scale_log2 : kNegInf;
        const float xb2 = (h0ok && t_hi < valid_b) ? sb[2] * scale_log2 : kNegInf;
        const float xb3 = (h1ok && t_hi < valid_b) ? sb[3] * scale_log2 : kNegInf;
        float mx0 = fmaxf(fmaxf(xa0, xa2), fmaxf(xb0, xb2));
        float mx1 = fmaxf(fmaxf(xa1, xa3), fmaxf(xb1, xb3));
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
        const float mu0 = mn0 == kNegInf ? 0.f : mn0, mu1 = mn1 == kNegInf ? 0.f : mn1;
        const float al0 = exp2_approx(m_run[0] - mu0), al1 = exp2_approx(m_run[1] - mu1);
        const float pa0 = exp2_approx(xa0 - mu0), pa1 = exp2_approx(xa1 - mu1);
        const float pa2 = exp2_approx(xa2 - mu0), pa3 = exp2_approx(xa3 - mu1);
        const float pb0 = exp2_approx(xb0 - mu0), pb1 = exp2_approx(xb1 - mu1);
        const float pb2 = exp2_approx(xb2 - mu0), pb3 = exp2_approx(xb3 - mu1);
        l_run[0] = l_run[0] * al0 + ((pa0 + pa2) + (pb0 + pb2));
        l_run[1] = l_run[1] * al1 + ((pa1 + pa3) + (pb1 + pb3));
        m_run[0] = mn0;
        m_run[1] = mn1;
#pragma unroll
        for (int mt = 0; mt < kMt; ++mt) {
            o[mt][0] *= al0;
            o[mt][1] *= al1;
            o[mt][2] *= al0;
            o[mt][3] *= al1;
        }
        pa[0] = movmatrix_trans(Mma<T>::pack(pa0, pa1));
        pa[1] = movmatrix_trans(Mma<T>::pack(pa2, pa3));
        pb[0] = movmatrix_trans(Mma<T>::pack(pb0, pb1));
        pb[1] = movmatrix_trans(Mma<T>::pack(pb2, pb3));
    }

    // Fragments of 16-token blocks (B = 16): K rows (tokens r, r+8; dims of
    // vector ks) and V^T rows (dims 16mt+r, +8; tokens 2c.., 2c+8..).
    template <bool E4M3>
    static __device__ __forceinline__ void k_frag(uint32_t kbase, int ks, int lane, uint32_t& a0, uint32_t& a1,
                                                  uint32_t& a2, uint32_t& a3) {
        const int r = lane >> 2, c = lane & 3;
        if constexpr (E4M3) {
            const uint32_t at = kbase + ((ks * 16 + r) * 16 + 4 * c);
            e4m3x4_to_frags(lds32(at), a0, a2);
            e4m3x4_to_frags(lds32(at + 8 * 16), a1, a3);
        } else {
            const int mtx = lane >> 3, row = lane & 7;
            const int tok = (mtx & 1) * 8 + row;
            const int chunk = 2 * ks + (mtx >> 1);
            ldsm_x4(kbase + (chunk * 16 + tok) * 16, a0, a1, a2, a3);
        }
    }
    template <bool E4M3>
    static __device__ __forceinline__ void v_frag(uint32_t vbase, int mt, int lane, uint32_t& a0, uint32_t& a1,
                                                  uint32_t& a2, uint32_t& a3) {
        const int r = lane >> 2, c = lane & 3;
        if constexpr (E4M3) {
            const uint32_t at = vbase + ((16 * mt + r) * 16 + 4 * c);
            e4m3x4_to_frags(lds32(at), a0, a2);
            e4m3x4_to_frags(lds32(at + 8 * 16), a1, a3);
        } else {
            const int mtx = lane >> 3, row = lane & 7;
            const int tok = (mtx >> 1) * 8 + row;
            const int chunk = 2 * mt + (mtx & 1);
            ldsm_x4_trans(vbase + (chunk * 16 + tok) * 16, a0, a1, a2, a3);
        }
    }

    // Two blocks of 16 tokens (a, b) in one step: the K and V tiles of each
    // staged as block() takes them; tokens >= valid_a (valid_b) masked out.
    template <bool E4M3 = false>
    __device__ __forceinline__ void block2(uint32_t ka, uint32_t va, int valid_a, uint32_t kb, uint32_t vb,
                                           int valid_b, int group, float scale_log2, int lane) {
        static_assert(B == 16, "16-token blocks");
        const int c = lane & 3;
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
            k_frag<E4M3>(ka, ks, lane, a0, a1, a2, a3);
            k_frag<E4M3>(kb, ks, lane, b0, b1, b2, b3);
            Mma<T>::k16(sa, a0, a1, a2, a3, qa[ks][0], qa[ks][1]);
            Mma<T>::k16(sb, b0, b1, b2, b3, qa[ks][0], qa[ks][1]);
        }
        uint32_t pa[2], pb[2];
        softmax_step2(sa, sb, valid_a, valid_b, group, scale_log2, lane, pa, pb);
        const int tlo = 2 * c, thi = tlo + 8;
#pragma unroll
        for (int mt = 0; mt < kMt; ++mt) {
            uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
            v_frag<E4M3>(va, mt, lane, a0, a1, a2, a3);
            v_frag<E4M3>(vb, mt, lane, b0, b1, b2, b3);
            if (valid_a < 16) {
                a0 = mask_pair(a0, tlo, valid_a);
                a1 = mask_pair(a1, tlo, valid_a);
                a2 = mask_pair(a2, thi, valid_a);
                a3 = mask_pair(a3, thi, valid_a);
            }
            if (valid_b < 16) {
                b0 = mask_pair(b0, tlo, valid_b);
                b1 = mask_pair(b1, tlo, valid_b);
                b2 = mask_pair(b2, thi, valid_b);
                b3 = mask_pair(b3, thi, valid_b);
            }
            Mma<T>::k16(o[mt], a0, a1, a2, a3, pa[0], pa[1]);
            Mma<T>::k16(o[mt], b0, b1, b2, b3, pb[0], pb[1]);
        }
    }

    __device__ __forceinline__ float head_sum(int e) const {
        float l = l_run[e];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        return l;
    }

    // Calls f(head, d, value) for every accumulator element of a valid head.
    template <typename F>
    __device__ __forceinline__ void for_each(int group, int lane, F&& f) const {
        const int r = lane >> 2, c = lane & 3;
#pragma unroll
        for (int mt = 0; mt < kMt; ++mt) {
            const int d0 = 16 * mt + r;
            if (2 * c < group) {
                f(0, d0, o[mt][0]);
                f(0, d0 + 8, o[mt][2]);
            }
            if (2 * c + 1 < group) {
                f(1, d0, o[mt][1]);
                f(1, d0 + 8, o[mt][3]);
            }
        }
    }

    // Writes this warp's (m, l, o) for its valid heads into the CTA-merge area.
    __device__ __forceinline__ void store_smem(float* mo, float* mml, int warp, int group, int lane) {
        const int r = lane >> 2, c = lane & 3;
        const float l0 = head_sum(0), l1 = head_sum(1);
        for_each(group, lane, [&](int e, int d, float v) { mo[(warp * kMaxGroup + 2 * c + e) * kMergeRow<D> + d] = v; });
        if (r == 0) {
            if (2 * c < group) {
                mml[(warp * kMaxGroup + 2 * c) * 2] = m_run[0];
                mml[(warp * kMaxGroup + 2 * c) * 2 + 1] = l0;
            }
            if (2 * c + 1 < group) {
                mml[(warp * kMaxGroup + 2 * c + 1) * 2] = m_run[1];
                mml[(warp * kMaxGroup + 2 * c + 1) * 2 + 1] = l1;
            }
        }
    }

    // Normalised output rows out[h][d] = o / l (zero when l == 0).
    __device__ __forceinline__ void write_out(T* rows, int group, int lane) {
        const int c = lane & 3;
        const float l0 = head_sum(0), l1 = head_sum(1);
        const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
        for_each(group, lane, [&](int e, int d, float v) {
            rows[(2 * c + e) * D + d] = from_float<T>(v * (e ? inv1 : inv0));
        });
    }

    __device__ __forceinline__ void write_record(float* rec, int group, int lane) {
        const int r = lane >> 2, c = lane & 3;
        const float l0 = head_sum(0), l1 = head_sum(1);
        for_each(group, lane, [&](int e, int d, float v) { rec[(2 * c + e) * D + d] = v; });
        if (r == 0) {
            if (2 * c < group) {
                rec[group * D + 2 * c] = m_run[0];
                rec[group * D + group + 2 * c] = l0;
            }
            if (2 * c + 1 < group) {
                rec[group * D + 2 * c + 1] = m_run[1];
                rec[group * D + group + 2 * c + 1] = l1;
            }
        }
    }
};

// ----------------------------------------------------------------------------
// fp32 inputs: CUDA-core FMA.  QK^T: lane -> (token t = lane % B, a 1/(32/B)
// share of D), reduced across the sharing lanes.  PV: lane -> one 16-byte
// vector of D (and, for D = 64, half of the tokens).  The query rows of the
// current pair are read from shared memory (`qs`, [g][D] floats).

template <int D, int B>
struct WarpF32 {
    static constexpr int kC = D / 4;          // 16-byte vectors per token row
    static constexpr int kTg = 32 / B;        // lanes sharing one token in QK^T
    static constexpr int kCpp = kC / kTg;     // vectors per lane in QK^T
    static constexpr int kGrp = 32 / kC;      // token groups in PV (1 for D=128, 2 for D=64)
    float o[kMaxGroup][4];
    float m_run[kMaxGroup];
    float l_run[kMaxGroup];
    const float* qs;

    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            o[h][0] = o[h][1] = o[h][2] = o[h][3] = 0.f;
            m_run[h] = kNegInf;
            l_run[h] = 0.f;
        }
    }

    // Copies the group's query rows into the warp's shared-memory slot.
    __device__ __forceinline__ void load_q(float* slot, const float* q_rows, int group, int lane) {
        __syncwarp();
        for (int i = lane; i < group * D; i += 32) slot[i] = q_rows[i];
        __syncwarp();
        qs = slot;
    }

    __device__ __forceinline__ void block(const float* ktile, const float* vtile, int valid, int group, float scale,
                                          int lane) {
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

    // Folds the two token groups of the D = 64 layout into lanes 0..15.
    __device__ __forceinline__ void fold_groups() {
        if constexpr (kGrp == 2) {
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h)
#pragma unroll
                for (int e = 0; e < 4; ++e) o[h][e] += __shfl_xor_sync(0xffffffffu, o[h][e], 16);
        }
    }

    __device__ __forceinline__ void store_smem(float* mo, float* mml, int warp, int group, int lane) {
        fold_groups();
        const int cj = lane % kC, tg = lane / kC;
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            if (h < group && tg == 0) {
                float* dst = mo + (warp * kMaxGroup + h) * kMergeRow<D> + cj * 4;
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

    __device__ __forceinline__ void write_out(float* rows, int group, int lane) {
        fold_groups();
        const int cj = lane % kC, tg = lane / kC;
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            if (h < group && tg == 0) {
                const float l = l_run[h];
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (l > 0.f) v = make_float4(o[h][0] / l, o[h][1] / l, o[h][2] / l, o[h][3] / l);
                *reinterpret_cast<float4*>(rows + h * D + cj * 4) = v;
            }
        }
    }

    __device__ __forceinline__ void write_record(float* rec, int group, int lane) {
        fold_groups();
        const int cj = lane % kC, tg = lane / kC;
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            if (h < group && tg == 0)
                *reinterpret_cast<float4*>(rec + h * D + cj * 4) = make_float4(o[h][0], o[h][1], o[h][2], o[h][3]);
            if (h < group && lane == 0) {
                rec[group * D + h] = m_run[h];
                rec[group * D + group + h] = l_run[h];
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

}  // namespace pa
