// 8-bit (e4m3) KV pools: the FP8 attention named as the next optimisation in
// "vLLM框架解析：PagedAttention技术如何实现LLM推理20倍加速" §7, read as an 8-bit
// KV cache with one fp32 scale per kv head for K and one for V.
//
//  * write: code = e4m3(x / scale), the division in fp32 (IEEE round to
//    nearest), the conversion rounding to nearest-even and saturating to
//    +-448 (CUDA's conversion, checked bit for bit against an independent
//    encoder in the tests);
//  * read: a code stands for e4m3_value(code) * scale.  Every e4m3 value is
//    exactly an fp16 value (3 mantissa bits, exponents 2^-9 .. 2^8), so a
//    staged tile is widened to fp16 without rounding and runs through the
//    fp16 tensor-core path; the K scale joins the score scale and the V
//    scale multiplies the finished output.
//  * pool layout: [num_blocks][Hkv][D/16][B][16] bytes (16 codes per 16-byte
//    vector), the same vector-outer / token-inner order as the 16-bit pools.
#pragma once

#include <cuda_fp8.h>

#include <type_traits>

#include "pa_device.cuh"

namespace pa {

template <typename T>
__device__ __forceinline__ float to_float(T x);
template <>
__device__ __forceinline__ float to_float<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_float<__half>(__half x) { return __half2float(x); }
template <>
__device__ __forceinline__ float to_float<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Two e4m3 codes (low byte first) -> two fp16 values in one 32-bit word.
__device__ __forceinline__ uint32_t e4m3x2_to_half2(uint32_t two_codes) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes & 0xffffu),
                                                      __NV_E4M3);
    return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

// Sixteen consecutive elements of a row -> sixteen codes (one 16-byte vector).
template <typename T>
__device__ __forceinline__ uint4 quantise16(const T* row, float scale) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int i = 4 * k + 2 * e;
            float2 f;
            f.x = __fdiv_rn(to_float<T>(row[i]), scale);
            f.y = __fdiv_rn(to_float<T>(row[i + 1]), scale);
            const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
            word |= static_cast<uint32_t>(c) << (16 * e);
        }
        w[k] = word;
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// A staged e4m3 (block, head) tile [D/16][B][16] -> an fp16 tile [D/8][B][8]
// in the warp's scratch area (the layout the fp16 MMA path reads).
template <int D, int B>
__device__ __forceinline__ void widen_tile(const uint8_t* src, uint8_t* dst, int lane) {
    constexpr int kVecs = D / 16 * B;
#pragma unroll
    for (int vi = lane; vi < kVecs; vi += 32) {
        const uint4 c = *reinterpret_cast<const uint4*>(src + vi * 16);
        const int v = vi / B, t = vi - v * B;
        uint4 lo, hi;
        lo.x = e4m3x2_to_half2(c.x);
        lo.y = e4m3x2_to_half2(c.x >> 16);
        lo.z = e4m3x2_to_half2(c.y);
        lo.w = e4m3x2_to_half2(c.y >> 16);
        hi.x = e4m3x2_to_half2(c.z);
        hi.y = e4m3x2_to_half2(c.z >> 16);
        hi.z = e4m3x2_to_half2(c.w);
        hi.w = e4m3x2_to_half2(c.w >> 16);
        *reinterpret_cast<uint4*>(dst + ((2 * v) * B + t) * 16) = lo;
        *reinterpret_cast<uint4*>(dst + ((2 * v + 1) * B + t) * 16) = hi;
    }
}

// Query fragments for the fp16 MMA from 16-bit query rows.  fp16 rows load
// as they are (shift 0).  bf16 rows are scaled by 2^shift, one power of two
// for the whole group, chosen so that the largest magnitude lands in
// [2^13, 2^14): the products are exact and the fp16 conversion keeps every
// element's significand except those below 2^-24 of that range.  The scores
// are then 2^shift too large; the caller divides it out.
template <typename TQ, int D>
__device__ __forceinline__ int load_q_half(uint32_t (&qa)[D / 16][2], const TQ* q_rows, int group, int lane) {
    const int r = lane >> 2, c = lane & 3;
    if constexpr (std::is_same<TQ, __half>::value) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            if (r < group) {
                const TQ* row = q_rows + r * D + ks * 16 + 2 * c;
                qa[ks][0] = *reinterpret_cast<const uint32_t*>(row);
                qa[ks][1] = *reinterpret_cast<const uint32_t*>(row + 8);
            } else {
                qa[ks][0] = qa[ks][1] = 0u;
            }
        }
        return 0;
    } else {
        float f[D / 16][4];
        float mx = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
            for (int e = 0; e < 4; ++e) f[ks][e] = 0.f;
            if (r < group) {
                const TQ* row = q_rows + r * D + ks * 16 + 2 * c;
                f[ks][0] = to_float<TQ>(row[0]);
                f[ks][1] = to_float<TQ>(row[1]);
                f[ks][2] = to_float<TQ>(row[8]);
                f[ks][3] = to_float<TQ>(row[9]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) mx = fmaxf(mx, fabsf(f[ks][e]));
        }
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        // floor(log2(mx)) from the exponent field (mx is a normal or zero bf16 value)
        const int e2 = mx > 0.f ? static_cast<int>((__float_as_uint(mx) >> 23) & 0xff) - 127 : 13;
        int shift = 13 - e2;
        shift = shift > 100 ? 100 : (shift < -100 ? -100 : shift);
        const float mul = __uint_as_float(static_cast<uint32_t>(127 + shift / 2) << 23);   // 2^(shift/2)
        const float mul2 = __uint_as_float(static_cast<uint32_t>(127 + shift - shift / 2) << 23);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const __half2 a = __floats2half2_rn(f[ks][0] * mul * mul2, f[ks][1] * mul * mul2);
            const __half2 b = __floats2half2_rn(f[ks][2] * mul * mul2, f[ks][3] * mul * mul2);
            qa[ks][0] = *reinterpret_cast<const uint32_t*>(&a);
            qa[ks][1] = *reinterpret_cast<const uint32_t*>(&b);
        }
        return shift;
    }
}

}  // namespace pa
