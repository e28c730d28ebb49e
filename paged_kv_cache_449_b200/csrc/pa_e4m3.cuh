// 8-bit (e4m3) KV pools: the FP8 attention named as the next optimisation in
// "vLLM框架解析：PagedAttention技术如何实现LLM推理20倍加速" §7, read as an 8-bit
// KV cache with one fp32 scale per kv head for K and one for V.
//
//  * write: code = e4m3(x / scale), the division in fp32 (IEEE round to
//    nearest), the conversion rounding to nearest-even and saturating to
//    +-448 (CUDA's conversion, checked bit for bit against an independent
//    encoder in the tests);
//  * read: a code stands for e4m3_value(code) * scale.  Every e4m3 value is
//    exactly an fp16 value (3 mantissa bits, exponents 2^-9 .. 2^8), so codes
//    are widened to fp16 without rounding and run through the fp16
//    tensor-core path; the K scale joins the score scale and the V scale
//    multiplies the finished output.
//  * pool layout (one (block, head) tile = B*D contiguous bytes): K as
//    [D/16][B][16] with dims 2c, 2c+1, 2c+8, 2c+9 of a 16-dim vector at bytes
//    4c..4c+3; V transposed, [D][B], with tokens 2c, 2c+1, 2c+8, 2c+9 of each
//    16-token group at bytes 4c..4c+3 (B = 8: natural order).  One 32-bit
//    shared-memory load then holds exactly the four codes a thread needs for
//    its part of an MMA A fragment (rows r, cols 2c.., 2c+8..), so staged
//    tiles feed the tensor cores without ldmatrix or a widened copy.
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

__device__ __forceinline__ uint32_t quantise2(float a, float b, float scale) {
    float2 f;
    f.x = __fdiv_rn(a, scale);
    f.y = __fdiv_rn(b, scale);
    return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3));
}

// Byte of token t inside a V row of B codes.
__device__ __forceinline__ int v_row_byte(int t, int B) {
    if (B == 8) return t;
    const int u = t & 15;
    return (t & ~15) + 4 * ((u & 7) >> 1) + 2 * (u >> 3) + (u & 1);
}

// Four codes (one 32-bit shared-memory word) -> the two fp16x2 fragment
// registers they form: bytes 0-1 and bytes 2-3.
//   PA_E4M3_CVT 0: CUDA's conversion intrinsic per pair;
//               1: the hardware conversion (cvt.rn.f16x2.e4m3x2) on the two
//                  16-bit halves of the word;
//               2: bit placement: code s.eeee.mmm becomes the fp16 pattern
//                  s.0eeee.mmm0000000, which is the code's value times 2^-8
//                  exactly (normal and subnormal codes alike; the 2^8 is
//                  folded into the K and V scales: kE4m3Unit).
#ifndef PA_E4M3_CVT
#define PA_E4M3_CVT 1
#endif
constexpr float kE4m3Unit = PA_E4M3_CVT == 2 ? 256.f : 1.f;

__device__ __forceinline__ void e4m3x4_to_frags(uint32_t w, uint32_t& lo, uint32_t& hi) {
#if PA_E4M3_CVT == 0
    lo = e4m3x2_to_half2(w);
    hi = e4m3x2_to_half2(w >> 16);
#elif PA_E4M3_CVT == 1
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi) : "r"(w));
#else
    // byte k of w to the high byte of a 16-bit lane, then drop the sign's
    // neighbour bit: (x & 0x8000) | ((x >> 1) & 0x3f80) per lane
    const uint32_t x0 = __byte_perm(w, 0u, 0x1404);   // [b1:00 | b0:00]
    const uint32_t x1 = __byte_perm(w, 0u, 0x3424);   // [b3:00 | b2:00]
    lo = (x0 & 0x80008000u) | ((x0 >> 1) & 0x3f803f80u);
    hi = (x1 & 0x80008000u) | ((x1 >> 1) & 0x3f803f80u);
#endif
}

// Two codes in the low 16 bits -> one fp16x2 register (same scaling as above).
__device__ __forceinline__ uint32_t e4m3x2_to_frag(uint32_t w) {
#if PA_E4M3_CVT == 0
    return e4m3x2_to_half2(w);
#elif PA_E4M3_CVT == 1
    uint32_t r;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, l;\n\t}" : "=r"(r) : "r"(w));
    return r;
#else
    const uint32_t x = __byte_perm(w, 0u, 0x1404);
    return (x & 0x80008000u) | ((x >> 1) & 0x3f803f80u);
#endif
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
