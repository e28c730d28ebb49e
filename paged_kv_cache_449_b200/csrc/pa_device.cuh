// Device-side building blocks for sm_100a: mbarrier-tracked bulk copies
// (the 1-D form of the Tensor Memory Accelerator copy, no multicast), shared
// memory matrix loads, warp-level tensor-core MMA, and small numeric helpers.
// All inline PTX here is hand-written from the public PTX ISA.
#pragma once

#include <cmath>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace pa {

// Device error word (one per GPU that loads the library).  Bits are the
// PA_DEVERR_* values of pa.h.
__device__ int g_device_error;

__device__ __forceinline__ void flag_error(int bit) { atomicOr(&g_device_error, bit); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the asynchronous (copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Non-blocking probe of a phase (try_wait may suspend the thread for a while).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait, far above any copy time

#ifdef PA_TEST_HOOKS
// Test builds only (libpa_test.so): the wait limit, and a switch that makes
// the first warp of the decode CTA of (sequence 0, kv head 0, partition 0)
// leave its first ring stage unfilled, so that its wait runs out and the
// kernel's timeout path runs (no copy is left in flight: the stage is simply
// never issued).
__device__ unsigned long long g_test_wait_limit_ns = kWaitLimitNs;
__device__ int g_test_skip_first_copy = 0;
__device__ __forceinline__ uint64_t wait_limit_ns() { return g_test_wait_limit_ns; }
#else
__device__ __forceinline__ constexpr uint64_t wait_limit_ns() { return kWaitLimitNs; }
#endif

// Waits for phase `parity` of `bar` to complete, giving up after `limit_ns`
// of wall time (returns false then).  Never spins without bound.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t start = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - start > limit_ns) return false;
    }
    return true;
}

// ---------------------------------------------------------------- bulk copy

// Orders this thread's generic-proxy shared-memory writes before later
// asynchronous-proxy (bulk copy) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// L2 policy: data read once (streamed KV tiles) is evicted first.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t policy;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
    return policy;
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses
// 16-byte aligned); completion is counted on `bar` as transaction bytes.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// Plain shared-memory loads (volatile: they must stay after the mbarrier
// wait that makes the staged bytes visible).
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t addr) {
    uint16_t v;
    asm volatile("ld.shared.b16 %0, [%1];" : "=h"(v) : "r"(addr) : "memory");
    return v;
}

// ---------------------------------------------------------------- ldmatrix / mma

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// Transpose of an 8x8 matrix of 16-bit elements held as one register per
// thread (thread t owns row t/4, columns 2(t%4), 2(t%4)+1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

template <typename T>
struct Mma;

template <>
struct Mma<__nv_bfloat16> {
    // D(16x8 f32) += A(16x16 bf16, row) * B(16x8 bf16, col)
    static __device__ __forceinline__ void k16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
    static __device__ __forceinline__ void k8(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
        asm volatile(
            "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(b0));
    }
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&v);
    }
};

template <>
struct Mma<__half> {
    static __device__ __forceinline__ void k16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
    static __device__ __forceinline__ void k8(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
        asm volatile(
            "mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(b0));
    }
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&v);
    }
};

// Every kernel is a programmatic dependent launch: its grid may become resident
// before the work ahead of it on the stream has ended, so a kernel reads and
// writes nothing before that work has completed (and its writes are visible),
// and then lets the launch after it become resident early in turn.  Only the
// launch latency is hidden; the order of the work is the stream's.
__device__ __forceinline__ void wait_for_prior_work() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
}

// ---------------------------------------------------------------- numerics

// 2^x by the hardware approximation (MUFU); 2^-inf = +0.
__device__ __forceinline__ float exp2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <typename T>
__device__ __forceinline__ T from_float(float x);
template <>
__device__ __forceinline__ float from_float<float>(float x) { return x; }
template <>
__device__ __forceinline__ __half from_float<__half>(float x) { return __float2half_rn(x); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Softmax exponent in the domain the scores are kept in: natural (fp32 path,
// accurate expf) or base 2 with the scale pre-multiplied by log2(e) (16-bit
// path, hardware ex2).
template <bool LOG2>
__device__ __forceinline__ float softmax_exp(float x) {
    if constexpr (LOG2) {
        return exp2_approx(x);
    } else {
        return expf(x);
    }
}

constexpr float kNegInf = -INFINITY;

// ---------------------------------------------------------------- shared-prefix decode

// A context of L tokens cannot take the shared-prefix form when it does not
// reach past the prefix_len shared tokens, or, appending, when its newest
// token (position L - 1) would land in a shared block.
__device__ __forceinline__ bool shared_prefix_refused(int L, int prefix_len, bool append) {
    return L < prefix_len + (append ? 1 : 0);
}

// The last step of the shared-prefix decode: the np partials of a query head
// row of (sequence, kv head) -- the prefix pass's key partitions and the
// sequence's own blocks; unnormalised output, reference maximum (base 2) and
// sum, [S][Hq][np][D] and [S][Hq][np][2] -- combined with log-sum-exp weights
// 2^(m_i - max_i m_i) into four output values (16-byte chunk c of the row;
// zero where `zero`).  U such outputs at once, four partials each step, so
// that their loads are in flight together; the partials were written by other
// CTAs, so they are read past L1.
template <typename T, int D, int U>
__device__ __forceinline__ void merge_shared_prefix(void* out, const float* part_acc, const float* part_ml, int np,
                                                    const long long (&row)[U], const int (&c)[U],
                                                    const bool (&use)[U], const bool (&zero)[U]) {
    constexpr int kStep = 4;
    float4 a[U];
    float M[U], den[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        a[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        M[u] = kNegInf;
        den[u] = 0.f;
    }
    for (int q0 = 0; q0 < np; q0 += kStep) {
        float m[U][kStep], l[U][kStep];
        float4 x[U][kStep];
#pragma unroll
        for (int u = 0; u < U; ++u) {
#pragma unroll
            for (int k = 0; k < kStep; ++k) {
                const bool in = use[u] && q0 + k < np;
                const long long sl = row[u] * np + q0 + k;
                m[u][k] = in ? __ldcg(part_ml + sl * 2) : kNegInf;
                l[u][k] = in ? __ldcg(part_ml + sl * 2 + 1) : 0.f;
                x[u][k] = in ? __ldcg(reinterpret_cast<const float4*>(part_acc + sl * D) + c[u])
                             : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
#pragma unroll
            for (int k = 0; k < kStep; ++k) {
                const float mn = fmaxf(M[u], m[u][k]);
                if (mn != kNegInf) {
                    const float sa = exp2_approx(M[u] - mn), sb = exp2_approx(m[u][k] - mn);
                    a[u].x = fmaf(a[u].x, sa, x[u][k].x * sb);
                    a[u].y = fmaf(a[u].y, sa, x[u][k].y * sb);
                    a[u].z = fmaf(a[u].z, sa, x[u][k].z * sb);
                    a[u].w = fmaf(a[u].w, sa, x[u][k].w * sb);
                    den[u] = fmaf(den[u], sa, l[u][k] * sb);
                    M[u] = mn;
                }
            }
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        if (!use[u]) continue;
        const float inv = (!zero[u] && den[u] > 0.f) ? 1.f / den[u] : 0.f;
        T* dst = reinterpret_cast<T*>(out) + row[u] * D + 4 * c[u];
        dst[0] = from_float<T>(a[u].x * inv);
        dst[1] = from_float<T>(a[u].y * inv);
        dst[2] = from_float<T>(a[u].z * inv);
        dst[3] = from_float<T>(a[u].w * inv);
    }
}

}  // namespace pa
