// Host side of the C ABI declared in include/pa.h: argument validation,
// kernel-variant dispatch on (dtype, head_dim, block_size), launches.
// Nothing here allocates device memory or synchronises, except
// pa_get_device_error which synchronises the given stream by contract.

#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>

#include "pa.h"
#include "pa_decode.cuh"
#include "pa_reshape.cuh"

// Per-warp shared-memory ring size and warps per CTA of the decode kernel.
#ifndef PA_DECODE_WARPS
#define PA_DECODE_WARPS 4
#endif
#ifndef PA_RING_BYTES_PER_WARP
#define PA_RING_BYTES_PER_WARP 32768
#endif

namespace {

template <typename T, int D, int B>
struct DecodeConfig {
    static constexpr int kStageBytes = 2 * B * D * static_cast<int>(sizeof(T));  // K + V tile
    static constexpr int kRingCap = 200 * 1024;                                   // ring bytes per CTA at most
    static constexpr int kMaxWarps = kRingCap / kStageBytes;
    static constexpr int kWarps = PA_DECODE_WARPS < kMaxWarps ? PA_DECODE_WARPS : kMaxWarps;
    static constexpr int kRaw = PA_RING_BYTES_PER_WARP / kStageBytes;
    static constexpr int kFit = kRingCap / (kWarps * kStageBytes);
    static constexpr int kStages0 = kRaw < 1 ? 1 : (kRaw > 16 ? 16 : kRaw);
    static constexpr int kStages = kStages0 < kFit ? kStages0 : kFit;
    using Smem = pa::DecodeSmem<T, D, B, kWarps, kStages>;
    static_assert(Smem::kTotal <= 227 * 1024, "shared memory per CTA");
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int elem_size(pa_dtype dt) { return dt == PA_F32 ? 4 : 2; }

bool dtype_ok(int dt) { return dt == PA_F32 || dt == PA_F16 || dt == PA_BF16; }

// Raises the dynamic shared-memory limit of one kernel once per device.
template <typename Kernel>
cudaError_t ensure_smem(Kernel kernel, int bytes, std::atomic<uint64_t>& done_mask) {
    if (bytes <= 48 * 1024) return cudaSuccess;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
    if (bit && (done_mask.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done_mask.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

template <typename T, int D, int B, bool SPLIT>
cudaError_t launch_decode(const pa::DecodeParams& p, dim3 grid, cudaStream_t stream) {
    using C = DecodeConfig<T, D, B>;
    auto kernel = pa::pa_decode_kernel<T, D, B, C::kWarps, C::kStages, SPLIT>;
    static std::atomic<uint64_t> done{0};
    cudaError_t e = ensure_smem(kernel, C::Smem::kTotal, done);
    if (e != cudaSuccess) return e;
    kernel<<<grid, C::kWarps * 32, C::Smem::kTotal, stream>>>(p);
    return cudaGetLastError();
}

template <typename T, int D, bool SPLIT>
cudaError_t decode_by_block(int B, const pa::DecodeParams& p, dim3 grid, cudaStream_t st) {
    switch (B) {
        case 8: return launch_decode<T, D, 8, SPLIT>(p, grid, st);
        case 16: return launch_decode<T, D, 16, SPLIT>(p, grid, st);
        case 32: return launch_decode<T, D, 32, SPLIT>(p, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T, bool SPLIT>
cudaError_t decode_by_dim(int D, int B, const pa::DecodeParams& p, dim3 grid, cudaStream_t st) {
    switch (D) {
        case 64: return decode_by_block<T, 64, SPLIT>(B, p, grid, st);
        case 128: return decode_by_block<T, 128, SPLIT>(B, p, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

template <bool SPLIT>
cudaError_t decode_dispatch(pa_dtype dt, int D, int B, const pa::DecodeParams& p, dim3 grid, cudaStream_t st) {
    switch (dt) {
        case PA_F32: return decode_by_dim<float, SPLIT>(D, B, p, grid, st);
        case PA_F16: return decode_by_dim<__half, SPLIT>(D, B, p, grid, st);
        case PA_BF16: return decode_by_dim<__nv_bfloat16, SPLIT>(D, B, p, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T, int D>
cudaError_t launch_merge(const pa::MergeParams& p, cudaStream_t st) {
    constexpr bool kLog2 = !pa::IsF32<T>::value;
    const long long warps = static_cast<long long>(p.num_seqs) * p.num_q_heads;
    const unsigned blocks = static_cast<unsigned>((warps + 3) / 4);
    pa::pa_merge_kernel<T, D, kLog2><<<blocks, 128, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t merge_dispatch(pa_dtype dt, int D, const pa::MergeParams& p, cudaStream_t st) {
    if (D == 64) {
        if (dt == PA_F32) return launch_merge<float, 64>(p, st);
        if (dt == PA_F16) return launch_merge<__half, 64>(p, st);
        return launch_merge<__nv_bfloat16, 64>(p, st);
    }
    if (dt == PA_F32) return launch_merge<float, 128>(p, st);
    if (dt == PA_F16) return launch_merge<__half, 128>(p, st);
    return launch_merge<__nv_bfloat16, 128>(p, st);
}

struct DecodeShape {
    int block_size, num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, max_context_len;
    long long num_blocks;
    int dtype;
};

pa_status check_decode(const void* out, const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* block_tables, const int32_t* context_lens, float scale,
                       const DecodeShape& sh) {
    if (sh.num_seqs < 0 || sh.num_q_heads <= 0 || sh.num_kv_heads <= 0 || sh.head_dim <= 0 ||
        sh.block_size <= 0 || sh.max_blocks_per_seq < 0 || sh.max_context_len < 0 || sh.num_blocks <= 0)
        return PA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
    if (!dtype_ok(sh.dtype)) return PA_ERR_UNSUPPORTED;
    if (sh.head_dim != 64 && sh.head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (sh.block_size != 8 && sh.block_size != 16 && sh.block_size != 32) return PA_ERR_UNSUPPORTED;
    if (sh.num_q_heads % sh.num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    const int g = sh.num_q_heads / sh.num_kv_heads;
    if (g != 1 && g != 2 && g != 4 && g != 8) return PA_ERR_UNSUPPORTED;
    if (sh.num_seqs > 65535 || sh.num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;  // grid limits
    if (sh.num_seqs == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned4(block_tables) || !aligned4(context_lens))
        return PA_ERR_INVALID_ARG;
    return PA_OK;
}

int context_cap(const DecodeShape& sh) {
    const long long by_table = static_cast<long long>(sh.max_blocks_per_seq) * sh.block_size;
    const long long cap = by_table < sh.max_context_len ? by_table : sh.max_context_len;
    return cap > INT_MAX ? INT_MAX : static_cast<int>(cap);
}

pa::DecodeParams make_params(void* out, const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, const int32_t* context_lens, float scale,
                             const DecodeShape& sh) {
    pa::DecodeParams p{};
    p.out = out;
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    // 16-bit path keeps scores in base 2: fold log2(e) into the scale.
    p.score_scale = sh.dtype == PA_F32 ? scale : scale * 1.4426950408889634f;
    p.num_seqs = sh.num_seqs;
    p.num_q_heads = sh.num_q_heads;
    p.num_kv_heads = sh.num_kv_heads;
    p.group = sh.num_q_heads / sh.num_kv_heads;
    p.max_blocks_per_seq = sh.max_blocks_per_seq;
    p.context_cap = context_cap(sh);
    p.num_blocks = sh.num_blocks;
    return p;
}

size_t splitk_bytes(long long seqs, long long heads, long long parts, long long head_dim) {
    return static_cast<size_t>(seqs * heads * parts * (head_dim + 2) * 4);
}

}  // namespace

extern "C" {

pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                               const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads,
                               int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype,
                               void* stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return PA_ERR_INVALID_ARG;
    if (!dtype_ok(dtype)) return PA_ERR_UNSUPPORTED;
    const int row_bytes = head_dim * elem_size(dtype);
    if (row_bytes % 16 != 0) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
        return PA_ERR_INVALID_ARG;
    pa::ReshapeParams p{};
    p.key = static_cast<const uint4*>(key);
    p.value = static_cast<const uint4*>(value);
    p.k_cache = static_cast<uint4*>(k_cache);
    p.v_cache = static_cast<uint4*>(v_cache);
    p.slot_mapping = slot_mapping;
    p.num_tokens = num_tokens;
    p.num_kv_heads = num_kv_heads;
    p.vecs_per_row = row_bytes / 16;
    p.block_size = block_size;
    p.num_slots = num_blocks * static_cast<long long>(block_size);
    const long long threads = num_tokens * num_kv_heads * static_cast<long long>(p.vecs_per_row);
    const long long blocks = (threads + 255) / 256;
    if (blocks > INT_MAX) return PA_ERR_UNSUPPORTED;
    pa::pa_reshape_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, const int32_t* context_lens, float scale, int block_size,
                    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                    int max_context_len, int64_t num_blocks, pa_dtype dtype, void* stream) {
    const DecodeShape sh{block_size, num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                         max_context_len, num_blocks, static_cast<int>(dtype)};
    pa_status st = check_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh);
    if (st != PA_OK || num_seqs == 0) return st;
    const pa::DecodeParams p = make_params(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh);
    const dim3 grid(1, num_kv_heads, num_seqs);
    const cudaError_t e = decode_dispatch<false>(dtype, head_dim, block_size, p, grid,
                                                 static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_decode_splitk_workspace_size(int num_seqs, int num_q_heads, int head_dim, int max_context_len,
                                          int partition_size, size_t* bytes) {
    if (!bytes || num_seqs < 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len < 0 ||
        partition_size <= 0)
        return PA_ERR_INVALID_ARG;
    const long long parts = (static_cast<long long>(max_context_len) + partition_size - 1) / partition_size;
    *bytes = splitk_bytes(num_seqs, num_q_heads, parts, head_dim);
    return PA_OK;
}

pa_status pa_decode_splitk(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens, float scale,
                           int block_size, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                           int max_blocks_per_seq, int max_context_len, int64_t num_blocks, pa_dtype dtype,
                           int partition_size, void* workspace, size_t workspace_bytes, void* stream) {
    const DecodeShape sh{block_size, num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                         max_context_len, num_blocks, static_cast<int>(dtype)};
    pa_status st = check_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh);
    if (st != PA_OK) return st;
    if (partition_size <= 0 || partition_size % 16 != 0 || partition_size % block_size != 0)
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    pa::DecodeParams p = make_params(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh);
    const int pb = partition_size / block_size;
    const long long cap_blocks = (static_cast<long long>(p.context_cap) + block_size - 1) / block_size;
    const long long parts = (cap_blocks + pb - 1) / pb;
    if (parts > INT_MAX) return PA_ERR_UNSUPPORTED;
    const size_t need = splitk_bytes(num_seqs, num_q_heads, parts, head_dim);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return PA_ERR_WORKSPACE;
    float* acc = static_cast<float*>(workspace);
    p.part_acc = acc;
    p.part_ml = acc + static_cast<size_t>(num_seqs) * num_q_heads * parts * head_dim;
    p.partition_blocks = pb;
    p.num_partitions = static_cast<int>(parts);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (parts > 0) {
        const dim3 grid(static_cast<unsigned>(parts), num_kv_heads, num_seqs);
        const cudaError_t e = decode_dispatch<true>(dtype, head_dim, block_size, p, grid, s);
        if (e != cudaSuccess) return PA_ERR_CUDA;
    }
    pa::MergeParams m{};
    m.out = out;
    m.part_acc = p.part_acc;
    m.part_ml = p.part_ml;
    m.context_lens = context_lens;
    m.num_seqs = num_seqs;
    m.num_q_heads = num_q_heads;
    m.context_cap = p.context_cap;
    m.block_size = block_size;
    m.partition_blocks = pb;
    m.num_partitions = static_cast<int>(parts);
    return merge_dispatch(dtype, head_dim, m, s) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_get_device_error(void* stream, int32_t* code) {
    if (!code) return PA_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PA_ERR_CUDA;
    int value = 0;
    if (cudaMemcpyFromSymbol(&value, pa::g_device_error, sizeof(int)) != cudaSuccess) return PA_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(pa::g_device_error, &zero, sizeof(int)) != cudaSuccess) return PA_ERR_CUDA;
    *code = value;
    return PA_OK;
}

const char* pa_status_string(pa_status status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
        case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
        case PA_ERR_CUDA: return "PA_ERR_CUDA";
        default: return "PA_UNKNOWN_STATUS";
    }
}

}  // extern "C"
