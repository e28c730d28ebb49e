// Host side of the C ABI declared in include/pa.h: argument validation,
// kernel-variant dispatch on (dtype, head_dim, block_size), launches.
// Nothing here allocates device memory or synchronises, except
// pa_get_device_error which synchronises the given stream by contract.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <utility>
#include <map>
#include <mutex>
#include <tuple>

#include "pa.h"
#include "pa_blocks.cuh"
#include "pa_copy.cuh"
#include "pa_decode.cuh"
#include "pa_prefill.cuh"
#include "pa_prefill_tc.cuh"
#include "pa_reshape.cuh"

// Two CTA shapes for the decode kernels, measured on B200 over the benchmark
// workloads (warps per CTA, shared-memory ring bytes per warp):
//  * deep: one large CTA per SM with a two-stage ring per warp; best when the
//    grid is at most PA_DEEP_MAX_CTAS_PER_SM CTAs per SM (few, long
//    sequences per SM), where each CTA streams long enough to amortise its
//    start-up;
//  * wide: small CTAs, several resident per SM, so one CTA's start-up
//    (block-table read, first copies) and final merge overlap other CTAs'
//    streaming; best for grids of many short CTAs (split-K partitions,
//    batches of short sequences).
// (12 warps: with the launches made early, the Llama-3-8B step 48.0 -> 46.9
// us against 8 warps; 10 and 11 warps lie between)
#ifndef PA_DEEP_WARPS
#define PA_DEEP_WARPS 12
#endif
#ifndef PA_DEEP_RING
#define PA_DEEP_RING 16384
#endif
#ifndef PA_WIDE_WARPS
#define PA_WIDE_WARPS 4
#endif
#ifndef PA_WIDE_RING
#define PA_WIDE_RING 12288
#endif
// The same two shapes for 8-bit pools, whose blocks carry half the bytes
// for the same tensor-core work per block.
// (12 warps: with the launches made early, the Llama-3-8B decode over 8-bit pools
// 39.8 -> 38.9 us against 16 warps, the appending step 40.2 -> 40.1 us)
#ifndef PA_FP8_DEEP_WARPS
#define PA_FP8_DEEP_WARPS 12
#endif
#ifndef PA_FP8_DEEP_RING
#define PA_FP8_DEEP_RING 12288
#endif
#ifndef PA_FP8_WIDE_WARPS
#define PA_FP8_WIDE_WARPS 4
#endif
#ifndef PA_FP8_WIDE_RING
#define PA_FP8_WIDE_RING 8192
#endif
// Shared-prefix decode: the decode pass overlaps the prefix pass (1), or
// starts after it (0).  The prefix pass takes about this many CTAs (0: a
// third of the SMs; the decode pass fills the rest meanwhile): on the
// 128-sequence, 1024-token-prefix workload 48 of 148 (3 key partitions) ran
// 38.2 us, 32 39.4, 16 55.5, 64 41.3 and 148 51.3.
#ifndef PA_PREFIX_OVERLAP
#define PA_PREFIX_OVERLAP 1
#endif
// Launches may become resident before the work ahead of them ends (1), or
// not (0).  On steps launched back to back: Llama-3-8B decode 49.2 -> 47.4 us,
// the mix at 16-token blocks 38.0 -> 36.2 us, the shared-prefix step 37.4 ->
// 35.4 us, a step through the device block manager (three launches) 63.1 ->
// 57.2 us.
#ifndef PA_EARLY_LAUNCH
#define PA_EARLY_LAUNCH 1
#endif
#ifndef PA_PREFIX_CTAS
#define PA_PREFIX_CTAS 0
#endif
// ... and the decode pass's wide grid starts the sequences whose own part is
// in the upper (8 - N) / 8 of its range first (0: one class; 4 ran 40.3 us
// there against 47.3 us for one class).
#ifndef PA_PREFIX_CLASS_EIGHTHS
#define PA_PREFIX_CLASS_EIGHTHS 4
#endif

#ifndef PA_TWO_CLASS
#define PA_TWO_CLASS 1
#endif
#ifndef PA_DEEP_MAX_CTAS_PER_SM
#define PA_DEEP_MAX_CTAS_PER_SM 4
#endif

namespace {

enum class Kind { kDeep, kWide };

template <Kind K, bool FP8>
struct KindTuning;
// kRingCap bounds the K/V ring of a CTA.
template <>
struct KindTuning<Kind::kDeep, false> {
    static constexpr int kWarps = PA_DEEP_WARPS, kRing = PA_DEEP_RING, kRingCap = 200 * 1024;
};
template <>
struct KindTuning<Kind::kWide, false> {
    static constexpr int kWarps = PA_WIDE_WARPS, kRing = PA_WIDE_RING, kRingCap = 200 * 1024;
};
template <>
struct KindTuning<Kind::kDeep, true> {
    static constexpr int kWarps = PA_FP8_DEEP_WARPS, kRing = PA_FP8_DEEP_RING, kRingCap = 200 * 1024;
};
template <>
struct KindTuning<Kind::kWide, true> {
    static constexpr int kWarps = PA_FP8_WIDE_WARPS, kRing = PA_FP8_WIDE_RING, kRingCap = 200 * 1024;
};


// 16-bit pools of 32-token blocks take wide CTAs of this many warps (one 16
// KiB stage each): on the continuous-batching mix two warps per CTA with the
// long sequences started first ran 40.1 us, four warps 41.7 us (and 43.2 with
// the long sequences first), three 41.2, one 54.4.
#ifndef PA_WIDE32_WARPS
#define PA_WIDE32_WARPS 2
#endif

// FP8: the pools hold 1-byte e4m3 codes, so a stage is half the size of a
// 16-bit one and the same ring bytes hold twice the stages.
template <typename T, int D, int B, Kind K, bool FP8 = false>
struct DecodeConfig {
    static constexpr int kElem = FP8 ? 1 : static_cast<int>(sizeof(T));
    static constexpr int kStageBytes = 2 * B * D * kElem;                       // K + V tile
    static constexpr int kRingCap = KindTuning<K, FP8>::kRingCap;                    // ring bytes per CTA at most
    static constexpr int kMaxWarps = kRingCap / kStageBytes;
    static constexpr int kWarpsWanted =
        (K == Kind::kWide && !FP8 && B == 32 && sizeof(T) == 2) ? PA_WIDE32_WARPS : KindTuning<K, FP8>::kWarps;
    static constexpr int kWarps = kWarpsWanted < kMaxWarps ? kWarpsWanted : kMaxWarps;
    static constexpr int kRaw = KindTuning<K, FP8>::kRing / kStageBytes;
    static constexpr int kFit = kRingCap / (kWarps * kStageBytes);
    static constexpr int kStages0 = kRaw < 1 ? 1 : (kRaw > 16 ? 16 : kRaw);
    static constexpr int kStages = kStages0 < kFit ? kStages0 : kFit;
    using Smem = pa::DecodeSmem<T, D, B, kWarps, kStages, FP8>;
    static_assert(kStages >= 1, "one stage per warp at least");
    static_assert(Smem::kTotal <= 227 * 1024, "shared memory per CTA");
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int elem_size(pa_dtype dt) { return dt == PA_F32 ? 4 : 2; }

bool dtype_ok(int dt) { return dt == PA_F32 || dt == PA_F16 || dt == PA_BF16; }

// Raises the dynamic shared-memory limit of `kernel` on the current device to
// the device's opt-in maximum, once per (kernel, device).  Setting it to the
// largest value (rather than to one launch's size) keeps every later launch
// of any size within the limit.
cudaError_t ensure_smem(const void* kernel) {
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, bool> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({kernel, dev})) return cudaSuccess;
    int optin = 0;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes attr{};
    e = cudaFuncGetAttributes(&attr, kernel);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - static_cast<int>(attr.sharedSizeBytes));
    if (e == cudaSuccess) done[{kernel, dev}] = true;
    return e;
}

// Every launch is a programmatic dependent launch (each kernel first waits
// for the work ahead of it on the stream, see wait_for_prior_work): a grid
// may take its places on the SMs before that work ends, which hides the
// launch latency between the library's launches.
template <typename... KArgs, typename... Args>
cudaError_t launch_early(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                         int early, Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = early;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename T>
struct TypeTag {
    using type = T;
};
template <int V>
struct IntTag {
    static constexpr int value = V;
};

// Calls f(TypeTag<T>, IntTag<D>, IntTag<B>) for the kernel variant of
// (dtype, head_dim, block_size); the shape has been validated already.
template <typename F>
cudaError_t with_variant(pa_dtype dt, int D, int B, F&& f) {
    auto by_block = [&](auto tt, auto dd) -> cudaError_t {
        switch (B) {
            case 8: return f(tt, dd, IntTag<8>{});
            case 16: return f(tt, dd, IntTag<16>{});
            case 32: return f(tt, dd, IntTag<32>{});
            default: return cudaErrorInvalidValue;
        }
    };
    auto by_dim = [&](auto tt) -> cudaError_t {
        switch (D) {
            case 64: return by_block(tt, IntTag<64>{});
            case 128: return by_block(tt, IntTag<128>{});
            default: return cudaErrorInvalidValue;
        }
    };
    switch (dt) {
        case PA_F32: return by_dim(TypeTag<float>{});
        case PA_F16: return by_dim(TypeTag<__half>{});
        case PA_BF16: return by_dim(TypeTag<__nv_bfloat16>{});
        default: return cudaErrorInvalidValue;
    }
}

template <typename T, int D, int B, bool SPLIT, Kind K, bool FP8 = false, bool PREFIX = false>
cudaError_t launch_decode(const pa::DecodeParams& p, dim3 grid, cudaStream_t stream) {
    using C = DecodeConfig<T, D, B, K, FP8>;
    auto kernel = pa::pa_decode_kernel<T, D, B, C::kWarps, C::kStages, SPLIT, FP8,
                                       !SPLIT && (!PREFIX || PA_PREFIX_CLASS_EIGHTHS > 0) && K == Kind::kWide,
                                       PREFIX>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kernel));
    if (e != cudaSuccess) return e;
    // The shared-prefix form's CTAs start while the prefix pass (the launch
    // before, on the same stream) still runs: the two grids meet only through
    // the arrival counters, and one CTA waits for the prefix pass to complete
    // (so that this grid ends after it).
    return launch_early(kernel, grid, dim3(C::kWarps * 32), C::Smem::kTotal, stream,
                        PREFIX ? PA_PREFIX_OVERLAP : PA_EARLY_LAUNCH, p);
}

// Streaming multiprocessors of the current device, once per device.
int sm_count() {
    static std::mutex mu;
    static std::map<int, int> counts;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    auto it = counts.find(dev);
    if (it != counts.end()) return it->second;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return counts[dev] = n;
}

// The split kernel always runs wide CTAs; the one-pass kernel runs deep CTAs
// unless its grid holds more than PA_DEEP_MAX_CTAS_PER_SM CTAs per SM.
template <bool SPLIT, bool FP8 = false, bool PREFIX = false>
cudaError_t decode_dispatch(pa_dtype dt, int D, int B, const pa::DecodeParams& p, dim3 grid, cudaStream_t st) {
    const long long ctas = static_cast<long long>(grid.x) * grid.y * grid.z;
    const bool deep = !SPLIT && ctas <= static_cast<long long>(PA_DEEP_MAX_CTAS_PER_SM) * sm_count();
    return with_variant(dt, D, B, [&](auto tt, auto dd, auto bb) -> cudaError_t {
        using T = typename decltype(tt)::type;
        constexpr int kD = decltype(dd)::value, kB = decltype(bb)::value;
        if constexpr ((FP8 || PREFIX) && pa::IsF32<T>::value) {
            return cudaErrorInvalidValue;  // 16-bit only (refused on the host first)
        } else if constexpr (PREFIX) {
            return deep ? launch_decode<T, kD, kB, false, Kind::kDeep, false, true>(p, grid, st)
                        : launch_decode<T, kD, kB, false, Kind::kWide, false, true>(p, grid, st);
        } else if constexpr (SPLIT) {
            return launch_decode<T, kD, kB, true, Kind::kWide, FP8>(p, grid, st);
        } else {
            return deep ? launch_decode<T, kD, kB, false, Kind::kDeep, FP8>(p, grid, st)
                        : launch_decode<T, kD, kB, false, Kind::kWide, FP8>(p, grid, st);
        }
    });
}

// A one-pass launch of many small CTAs (the wide shape) without a start
// order from the host starts the long sequences first by running the grid
// twice over: the first half takes the sequences of at least a quarter of
// max_context_len tokens, the second half the others (CTAs start roughly in
// blockIdx order; a CTA of the other class leaves at once).
dim3 two_class_grid(pa::DecodeParams& p, dim3 grid, int max_context_len, int block_size, int threshold = -1) {
    const long long ctas = static_cast<long long>(grid.x) * grid.y * grid.z;
    const bool wide = ctas > static_cast<long long>(PA_DEEP_MAX_CTAS_PER_SM) * sm_count();
    if (threshold < 0) threshold = PA_TWO_CLASS && max_context_len >= 4 ? max_context_len / 4 : 0;
    if (threshold <= 0 || !wide || p.seq_order != nullptr || 2LL * grid.z > 65535)
        return grid;
    p.class_threshold = threshold;
    grid.z *= 2;
    return grid;
}

template <typename T, int D>
cudaError_t launch_merge(const pa::MergeParams& p, cudaStream_t st) {
    constexpr bool kLog2 = !pa::IsF32<T>::value;
    const long long warps = static_cast<long long>(p.num_seqs) * p.num_q_heads;
    const unsigned blocks = static_cast<unsigned>((warps + 3) / 4);
    return launch_early(pa::pa_merge_kernel<T, D, kLog2>, dim3(blocks), dim3(128), 0, st, PA_EARLY_LAUNCH, p);
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

// 64-key tiles of a shared prefix of prefix_blocks blocks: the most key
// partitions the prefix pass can take.
int shared_prefix_tiles(int prefix_blocks, int block_size) {
    return static_cast<int>((static_cast<long long>(prefix_blocks) * block_size + 63) / 64);
}

// Device memory, or page-locked host memory mapped into the device's address
// space (what the copy kernel can dereference).
bool device_accessible(const void* p) {
    cudaPointerAttributes attr{};
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();  // the failed query leaves an error behind; clear it
        return false;
    }
    if (attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged) return true;
    return attr.type == cudaMemoryTypeHost && attr.devicePointer == p;
}

// Chunked prefill: 4 warps (64 MMA rows) per CTA, a 4-stage block ring.
constexpr int kPrefillWarps = 4;
constexpr int kPrefillStages = 4;

// Blocks of 8, 16 or 32 tokens run the 5th-generation tensor-core kernel (two
// query tiles of 128 MMA rows per CTA); PA_PREFILL_TC=0 or a K pool that no
// tensor map can describe run the warp-level one.
#ifndef PA_PREFILL_TC
#define PA_PREFILL_TC 1
#endif

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (the library links no driver library); null where there is no driver.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    return fn;
}

// The K pool viewed as a 2-D tensor of rows (block, kv head, 8-dim chunk), each
// row the chunk's B tokens x 8 elements (B * 16 bytes), one row per box: the
// operand of the prefill kernel's gather4 loads.  False when it cannot be
// described (no driver, or more rows than a 32-bit coordinate reaches).
bool encode_k_rows(CUtensorMap* map, const void* k_cache, pa_dtype dt, int B, int D, int Hkv, long long num_blocks) {
    const PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (!encode) return false;
    const long long rows = num_blocks * Hkv * (D / 8);
    if (rows <= 0 || rows > INT_MAX) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(B) * 8, static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(B) * 16};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(B) * 8, 1};
    const cuuint32_t elem_strides[2] = {1, 1};
    const CUtensorMapDataType type =
        dt == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    return encode(map, type, 2, const_cast<void*>(k_cache), dims, strides, box, elem_strides,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tensor-core kernel's K operand: blocks of 8 tokens are bulk-copied
// whole and need no tensor map; larger blocks are gathered through one.
bool prefill_k_source(CUtensorMap* map, const void* k_cache, pa_dtype dt, int B, int D, int Hkv,
                      long long num_blocks) {
    return B == 8 || encode_k_rows(map, k_cache, dt, B, D, Hkv, num_blocks);
}

// Query tiles (of 128 MMA rows) per tensor-core prefill CTA: 2 (one CTA per
// SM, the two tiles sharing every K/V tile) or 1 (two CTAs per SM, each with
// its own K/V stream).  On the chunked-prefill workload one tile per CTA ran
// 197.4 against 208.6 us at 32-token blocks, but 228.0 against 221.1 at 16 and
// 273.2 against 236.6 at 8 (twice the copies per SM), and the shared-prefix
// step 44.3 against 36.1 us; so 32-token blocks take one (PA_PF_QT32).
#ifndef PA_PF_QT32
#define PA_PF_QT32 1
#endif
constexpr int prefill_tiles_per_cta(int block_size, bool prefix) {
    return (block_size == 32 && !prefix) ? PA_PF_QT32 : 2;
}

template <typename T, int D, int B, bool PREFIX = false>
cudaError_t launch_prefill_tc(const pa::PrefillParams& p, const CUtensorMap& k_rows, dim3 grid, cudaStream_t st) {
    constexpr int kQT = prefill_tiles_per_cta(B, PREFIX);
    using Sm = pa::PrefillTcSmem<T, D, B, kQT>;
    auto kernel = pa::pa_prefill_tc_kernel<T, D, B, PREFIX, kQT>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kernel));
    if (e != cudaSuccess) return e;
    return launch_early(kernel, grid, dim3((6 * kQT + 2) * 32), Sm::kTotal, st, PA_EARLY_LAUNCH, p, k_rows);
}

template <typename T, int D, int B>
cudaError_t launch_prefill(const pa::PrefillParams& p, dim3 grid, cudaStream_t st) {
    using Sm = pa::PrefillSmem<T, D, B, kPrefillWarps, kPrefillStages>;
    auto kernel = pa::pa_prefill_kernel<T, D, B, kPrefillWarps, kPrefillStages>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kernel));
    if (e != cudaSuccess) return e;
    return launch_early(kernel, grid, dim3(kPrefillWarps * 32), Sm::kTotal, st, PA_EARLY_LAUNCH, p);
}

// The one-pass and split decode bodies, shared by the 16-bit-pool entries
// (FP8 = false) and the 8-bit-pool entries (FP8 = true, with K/V scales).
template <bool FP8>
pa_status check_scales(const DecodeShape& sh, const float* k_scale, const float* v_scale) {
    if constexpr (FP8) {
        if (sh.dtype == PA_F32) return PA_ERR_UNSUPPORTED;  // 8-bit pools take 16-bit queries
        if (sh.num_seqs > 0 && (!k_scale || !v_scale || !aligned4(k_scale) || !aligned4(v_scale)))
            return PA_ERR_INVALID_ARG;
    }
    return PA_OK;
}

template <bool FP8>
pa_status decode_one_pass(void* out, const void* q, const void* k_cache, const void* v_cache, const float* k_scale,
                          const float* v_scale, const int32_t* block_tables, const int32_t* context_lens,
                          float scale, const DecodeShape& sh, const int32_t* seq_order, void* stream,
                          const void* new_key = nullptr, const void* new_value = nullptr,
                          const int32_t* ref_counts = nullptr) {
    pa_status st = check_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh);
    if (st == PA_OK) st = check_scales<FP8>(sh, k_scale, v_scale);
    if (st != PA_OK || sh.num_seqs == 0) return st;
    if (!aligned4(seq_order)) return PA_ERR_INVALID_ARG;
    pa::DecodeParams p = make_params(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh);
    p.seq_order = seq_order;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.new_key = new_key;
    p.new_value = new_value;
    p.ref_counts = ref_counts;
    const dim3 grid = two_class_grid(p, dim3(1, sh.num_kv_heads, sh.num_seqs), sh.max_context_len, sh.block_size);
    const cudaError_t e = decode_dispatch<false, FP8>(static_cast<pa_dtype>(sh.dtype), sh.head_dim, sh.block_size,
                                                      p, grid, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <bool FP8>
pa_status decode_split(void* out, const void* q, const void* k_cache, const void* v_cache, const float* k_scale,
                       const float* v_scale, const int32_t* block_tables, const int32_t* context_lens, float scale,
                       const DecodeShape& sh, int partition_size, void* workspace, size_t workspace_bytes,
                       int32_t* counters, int64_t num_counters, const int32_t* seq_order, void* stream) {
    pa_status st = check_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh);
    if (st == PA_OK) st = check_scales<FP8>(sh, k_scale, v_scale);
    if (st != PA_OK) return st;
    const int block_size = sh.block_size, num_seqs = sh.num_seqs, num_q_heads = sh.num_q_heads;
    const int num_kv_heads = sh.num_kv_heads, head_dim = sh.head_dim;
    const pa_dtype dtype = static_cast<pa_dtype>(sh.dtype);
    if (partition_size <= 0 || partition_size % 16 != 0 || partition_size % block_size != 0)
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    if (!aligned4(seq_order)) return PA_ERR_INVALID_ARG;
    pa::DecodeParams p = make_params(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh);
    p.seq_order = seq_order;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
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
    if (counters != nullptr) {
        if (!aligned4(counters) || num_counters < static_cast<int64_t>(num_seqs) * num_kv_heads)
            return PA_ERR_WORKSPACE;
        p.counters = counters;
    }
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (parts > 0) {
        const dim3 grid(static_cast<unsigned>(parts), num_kv_heads, num_seqs);
        const cudaError_t e = decode_dispatch<true, FP8>(dtype, head_dim, block_size, p, grid, s);
        if (e != cudaSuccess) return PA_ERR_CUDA;
        if (counters != nullptr) return PA_OK;  // merged inside the partition kernel
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
    return launch_early(pa::pa_reshape_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                        static_cast<cudaStream_t>(stream), PA_EARLY_LAUNCH, p) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, const int32_t* context_lens, float scale, int block_size,
                    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                    int max_context_len, int64_t num_blocks, pa_dtype dtype, const int32_t* seq_order,
                    void* stream) {
    const DecodeShape sh{block_size, num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                         max_context_len, num_blocks, static_cast<int>(dtype)};
    return decode_one_pass<false>(out, q, k_cache, v_cache, nullptr, nullptr, block_tables, context_lens, scale, sh,
                                  seq_order, stream);
}

pa_status pa_decode_append(void* out, const void* q, const void* key, const void* value, void* k_cache, void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens, float scale, int block_size,
                           int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                           int max_context_len, int64_t num_blocks, pa_dtype dtype, const int32_t* ref_counts,
                           const int32_t* seq_order, void* stream) {
    const DecodeShape sh{block_size, num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                         max_context_len, num_blocks, static_cast<int>(dtype)};
    pa_status st = check_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh);
    if (st != PA_OK || num_seqs == 0) return st;
    if (!key || !value || !aligned16(key) || !aligned16(value)) return PA_ERR_INVALID_ARG;
    if (!aligned4(seq_order) || !aligned4(ref_counts)) return PA_ERR_INVALID_ARG;
    pa::DecodeParams p = make_params(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh);
    p.seq_order = seq_order;
    p.new_key = key;
    p.new_value = value;
    p.ref_counts = ref_counts;
    const dim3 grid = two_class_grid(p, dim3(1, num_kv_heads, num_seqs), max_context_len, block_size);
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
                           int partition_size, void* workspace, size_t workspace_bytes, int32_t* counters,
                           int64_t num_counters, const int32_t* seq_order, void* stream) {
    const DecodeShape sh{block_size, num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                         max_context_len, num_blocks, static_cast<int>(dtype)};
    return decode_split<false>(out, q, k_cache, v_cache, nullptr, nullptr, block_tables, context_lens, scale, sh,
                               partition_size, workspace, workspace_bytes, counters, num_counters, seq_order,
                               stream);
}

pa_status pa_reshape_and_cache_fp8(const void* key, const void* value, void* k_cache, void* v_cache,
                                   const int64_t* slot_mapping, const float* k_scale, const float* v_scale,
                                   int64_t num_tokens, int num_kv_heads, int head_dim, int block_size,
                                   int64_t num_blocks, pa_dtype dtype, void* stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return PA_ERR_INVALID_ARG;
    if (!dtype_ok(dtype)) return PA_ERR_UNSUPPORTED;
    if (head_dim % 16 != 0) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping || !k_scale || !v_scale) return PA_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u) || !aligned4(k_scale) || !aligned4(v_scale))
        return PA_ERR_INVALID_ARG;
    if (block_size != 8 && block_size % 16 != 0) return PA_ERR_UNSUPPORTED;
    pa::ReshapeE4m3Params p{};
    p.key = key;
    p.value = value;
    p.k_cache = static_cast<uint32_t*>(k_cache);
    p.v_cache = static_cast<uint8_t*>(v_cache);
    p.slot_mapping = slot_mapping;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.num_tokens = num_tokens;
    p.num_kv_heads = num_kv_heads;
    p.head_dim = head_dim;
    p.block_size = block_size;
    p.num_slots = num_blocks * static_cast<long long>(block_size);
    const long long threads = num_tokens * num_kv_heads * static_cast<long long>(head_dim / 4);
    const long long blocks = (threads + 255) / 256;
    if (blocks > INT_MAX) return PA_ERR_UNSUPPORTED;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const unsigned g = static_cast<unsigned>(blocks);
    cudaError_t e;
    switch (dtype) {
        case PA_F32: e = launch_early(pa::pa_reshape_e4m3_kernel<float>, dim3(g), dim3(256), 0, st, PA_EARLY_LAUNCH, p); break;
        case PA_F16: e = launch_early(pa::pa_reshape_e4m3_kernel<__half>, dim3(g), dim3(256), 0, st, PA_EARLY_LAUNCH, p); break;
        default:
            e = launch_early(pa::pa_reshape_e4m3_kernel<__nv_bfloat16>, dim3(g), dim3(256), 0, st, PA_EARLY_LAUNCH, p);
            break;
    }
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache, const float* k_scale,
                        const float* v_scale, const int32_t* block_tables, const int32_t* context_lens, float scale,
                        int block_size, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                        int max_blocks_per_seq, int max_context_len, int64_t num_blocks, pa_dtype dtype,
                        const int32_t* seq_order, void* stream) {
    const DecodeShape sh{block_size, num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                         max_context_len, num_blocks, static_cast<int>(dtype)};
    return decode_one_pass<true>(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale, sh,
                                 seq_order, stream);
}

pa_status pa_decode_append_fp8(void* out, const void* q, const void* key, const void* value, void* k_cache,
                               void* v_cache, const float* k_scale, const float* v_scale, const int32_t* block_tables,
                               const int32_t* context_lens, float scale, int block_size, int num_seqs,
                               int num_q_heads, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                               int max_context_len, int64_t num_blocks, pa_dtype dtype,
                               const int32_t* ref_counts, const int32_t* seq_order, void* stream) {
    const DecodeShape sh{block_size, num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                         max_context_len, num_blocks, static_cast<int>(dtype)};
    if (num_seqs > 0 && (!key || !value || !aligned16(key) || !aligned16(value))) return PA_ERR_INVALID_ARG;
    if (!aligned4(ref_counts)) return PA_ERR_INVALID_ARG;
    return decode_one_pass<true>(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale, sh,
                                 seq_order, stream, key, value, ref_counts);
}

pa_status pa_decode_splitk_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const float* k_scale, const float* v_scale, const int32_t* block_tables,
                               const int32_t* context_lens, float scale, int block_size, int num_seqs,
                               int num_q_heads, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                               int max_context_len, int64_t num_blocks, pa_dtype dtype, int partition_size,
                               void* workspace, size_t workspace_bytes, int32_t* counters, int64_t num_counters,
                               const int32_t* seq_order, void* stream) {
    const DecodeShape sh{block_size, num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                         max_context_len, num_blocks, static_cast<int>(dtype)};
    return decode_split<true>(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale, sh,
                              partition_size, workspace, workspace_bytes, counters, num_counters, seq_order, stream);
}

pa_status pa_copy_blocks(void* dst_k_cache, void* dst_v_cache, const void* src_k_cache, const void* src_v_cache,
                         const int64_t* block_mapping, int64_t num_pairs, int num_kv_heads, int head_dim,
                         int block_size, int64_t src_num_blocks, int64_t dst_num_blocks, pa_dtype dtype,
                         void* stream) {
    if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || src_num_blocks <= 0 ||
        dst_num_blocks <= 0)
        return PA_ERR_INVALID_ARG;
    if (!dtype_ok(dtype)) return PA_ERR_UNSUPPORTED;
    const long long block_bytes =
        static_cast<long long>(num_kv_heads) * block_size * head_dim * elem_size(dtype);
    if ((static_cast<long long>(head_dim) * elem_size(dtype)) % 16 != 0) return PA_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PA_OK;
    if (!dst_k_cache || !dst_v_cache || !src_k_cache || !src_v_cache || !block_mapping) return PA_ERR_INVALID_ARG;
    if (!aligned16(dst_k_cache) || !aligned16(dst_v_cache) || !aligned16(src_k_cache) ||
        !aligned16(src_v_cache) || (reinterpret_cast<uintptr_t>(block_mapping) & 7u))
        return PA_ERR_INVALID_ARG;
    if (!device_accessible(dst_k_cache) || !device_accessible(dst_v_cache) || !device_accessible(src_k_cache) ||
        !device_accessible(src_v_cache) || !device_accessible(block_mapping))
        return PA_ERR_INVALID_ARG;
    pa::CopyParams p{};
    p.dst[0] = static_cast<uint4*>(dst_k_cache);
    p.dst[1] = static_cast<uint4*>(dst_v_cache);
    p.src[0] = static_cast<const uint4*>(src_k_cache);
    p.src[1] = static_cast<const uint4*>(src_v_cache);
    p.mapping = block_mapping;
    p.num_pairs = num_pairs;
    p.vecs_per_block = block_bytes / 16;
    p.src_blocks = src_num_blocks;
    p.dst_blocks = dst_num_blocks;
    p.chunks = static_cast<int>((p.vecs_per_block + pa::kChunkVecs - 1) / pa::kChunkVecs);
    const long long ctas = num_pairs * 2 * p.chunks;
    if (ctas > INT_MAX) return PA_ERR_UNSUPPORTED;
    return launch_early(pa::pa_copy_blocks_kernel, dim3(static_cast<unsigned>(ctas)), dim3(pa::kCopyThreads), 0,
                        static_cast<cudaStream_t>(stream), PA_EARLY_LAUNCH, p) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

pa_status pa_prefill(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                     const int32_t* context_lens, const int32_t* query_start, float scale, int block_size,
                     int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                     int max_context_len, int max_query_len, int64_t num_blocks, pa_dtype dtype, void* stream) {
    const DecodeShape sh{block_size, num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                         max_context_len, num_blocks, static_cast<int>(dtype)};
    pa_status st = check_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh);
    if (st != PA_OK) return st;
    if (dtype == PA_F32) return PA_ERR_UNSUPPORTED;  // the tensor-core path takes 16-bit inputs
    if (max_query_len < 0) return PA_ERR_INVALID_ARG;
    if (num_seqs == 0 || max_query_len == 0) return PA_OK;
    if (!query_start || !aligned4(query_start)) return PA_ERR_INVALID_ARG;
    pa::PrefillParams p{};
    p.out = out;
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.query_start = query_start;
    p.score_scale = scale * 1.4426950408889634f;
    p.num_seqs = num_seqs;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = num_q_heads / num_kv_heads;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.context_cap = context_cap(sh);
    p.num_blocks = num_blocks;
    CUtensorMap k_rows{};
    const bool use_tc = PA_PREFILL_TC &&
                        prefill_k_source(&k_rows, k_cache, dtype, block_size, head_dim, num_kv_heads, num_blocks);
    p.tile_tokens = (use_tc ? 128 : kPrefillWarps * 16) / p.group;
    // the tensor-core kernel takes one or two query tiles per CTA
    const long long per_cta =
        use_tc ? static_cast<long long>(prefill_tiles_per_cta(block_size, false)) * p.tile_tokens : p.tile_tokens;
    const long long tiles = (static_cast<long long>(max_query_len) + per_cta - 1) / per_cta;
    if (tiles > INT_MAX) return PA_ERR_UNSUPPORTED;
    const dim3 grid(static_cast<unsigned>(tiles), num_kv_heads, num_seqs);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e = with_variant(dtype, head_dim, block_size, [&](auto tt, auto dd, auto bb) -> cudaError_t {
        using T = typename decltype(tt)::type;
        constexpr int kD = decltype(dd)::value, kB = decltype(bb)::value;
        if constexpr (pa::IsF32<T>::value) {
            return cudaErrorInvalidValue;
        } else {
            return use_tc ? launch_prefill_tc<T, kD, kB>(p, k_rows, grid, s) : launch_prefill<T, kD, kB>(p, grid, s);
        }
    });
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_decode_shared_prefix_workspace_size(int num_seqs, int num_q_heads, int head_dim, int prefix_blocks,
                                                 int block_size, size_t* bytes) {
    if (!bytes || num_seqs < 0 || num_q_heads <= 0 || head_dim <= 0 || prefix_blocks <= 0 || block_size <= 0)
        return PA_ERR_INVALID_ARG;
    *bytes = splitk_bytes(num_seqs, num_q_heads, shared_prefix_tiles(prefix_blocks, block_size) + 1, head_dim);
    return PA_OK;
}

pa_status pa_decode_shared_prefix(void* out, const void* q, const void* key, const void* value, void* k_cache,
                                  void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
                                  float scale, int block_size, int num_seqs, int num_q_heads, int num_kv_heads,
                                  int head_dim, int max_blocks_per_seq, int max_context_len, int64_t num_blocks,
                                  pa_dtype dtype, int prefix_blocks, void* workspace, size_t workspace_bytes,
                                  int32_t* counters, int64_t num_counters, const int32_t* ref_counts,
                                  void* stream) {
    const DecodeShape sh{block_size, num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                         max_context_len, num_blocks, static_cast<int>(dtype)};
    pa_status st = check_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh);
    if (st != PA_OK) return st;
    if (dtype == PA_F32) return PA_ERR_UNSUPPORTED;  // the prefix pass runs on the tensor cores
    if (prefix_blocks <= 0 || prefix_blocks > max_blocks_per_seq ||
        static_cast<long long>(prefix_blocks) * block_size > max_context_len)
        return PA_ERR_INVALID_ARG;
    if ((key == nullptr) != (value == nullptr)) return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    if (key && (!aligned16(key) || !aligned16(value))) return PA_ERR_INVALID_ARG;
    if (!aligned4(ref_counts)) return PA_ERR_INVALID_ARG;
    const int tiles = shared_prefix_tiles(prefix_blocks, block_size);
    if (!workspace || !aligned16(workspace) ||
        workspace_bytes < splitk_bytes(num_seqs, num_q_heads, tiles + 1, head_dim))
        return PA_ERR_WORKSPACE;
    if (!counters || !aligned4(counters) || num_counters < static_cast<int64_t>(num_seqs) * num_kv_heads)
        return PA_ERR_WORKSPACE;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    CUtensorMap k_rows{};
    if (!PA_PREFILL_TC ||
        !prefill_k_source(&k_rows, k_cache, dtype, block_size, head_dim, num_kv_heads, num_blocks)) {
        // no tensor map for the prefix pass: the plain decode gives the same result
        pa::DecodeParams p = make_params(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh);
        p.new_key = key;
        p.new_value = value;
        p.ref_counts = ref_counts;
        const dim3 grid = two_class_grid(p, dim3(1, num_kv_heads, num_seqs), max_context_len, block_size);
        return decode_dispatch<false>(dtype, head_dim, block_size, p, grid, s) == cudaSuccess ? PA_OK
                                                                                               : PA_ERR_CUDA;
    }
    // Pass 1 (tensor cores): the prefix once per kv head for all sequences,
    // key partitions spread over the SMs, unnormalised partials to the workspace.
    const int group = num_q_heads / num_kv_heads;
    const int tile_tokens = 128 / group;
    const int qt = prefill_tiles_per_cta(block_size, true);
    const long long row_ctas = (static_cast<long long>(num_seqs) + qt * tile_tokens - 1) / (qt * tile_tokens);
    const long long per_part = row_ctas * num_kv_heads;
    long long want = (PA_PREFIX_CTAS > 0 ? PA_PREFIX_CTAS : sm_count() / 3) / per_part;
    want = want < 1 ? 1 : (want > tiles ? tiles : want);
    const int tiles_per = static_cast<int>((tiles + want - 1) / want);
    const int parts = (tiles + tiles_per - 1) / tiles_per;   // every partition holds >= 1 tile (<= tiles)
    const int slots = parts + 1;                               // + the sequence's own blocks
    float* acc = static_cast<float*>(workspace);
    float* ml = acc + static_cast<size_t>(num_seqs) * num_q_heads * slots * head_dim;
    pa::PrefillParams pp{};
    pp.out = out;
    pp.context_lens = context_lens;
    pp.counters = counters;
    pp.prefix_append = key != nullptr;
    pp.q = q;
    pp.k_cache = k_cache;
    pp.v_cache = v_cache;
    pp.block_tables = block_tables;
    pp.score_scale = scale * 1.4426950408889634f;
    pp.num_seqs = num_seqs;
    pp.num_q_heads = num_q_heads;
    pp.num_kv_heads = num_kv_heads;
    pp.group = group;
    pp.max_blocks_per_seq = max_blocks_per_seq;
    pp.context_cap = context_cap(sh);
    pp.num_blocks = num_blocks;
    pp.tile_tokens = tile_tokens;
    pp.part_acc = acc;
    pp.part_ml = ml;
    pp.num_partitions = slots;
    pp.prefix_len = prefix_blocks * block_size;
    pp.prefix_tiles = tiles_per;
    const dim3 pgrid(static_cast<unsigned>(row_ctas), num_kv_heads, parts);
    cudaError_t e = with_variant(dtype, head_dim, block_size, [&](auto tt, auto dd, auto bb) -> cudaError_t {
        using T = typename decltype(tt)::type;
        constexpr int kD = decltype(dd)::value, kB = decltype(bb)::value;
        if constexpr (pa::IsF32<T>::value) {
            return cudaErrorInvalidValue;
        } else {
            return launch_prefill_tc<T, kD, kB, true>(pp, k_rows, pgrid, s);
        }
    });
    if (e != cudaSuccess) return PA_ERR_CUDA;
    // Pass 2: each sequence's own blocks (and newest token), the prefix
    // partials folded into the same merge.
    pa::DecodeParams p = make_params(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh);
    p.new_key = key;
    p.new_value = value;
    p.ref_counts = ref_counts;
    p.part_acc = acc;
    p.part_ml = ml;
    p.first_block = prefix_blocks;
    p.num_partitions = slots;
    p.counters = counters;
    const int pre = prefix_blocks * block_size;
    const dim3 grid = two_class_grid(p, dim3(1, num_kv_heads, num_seqs), max_context_len, block_size,
                                     PA_PREFIX_CLASS_EIGHTHS > 0
                                         ? pre + static_cast<int>((static_cast<long long>(max_context_len - pre) *
                                                                   PA_PREFIX_CLASS_EIGHTHS) / 8)
                                         : 0);
    e = decode_dispatch<false, false, true>(dtype, head_dim, block_size, p, grid, s);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // extern "C"

// ---- block management (pa_blocks.cuh)

namespace {

bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

pa_status check_block_state(const int32_t* ref_counts, const int32_t* free_ids, const int64_t* free_state,
                            int64_t num_blocks) {
    if (num_blocks <= 0 || num_blocks > INT_MAX) return PA_ERR_INVALID_ARG;
    if (!ref_counts || !free_ids || !free_state) return PA_ERR_INVALID_ARG;
    if (!aligned4(ref_counts) || !aligned4(free_ids) || !aligned8(free_state)) return PA_ERR_INVALID_ARG;
    return PA_OK;
}

pa_status check_rows(const int32_t* block_tables, const int32_t* context_lens, int num_seqs, int max_blocks_per_seq,
                     int block_size) {
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
    if (static_cast<long long>(max_blocks_per_seq) * block_size > INT_MAX) return PA_ERR_UNSUPPORTED;
    if (num_seqs > 0 && (!block_tables || !context_lens || !aligned4(block_tables) || !aligned4(context_lens)))
        return PA_ERR_INVALID_ARG;
    return PA_OK;
}

pa::BlockState block_state(int32_t* ref_counts, const int32_t* free_ids, int64_t* free_state, int64_t num_blocks) {
    pa::BlockState st{};
    st.ref = ref_counts;
    st.free_ids = const_cast<int32_t*>(free_ids);
    st.free_state = reinterpret_cast<long long*>(free_state);
    st.num_blocks = num_blocks;
    return st;
}

}  // namespace

extern "C" {

pa_status pa_blocks_init(int32_t* ref_counts, int32_t* free_ids, int64_t* free_state, int64_t num_blocks,
                         void* stream) {
    const pa_status st = check_block_state(ref_counts, free_ids, free_state, num_blocks);
    if (st != PA_OK) return st;
    const long long blocks = std::min<long long>((num_blocks + 255) / 256, 4096);
    return launch_early(pa::pa_blocks_init_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                        static_cast<cudaStream_t>(stream), PA_EARLY_LAUNCH,
                        block_state(ref_counts, free_ids, free_state, num_blocks)) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

pa_status pa_blocks_append(int32_t* block_tables, int32_t* context_lens, const int32_t* num_new_tokens,
                           int32_t* ref_counts, const int32_t* free_ids, int64_t* free_state, int64_t* slot_mapping,
                           int64_t num_slots, int64_t* copy_pairs, int num_seqs, int max_blocks_per_seq,
                           int block_size, int64_t num_blocks, void* stream) {
    pa_status st = check_block_state(ref_counts, free_ids, free_state, num_blocks);
    if (st == PA_OK) st = check_rows(block_tables, context_lens, num_seqs, max_blocks_per_seq, block_size);
    if (st != PA_OK) return st;
    if (num_slots < 0) return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    if (!num_new_tokens || !copy_pairs || !aligned4(num_new_tokens) || !aligned8(copy_pairs)) return PA_ERR_INVALID_ARG;
    if (num_slots > 0 && (!slot_mapping || !aligned8(slot_mapping))) return PA_ERR_INVALID_ARG;
    pa::AppendParams p{};
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.num_new = num_new_tokens;
    p.st = block_state(ref_counts, free_ids, free_state, num_blocks);
    p.slots = reinterpret_cast<long long*>(slot_mapping);
    p.num_slots = num_slots;
    p.pairs = reinterpret_cast<long long*>(copy_pairs);
    p.num_seqs = num_seqs;
    p.max_blocks = max_blocks_per_seq;
    p.block_size = block_size;
    const int threads = std::min(pa::kBlocksThreads, (num_seqs + 31) / 32 * 32);
    return launch_early(pa::pa_blocks_append_kernel, dim3(1), dim3(threads), 0, static_cast<cudaStream_t>(stream),
                        PA_EARLY_LAUNCH, p) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

pa_status pa_blocks_fork(int32_t* block_tables, int32_t* context_lens, int32_t* ref_counts, const int32_t* forks,
                         int num_forks, int num_seqs, int max_blocks_per_seq, int block_size, int64_t num_blocks,
                         void* stream) {
    pa_status st = check_rows(block_tables, context_lens, num_seqs, max_blocks_per_seq, block_size);
    if (st != PA_OK) return st;
    if (num_forks < 0 || num_blocks <= 0 || num_blocks > INT_MAX) return PA_ERR_INVALID_ARG;
    if (num_forks == 0 || num_seqs == 0) return PA_OK;
    if (!ref_counts || !forks || !aligned4(ref_counts) || !aligned4(forks)) return PA_ERR_INVALID_ARG;
    pa::ForkParams p{};
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.ref = ref_counts;
    p.forks = forks;
    p.num_forks = num_forks;
    p.num_seqs = num_seqs;
    p.max_blocks = max_blocks_per_seq;
    p.block_size = block_size;
    p.num_blocks = num_blocks;
    return launch_early(pa::pa_blocks_fork_kernel, dim3(1), dim3(pa::kBlocksThreads), 0,
                        static_cast<cudaStream_t>(stream), PA_EARLY_LAUNCH, p) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

pa_status pa_blocks_release(int32_t* block_tables, int32_t* context_lens, int32_t* ref_counts, int32_t* free_ids,
                            int64_t* free_state, const int32_t* seqs, int num_release, int num_seqs,
                            int max_blocks_per_seq, int block_size, int64_t num_blocks, void* stream) {
    pa_status st = check_block_state(ref_counts, free_ids, free_state, num_blocks);
    if (st == PA_OK) st = check_rows(block_tables, context_lens, num_seqs, max_blocks_per_seq, block_size);
    if (st != PA_OK) return st;
    if (num_release < 0) return PA_ERR_INVALID_ARG;
    if (num_release == 0 || num_seqs == 0) return PA_OK;
    if (!seqs || !aligned4(seqs)) return PA_ERR_INVALID_ARG;
    pa::ReleaseParams p{};
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.st = block_state(ref_counts, free_ids, free_state, num_blocks);
    p.seqs = seqs;
    p.num_release = num_release;
    p.num_seqs = num_seqs;
    p.max_blocks = max_blocks_per_seq;
    p.block_size = block_size;
    return launch_early(pa::pa_blocks_release_kernel, dim3(1), dim3(pa::kBlocksThreads), 0,
                        static_cast<cudaStream_t>(stream), PA_EARLY_LAUNCH, p) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
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

// ----------------------------------------------------------------------------
// Split-K decode with library-owned scratch (no allocation by the caller or
// the library).  Some callers cannot allocate device memory when they launch
// work: plugins of inference runtimes that are handed only their inputs and
// outputs at enqueue time, or latency-critical loops where cudaMalloc's
// implicit device synchronisation would stall other streams.  For them, the
// fp32 partial results live in one fixed array in the library's device image.

namespace {

// The array is part of the module, so every GPU that loads the library holds
// it until the process exits.
constexpr size_t kStaticScratchBytes = PA_SPLITK_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) float g_splitk_scratch[kStaticScratchBytes / sizeof(float)];

// Device address of g_splitk_scratch on the current device.  In host code
// the name g_splitk_scratch is only a host-side stand-in, so the address is
// looked up once per device (with that device current) and cached.
// A failed runtime call leaves its error as the thread's last error; it is
// cleared here so that a later launch check does not report it for an
// unrelated call.
pa_status static_scratch_address(void** ptr) {
    static std::mutex mu;
    static std::map<int, void*> cached;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return PA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(mu);
    auto it = cached.find(dev);
    if (it == cached.end()) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_splitk_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return PA_ERR_CUDA;
        }
        it = cached.emplace(dev, p).first;
    }
    *ptr = it->second;
    return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_splitk_static(void* out, const void* q, const void* k_cache, const void* v_cache,
                                             const int32_t* block_tables, const int32_t* context_lens, float scale,
                                             int block_size, int num_seqs, int num_q_heads, int num_kv_heads,
                                             int head_dim, int max_blocks_per_seq, int max_context_len,
                                             int64_t num_blocks, pa_dtype dtype, int partition_size,
                                             void* stream) {
    // Requests whose partials do not fit the fixed array are refused before
    // any device work.
    size_t need = 0;
    const pa_status size_status =
        pa_decode_splitk_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len, partition_size, &need);
    if (size_status != PA_OK) return size_status;
    if (need > kStaticScratchBytes) return PA_ERR_WORKSPACE;
    void* scratch = nullptr;
    const pa_status addr_status = static_scratch_address(&scratch);
    if (addr_status != PA_OK) return addr_status;
    // Two-launch form (no arrival counters): the partition kernel writes every
    // partial that the merge kernel reads (a partition whose copies timed out
    // is written as empty), so no part of the array has to start at zero and
    // the previous call's leftovers are never read.
    return pa_decode_splitk(out, q, k_cache, v_cache, block_tables, context_lens, scale, block_size, num_seqs,
                            num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, max_context_len, num_blocks,
                            dtype, partition_size, scratch, kStaticScratchBytes, nullptr, 0, nullptr, stream);
}

#ifdef PA_TEST_HOOKS
// ----------------------------------------------------------------------------
// Test hooks (libpa_test.so only; declared in pa_test.h).

namespace {

// One warp waits on an mbarrier that no thread or copy ever completes.
__global__ void pa_test_wait_kernel(unsigned long long limit_ns, long long* elapsed_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        pa::mbar_init(&bar, 1);
        pa::fence_barrier_init();
    }
    __syncwarp();
    const uint64_t t0 = pa::global_timer_ns();
    const bool done = pa::mbar_wait_bounded(&bar, 0, limit_ns);
    const uint64_t t1 = pa::global_timer_ns();
    if (threadIdx.x == 0) {
        if (!done) pa::flag_error(PA_DEVERR_TIMEOUT);
        *elapsed_ns = static_cast<long long>(t1 - t0);
    }
}

}  // namespace

extern "C" pa_status pa_test_set_hooks(int64_t wait_limit_ns, int skip_first_copy) {
    if (wait_limit_ns <= 0) return PA_ERR_INVALID_ARG;
    const unsigned long long limit = static_cast<unsigned long long>(wait_limit_ns);
    if (cudaMemcpyToSymbol(pa::g_test_wait_limit_ns, &limit, sizeof(limit)) != cudaSuccess) return PA_ERR_CUDA;
    if (cudaMemcpyToSymbol(pa::g_test_skip_first_copy, &skip_first_copy, sizeof(int)) != cudaSuccess)
        return PA_ERR_CUDA;
    return PA_OK;
}

extern "C" pa_status pa_test_wait_timeout(int64_t limit_ns, int64_t* elapsed_ns, void* stream) {
    if (limit_ns <= 0 || !elapsed_ns || (reinterpret_cast<uintptr_t>(elapsed_ns) & 7u)) return PA_ERR_INVALID_ARG;
    pa_test_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<unsigned long long>(limit_ns),
                                                                         reinterpret_cast<long long*>(elapsed_ns));
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
#endif  // PA_TEST_HOOKS
