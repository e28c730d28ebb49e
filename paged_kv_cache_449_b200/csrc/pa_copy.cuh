// Whole-block copies between pool pairs: the copy-on-write duplicate of a
// shared block ("vLLM框架解析：PagedAttention技术如何实现LLM推理20倍加速" §2.3)
// and the swap-out / swap-in of a preempted sequence's blocks to and from
// host memory ("vLLM核心架构总览" §4.2).
//
// A block of one pool is Hkv * B * D elements, contiguous in the pool layout
// ([num_blocks][Hkv][D/X][B][X]), so a copy is a contiguous byte range per
// (pair, pool): no layout arithmetic is needed.  Each CTA moves one chunk of
// kChunkVecs 16-byte vectors of one block of one pool; every thread issues
// kUnroll independent loads before its stores so that enough bytes are in
// flight for HBM (device pools) or PCIe (page-locked host pools, reached
// through the unified address space).
#pragma once

#include "pa_device.cuh"

namespace pa {

struct CopyParams {
    uint4* dst[2];               // K pool, V pool (device or page-locked host memory)
    const uint4* src[2];
    const int64_t* mapping;      // [num_pairs][2]: source block, destination block
    long long num_pairs;
    long long vecs_per_block;    // Hkv * B * D * e / 16
    long long src_blocks;
    long long dst_blocks;
    int chunks;                  // chunks per block
};

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;
constexpr int kChunkVecs = kCopyThreads * kCopyUnroll;  // 16 KiB

__global__ void __launch_bounds__(kCopyThreads) pa_copy_blocks_kernel(const __grid_constant__ CopyParams p) {
    wait_for_prior_work();
    const long long unit = blockIdx.x;
    const int chunk = static_cast<int>(unit % p.chunks);
    const long long rest = unit / p.chunks;
    const int pool = static_cast<int>(rest & 1);
    const long long pair = rest >> 1;
    const long long src = p.mapping[2 * pair];
    const long long dst = p.mapping[2 * pair + 1];
    if (src < 0) return;  // an empty entry (no copy for this pair)
    if (src >= p.src_blocks || dst < 0 || dst >= p.dst_blocks) {
        if (threadIdx.x == 0 && pool == 0 && chunk == 0) flag_error(1 /* PA_DEVERR_BLOCK_ID */);
        return;
    }
    const uint4* from = p.src[pool] + src * p.vecs_per_block;
    uint4* to = p.dst[pool] + dst * p.vecs_per_block;
    const long long v0 = static_cast<long long>(chunk) * kChunkVecs;
    const long long v1 = min(v0 + kChunkVecs, p.vecs_per_block);
    uint4 r[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const long long v = v0 + threadIdx.x + u * kCopyThreads;
        if (v < v1) r[u] = from[v];
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const long long v = v0 + threadIdx.x + u * kCopyThreads;
        if (v < v1) to[v] = r[u];
    }
}

}  // namespace pa
