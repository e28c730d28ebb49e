// KV-cache write: scatter the K/V rows of new tokens into the pools through
// slot_mapping ("从源码剖析 vLLM 的显存管理与连续批处理" §2.1, BlockTable.append_token:
// the physical address of a token is its block's address plus its offset).
//
// One thread moves one 16-byte vector of K and the matching vector of V:
// the source rows are read fully coalesced, and each destination vector is a
// single aligned 128-bit store (the pool keeps D split into 16-byte vectors).
// The copy is a bit copy, so it is independent of the element type.
#pragma once

#include "pa_device.cuh"

namespace pa {

struct ReshapeParams {
    const uint4* key;        // [T][Hkv][V] vectors
    const uint4* value;
    uint4* k_cache;          // [N][Hkv][V][B] vectors
    uint4* v_cache;
    const int64_t* slot_mapping;
    long long num_tokens;
    int num_kv_heads;
    int vecs_per_row;        // head_dim * elem_size / 16
    int block_size;
    long long num_slots;     // num_blocks * block_size
};

__global__ void __launch_bounds__(256) pa_reshape_kernel(const __grid_constant__ ReshapeParams p) {
    const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long per_token = static_cast<long long>(p.num_kv_heads) * p.vecs_per_row;
    if (idx >= p.num_tokens * per_token) return;
    const long long i = idx / per_token;
    const long long slot = p.slot_mapping[i];
    if (slot < 0) return;  // padding token
    if (slot >= p.num_slots) {
        flag_error(4 /* PA_DEVERR_SLOT */);
        return;
    }
    const int rem = static_cast<int>(idx - i * per_token);
    const int h = rem / p.vecs_per_row;
    const int j = rem - h * p.vecs_per_row;
    const long long block = slot / p.block_size;
    const int offset = static_cast<int>(slot - block * p.block_size);
    const long long dst = ((block * p.num_kv_heads + h) * p.vecs_per_row + j) * p.block_size + offset;
    const uint4 k = p.key[idx];
    const uint4 v = p.value[idx];
    p.k_cache[dst] = k;
    p.v_cache[dst] = v;
}

}  // namespace pa
