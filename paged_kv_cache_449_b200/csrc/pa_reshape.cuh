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
#include "pa_e4m3.cuh"

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
    wait_for_prior_work();
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

// The 8-bit pools' write: one thread quantises four elements of a K row
// (dims 2w, 2w+1, 2w+8, 2w+9 of a 16-dim vector: one 32-bit word of the K
// tile) and the same four of the V row (one byte in each of four dim rows of
// the transposed V tile), with its kv head's scales.
struct ReshapeE4m3Params {
    const void* key;         // [T][Hkv][D] elements of the input type
    const void* value;
    uint32_t* k_cache;       // tiles of [D/16][B][4] words of 4 codes
    uint8_t* v_cache;        // tiles of [D][B] codes
    const int64_t* slot_mapping;
    const float* k_scale;    // [Hkv]
    const float* v_scale;
    long long num_tokens;
    int num_kv_heads;
    int head_dim;
    int block_size;
    long long num_slots;
};

template <typename T>
__global__ void __launch_bounds__(256) pa_reshape_e4m3_kernel(const __grid_constant__ ReshapeE4m3Params p) {
    wait_for_prior_work();
    const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int words = p.head_dim / 4;   // four words per 16-dim vector
    const long long per_token = static_cast<long long>(p.num_kv_heads) * words;
    if (idx >= p.num_tokens * per_token) return;
    const long long i = idx / per_token;
    const long long slot = p.slot_mapping[i];
    if (slot < 0) return;  // padding token
    if (slot >= p.num_slots) {
        flag_error(4 /* PA_DEVERR_SLOT */);
        return;
    }
    const int rem = static_cast<int>(idx - i * per_token);
    const int h = rem / words;
    const int wi = rem - h * words;
    const int j = wi >> 2, w = wi & 3;          // vector j, word w
    const int d0 = 16 * j + 2 * w, d1 = d0 + 8;  // dims d0, d0+1, d1, d1+1
    const long long block = slot / p.block_size;
    const int offset = static_cast<int>(slot - block * p.block_size);
    const long long tile = block * p.num_kv_heads + h;
    const T* krow = reinterpret_cast<const T*>(p.key) + (i * p.num_kv_heads + h) * p.head_dim;
    const T* vrow = reinterpret_cast<const T*>(p.value) + (i * p.num_kv_heads + h) * p.head_dim;
    const float ks = p.k_scale[h], vs = p.v_scale[h];
    p.k_cache[((tile * (p.head_dim / 16) + j) * p.block_size + offset) * 4 + w] =
        quantise2(to_float<T>(krow[d0]), to_float<T>(krow[d0 + 1]), ks) |
        (quantise2(to_float<T>(krow[d1]), to_float<T>(krow[d1 + 1]), ks) << 16);
    const uint32_t v01 = quantise2(to_float<T>(vrow[d0]), to_float<T>(vrow[d0 + 1]), vs);
    const uint32_t v89 = quantise2(to_float<T>(vrow[d1]), to_float<T>(vrow[d1 + 1]), vs);
    uint8_t* vt = p.v_cache + tile * p.head_dim * p.block_size + v_row_byte(offset, p.block_size);
    vt[d0 * p.block_size] = static_cast<uint8_t>(v01 & 0xff);
    vt[(d0 + 1) * p.block_size] = static_cast<uint8_t>(v01 >> 8);
    vt[d1 * p.block_size] = static_cast<uint8_t>(v89 & 0xff);
    vt[(d1 + 1) * p.block_size] = static_cast<uint8_t>(v89 >> 8);
}

}  // namespace pa
