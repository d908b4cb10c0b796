// pa_append.cuh -- slot-mapped KV-cache append ("reshape_and_cache").
//
// Each thread moves one 16-byte chunk (8 bf16) of one (token, kv head) row
// of K and the same chunk of V into row slot % bs of block slot / bs of the
// [NB][Hkv][bs][D] caches.  Loads and stores are 128-bit and coalesced on
// both sides (a row is D*2 contiguous bytes in k_new and in the cache).
// It is a bit copy, so the result is exact.
#pragma once

#include "pa_device.cuh"

namespace pa {

struct AppendParams {
    const uint4* k_new;  // [T][Hkv][D] bf16, viewed as 16-byte chunks
    const uint4* v_new;
    const int32_t* slot_mapping;  // [T]
    uint4* k_cache;               // [NB][Hkv][bs][D]
    uint4* v_cache;
    int64_t num_chunks;           // T * Hkv * D / 8
    int32_t chunks_per_row;       // D / 8
    int32_t kv_heads;
    int32_t block_size;
    int32_t num_blocks;
};

constexpr int kAppendThreads = 256;

__global__ void __launch_bounds__(kAppendThreads) append_kernel(AppendParams p) {
    const int64_t idx = int64_t(blockIdx.x) * kAppendThreads + threadIdx.x;
    if (idx >= p.num_chunks) return;
    const int64_t per_token = int64_t(p.kv_heads) * p.chunks_per_row;
    const int64_t t = idx / per_token;
    const int64_t rem = idx - t * per_token;  // g * chunks_per_row + c
    const int32_t slot = __ldg(p.slot_mapping + t);
    if (slot < 0) return;  // padding token
    const int64_t block = slot / p.block_size;
    const int64_t offset = slot - block * p.block_size;
    if (block >= p.num_blocks) {
        if (rem == 0) raise_error(PA_DEVERR_SLOT);
        return;
    }
    const int64_t g = rem / p.chunks_per_row;
    const int64_t c = rem - g * p.chunks_per_row;
    const int64_t dst = ((block * p.kv_heads + g) * p.block_size + offset) * p.chunks_per_row + c;
    const uint4 kv = __ldg(p.k_new + idx);
    const uint4 vv = __ldg(p.v_new + idx);
    p.k_cache[dst] = kv;
    p.v_cache[dst] = vv;
}

}  // namespace pa
