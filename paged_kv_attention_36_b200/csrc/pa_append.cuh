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

// ---- fp8 (E4M3) caches --------------------------------------------------------
// k_cache8 [NB][Hkv][16][D] (token-major) and v_cache8 [NB][Hkv][D][16]: each
// (block, kv head) V tile is stored transposed, row d holding the 16 tokens'
// column-d codes, token t at position 4*((t % 8) / 2) + 2*(t / 8) + t % 2.  This
// order lets the decode's tensor-core fragments of V^T come from a plain
// ldmatrix of 8-byte groups (two tokens t, t+1 then t+8, t+9 per 4 bytes).
// Codes are e4m3(x / scale[g]): fp32 division, nearest code, ties to even,
// saturating at +-448.
struct AppendFp8Params {
    const uint4* k_new;           // [T][Hkv][D] bf16, 16-byte chunks
    const uint4* v_new;
    const int32_t* slot_mapping;  // [T]
    uint8_t* k_cache;             // [NB][Hkv][16][D] e4m3
    uint8_t* v_cache;             // [NB][Hkv][D][16] e4m3
    const float* k_scale;         // [Hkv]
    const float* v_scale;         // [Hkv]
    int64_t num_chunks;           // T * Hkv * D / 8
    int32_t chunks_per_row;       // D / 8
    int32_t kv_heads;
    int32_t num_blocks;
};

__device__ __forceinline__ int vt_position(int t) { return 4 * ((t & 7) >> 1) + 2 * (t >> 3) + (t & 1); }

// Encodes and stores chunk idx (8 values of one (token, kv head) row of K
// and of V) of the step's new rows; the body of append_fp8_kernel, also run
// by the fused fp8 append + decode.
__device__ __forceinline__ void append_fp8_chunk(const uint4* k_new, const uint4* v_new, const int32_t* slot_mapping,
                                                 uint8_t* k_cache, uint8_t* v_cache, const float* k_scale,
                                                 const float* v_scale, int kv_heads, int chunks_per_row,
                                                 int num_blocks, int64_t idx) {
    const int64_t per_token = int64_t(kv_heads) * chunks_per_row;
    const int64_t t = idx / per_token;
    const int64_t rem = idx - t * per_token;
    const int32_t slot = __ldg(slot_mapping + t);
    if (slot < 0) return;
    const int64_t block = slot >> 4;
    const int offset = slot & 15;
    if (block >= num_blocks) {
        if (rem == 0) raise_error(PA_DEVERR_SLOT);
        return;
    }
    const int g = int(rem / chunks_per_row);
    const int c = int(rem - int64_t(g) * chunks_per_row);
    const int D = chunks_per_row * 8;
    const int64_t tile = block * kv_heads + g;
    const float ks = __ldg(k_scale + g), vs = __ldg(v_scale + g);
    const uint4 kv = __ldg(k_new + idx), vv = __ldg(v_new + idx);
    const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w}, vw[4] = {vv.x, vv.y, vv.z, vv.w};
    uint16_t k8[4], v8[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 kf = bf16x2_to_float2(kw[j]), vf = bf16x2_to_float2(vw[j]);
        k8[j] = f32x2_to_e4m3x2(__fdiv_rn(kf.x, ks), __fdiv_rn(kf.y, ks));
        v8[j] = f32x2_to_e4m3x2(__fdiv_rn(vf.x, vs), __fdiv_rn(vf.y, vs));
    }
    // K: 8 consecutive codes of row `offset`
    *reinterpret_cast<uint2*>(k_cache + (tile * 16 + offset) * D + c * 8) =
        make_uint2(uint32_t(k8[0]) | (uint32_t(k8[1]) << 16), uint32_t(k8[2]) | (uint32_t(k8[3]) << 16));
    // V: one code in each of the rows c*8 .. c*8+7 of the transposed tile
    uint8_t* vrow = v_cache + (tile * D + c * 8) * 16 + vt_position(offset);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        vrow[(2 * j) * 16] = uint8_t(v8[j] & 0xff);
        vrow[(2 * j + 1) * 16] = uint8_t(v8[j] >> 8);
    }
}

__global__ void __launch_bounds__(kAppendThreads) append_fp8_kernel(AppendFp8Params p) {
    const int64_t idx = int64_t(blockIdx.x) * kAppendThreads + threadIdx.x;
    if (idx >= p.num_chunks) return;
    append_fp8_chunk(p.k_new, p.v_new, p.slot_mapping, p.k_cache, p.v_cache, p.k_scale, p.v_scale, p.kv_heads,
                     p.chunks_per_row, p.num_blocks, idx);
}

}  // namespace pa
