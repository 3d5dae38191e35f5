// KV append through a slot mapping (reshape-and-cache) and copy-on-write block
// copy.  Both are pure data movement: 16-byte vector loads and stores, every
// thread moving whole 16-byte chunks, grids sized to cover the bytes once.
//
// Sources: "vLLM 深度拆解" (chenxutan) 3.1 -- each step writes the new token's K/V
// back into the cache; devpress vLLM v0.6.x teardown, 关键设计二 -- copy-on-write
// copies a whole shared block into a freshly allocated one.
#include <cuda_fp8.h>

#include "cache_write.cuh"
#include "pa_common.cuh"
#include "pa_launch.h"

namespace pa {

// One thread per 16-byte chunk of one (token, kv head) row of K (and of V).
__global__ void __launch_bounds__(256) cache_write_kernel(
    const uint4 *__restrict__ key, const uint4 *__restrict__ value,
    const int64_t *__restrict__ slot_mapping, int32_t num_tokens, uint4 *__restrict__ key_cache,
    uint4 *__restrict__ value_cache, int32_t num_kv_heads, int32_t chunks_per_row,
    int64_t num_slots, int32_t *err) {
    // a decode launched behind this write (pa_append_decode) may start launching;
    // whatever of it reads the cache waits for this grid to finish
    grid_dep_launch();
    write_chunk((int64_t)blockIdx.x * blockDim.x + threadIdx.x, key, value, slot_mapping, num_tokens, key_cache,
                value_cache, num_kv_heads, chunks_per_row, num_slots, err);
}

// FP8 pools: one thread per 8 elements (16 bytes of bf16 in, 8 bytes of e4m3
// out) of one (token, kv head) row.  code = e4m3(fp32(x) / scale): an IEEE
// division, then the hardware conversion (nearest even, saturated to +-448).
__device__ __forceinline__ uint32_t quantise4(uint32_t lo, uint32_t hi, float scale) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&lo));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&hi));
    const uint32_t c0 = __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(a.x, scale), __fdiv_rn(a.y, scale)),
                                                 __NV_SATFINITE, __NV_E4M3);
    const uint32_t c1 = __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(b.x, scale), __fdiv_rn(b.y, scale)),
                                                 __NV_SATFINITE, __NV_E4M3);
    return c0 | (c1 << 16);
}

__global__ void __launch_bounds__(256) cache_write_fp8_kernel(
    const uint4 *__restrict__ key, const uint4 *__restrict__ value,
    const int64_t *__restrict__ slot_mapping, int32_t num_tokens, uint2 *__restrict__ key_cache,
    uint2 *__restrict__ value_cache, int32_t num_kv_heads, int32_t chunks_per_row,
    int64_t num_slots, float k_scale, float v_scale, int32_t *err) {
    grid_dep_launch();
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t per_token = (int64_t)num_kv_heads * chunks_per_row;
    const int64_t token = idx / per_token;
    if (token >= num_tokens) return;
    const int64_t slot = slot_mapping[token];
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (idx % per_token == 0) flag_error(err, PA_DEVERR_SLOT);
        return;
    }
    const int64_t rem = idx - token * per_token;
    const int64_t head = rem / chunks_per_row;
    const int64_t chunk = rem - head * chunks_per_row;
    const int64_t block = slot / kBlockSize, offset = slot % kBlockSize;
    const int64_t dst = ((block * num_kv_heads + head) * kBlockSize + offset) * chunks_per_row + chunk;
    const uint4 k = key[idx], v = value[idx];
    key_cache[dst] = make_uint2(quantise4(k.x, k.y, k_scale), quantise4(k.z, k.w, k_scale));
    value_cache[dst] = make_uint2(quantise4(v.x, v.y, v_scale), quantise4(v.z, v.w, v_scale));
}

// grid = (num_pairs, ceil(chunks_per_block / (256 * kCopyUnroll)), 2): z selects K or V.
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4 *__restrict__ key_cache,
                                                          uint4 *__restrict__ value_cache,
                                                          const int32_t *__restrict__ pairs,
                                                          int64_t chunks_per_block,
                                                          int32_t num_blocks, int32_t *err) {
    const int32_t src = pairs[2 * blockIdx.x], dst = pairs[2 * blockIdx.x + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) flag_error(err, PA_DEVERR_PAIR);
        return;
    }
    uint4 *cache = blockIdx.z == 0 ? key_cache : value_cache;
    const uint4 *s = cache + (int64_t)src * chunks_per_block;
    uint4 *d = cache + (int64_t)dst * chunks_per_block;
    const int64_t base = (int64_t)blockIdx.y * blockDim.x * kCopyUnroll + threadIdx.x;
    uint4 buf[kCopyUnroll];
#pragma unroll
    for (int k = 0; k < kCopyUnroll; ++k) {
        const int64_t c = base + (int64_t)k * blockDim.x;
        if (c < chunks_per_block) buf[k] = s[c];
    }
#pragma unroll
    for (int k = 0; k < kCopyUnroll; ++k) {
        const int64_t c = base + (int64_t)k * blockDim.x;
        if (c < chunks_per_block) d[c] = buf[k];
    }
}

cudaError_t launch_cache_write(const void *key, const void *value, const int64_t *slot_mapping,
                               int32_t num_tokens, void *key_cache, void *value_cache,
                               const pa_cache_desc &c, int32_t *err, cudaStream_t stream) {
    if (c.dtype == PA_FP8_E4M3) {
        const int32_t chunks_per_row = c.head_dim / 8;
        const int64_t blocks = ((int64_t)num_tokens * c.num_kv_heads * chunks_per_row + 255) / 256;
        cache_write_fp8_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
            static_cast<const uint4 *>(key), static_cast<const uint4 *>(value), slot_mapping,
            num_tokens, static_cast<uint2 *>(key_cache), static_cast<uint2 *>(value_cache),
            c.num_kv_heads, chunks_per_row, (int64_t)c.num_blocks * kBlockSize, c.k_scale, c.v_scale, err);
        return cudaGetLastError();
    }
    const int32_t chunks_per_row = c.head_dim * dtype_bytes(c.dtype) / 16;
    const int64_t threads = (int64_t)num_tokens * c.num_kv_heads * chunks_per_row;
    const int64_t blocks = (threads + 255) / 256;
    cache_write_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const uint4 *>(key), static_cast<const uint4 *>(value), slot_mapping,
        num_tokens, static_cast<uint4 *>(key_cache), static_cast<uint4 *>(value_cache),
        c.num_kv_heads, chunks_per_row, (int64_t)c.num_blocks * kBlockSize, err);
    return cudaGetLastError();
}

cudaError_t launch_copy_blocks(void *key_cache, void *value_cache, const int32_t *pairs,
                               int32_t num_pairs, const pa_cache_desc &c, int32_t *err,
                               cudaStream_t stream) {
    const int64_t chunks_per_block =
        (int64_t)c.num_kv_heads * kBlockSize * c.head_dim * dtype_bytes(c.dtype) / 16;
    const int64_t per_cta = 256 * kCopyUnroll;
    dim3 grid((unsigned)num_pairs, (unsigned)((chunks_per_block + per_cta - 1) / per_cta), 2);
    copy_blocks_kernel<<<grid, 256, 0, stream>>>(static_cast<uint4 *>(key_cache),
                                                 static_cast<uint4 *>(value_cache), pairs,
                                                 chunks_per_block, c.num_blocks, err);
    return cudaGetLastError();
}

}  // namespace pa
