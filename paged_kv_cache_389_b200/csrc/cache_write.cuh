// The bf16 / fp32 cache write of one 16-byte chunk (shared by the write kernel and
// the one-call step's fused write + detection kernel).
#pragma once

#include "pa_common.cuh"

namespace pa {

// Chunk idx of the new tokens' K/V rows ([num_tokens, Hkv, chunks_per_row]
// 16-byte chunks): copied to slot slot_mapping[token] of the pools
// ([blocks, Hkv, 16, chunks_per_row]); slot < 0 is padding, slot >= num_slots
// is flagged and skipped.
__device__ __forceinline__ void write_chunk(int64_t idx, const uint4 *__restrict__ key,
                                            const uint4 *__restrict__ value,
                                            const int64_t *__restrict__ slot_mapping, int32_t num_tokens,
                                            uint4 *__restrict__ key_cache, uint4 *__restrict__ value_cache,
                                            int32_t num_kv_heads, int32_t chunks_per_row, int64_t num_slots,
                                            int32_t *err) {
    const int64_t per_token = (int64_t)num_kv_heads * chunks_per_row;
    const int64_t token = idx / per_token;
    if (token >= num_tokens) return;
    const int64_t slot = slot_mapping[token];
    if (slot < 0) return;  // padding
    if (slot >= num_slots) {
        if (idx % per_token == 0) flag_error(err, PA_DEVERR_SLOT);
        return;
    }
    const int64_t rem = idx - token * per_token;      // (head, chunk) inside the token
    const int64_t head = rem / chunks_per_row;
    const int64_t chunk = rem - head * chunks_per_row;
    const int64_t block = slot / kBlockSize, offset = slot % kBlockSize;
    const int64_t dst = ((block * num_kv_heads + head) * kBlockSize + offset) * chunks_per_row + chunk;
    key_cache[dst] = key[idx];
    value_cache[dst] = value[idx];
}

}  // namespace pa
