// Internal launch interface between the C ABI (pa_api.cu) and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "pa.h"

namespace pa {

inline int dtype_bytes(int32_t dtype) { return dtype == PA_F32 ? 4 : dtype == PA_FP8_E4M3 ? 1 : 2; }

// Launch `kern` behind the previous grid on `stream` with programmatic stream
// serialization: it may start before that grid ends and must call grid_dep_wait
// (pa_common.cuh) before reading what that grid writes.
template <typename... Args>
cudaError_t launch_after(void (*kern)(Args...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                         const Args &...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

cudaError_t launch_cache_write(const void *key, const void *value, const int64_t *slot_mapping,
                               int32_t num_tokens, void *key_cache, void *value_cache,
                               const pa_cache_desc &c, int32_t *err, cudaStream_t stream);

cudaError_t launch_copy_blocks(void *key_cache, void *value_cache, const int32_t *pairs,
                               int32_t num_pairs, const pa_cache_desc &c, int32_t *err,
                               cudaStream_t stream);

struct DecodeLaunch {
    const void *query;
    const void *key_cache;
    const void *value_cache;
    const int32_t *block_tables;
    int32_t max_blocks_per_seq;
    const int32_t *context_lens;
    int32_t max_context_len;
    int32_t num_seqs;
    int32_t num_q_heads;
    float scale;
    int32_t partition_size;  // 0 = no split
    int32_t max_partitions;  // ceil(max_context_len / partition_size) when split
    float *ws_acc;           // [S][Hq][Pmax][D] unnormalised partial accumulators
    float2 *ws_ml;           // [S][Hq][Pmax] (running max in log2 units, running sum)
    void *ws_group;          // shared-prefix group bookkeeping (split contexts), or null
    void *out;
    pa_cache_desc cache;
    int32_t *err;
    bool after_write;  // launched behind a cache write on the same stream (pa_append_decode)
    const struct StepWrite *write;  // the step's write, done inside the first decode kernel (or null)
};

// The new tokens' cache write of a one-call step (pa_append_decode).
struct StepWrite {
    const void *key;
    const void *value;
    const int64_t *slot_mapping;
    int32_t num_tokens;
    void *key_cache;
    void *value_cache;
};

// Largest num_seqs a split decode supports (the per-CTA partition prefix sum
// lives in shared memory).
constexpr int32_t kMaxSplitSeqs = 4096;

cudaError_t launch_decode(const DecodeLaunch &a, cudaStream_t stream);

// The one-call step: the write, then the decode chain.  When the decode takes the
// shared-prefix path the write runs inside the detection kernel's grid (no
// launch of its own); otherwise it is launch_cache_write followed by launch_decode.
cudaError_t launch_append_decode(const StepWrite &w, DecodeLaunch a, cudaStream_t stream);

struct PrefillLaunch {
    const void *query;
    const void *key_cache;
    const void *value_cache;
    const int32_t *block_tables;
    int32_t max_blocks_per_seq;
    const int32_t *context_lens;
    const int32_t *chunk_lens;
    int32_t num_seqs;
    int32_t max_chunk;
    int32_t num_q_heads;
    float scale;
    void *out;
    pa_cache_desc cache;
    int32_t *err;
};

cudaError_t launch_prefill(const PrefillLaunch &a, cudaStream_t stream);

// Shared-prefix group units of a split bf16 / head_dim 128 decode, on the tcgen05
// tile kernel: one unit per (group, kv head), rows = the group's members x g query
// heads, keys = the leading full blocks the members share; it writes one partial
// (slot 0 of each member).  groups / meta are the decode's detection output (device memory).
struct GroupTileLaunch {
    const void *query;       // [num_seqs, num_q_heads, 128] bf16
    int32_t num_seqs;
    const void *key_cache;
    const void *value_cache;
    const int32_t *block_tables;
    int32_t max_blocks_per_seq;
    const int4 *groups;
    const int32_t *meta;
    float *ws_acc;
    float2 *ws_ml;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t num_blocks;
    int32_t max_partitions;
    float scale;
    int32_t *err;
};
cudaError_t launch_group_tiles(const GroupTileLaunch &a, int sms, cudaStream_t stream);

int num_sms(int device);

// Bound of every in-kernel wait for launches made from now on, in ns
// (pa_set_wait_timeout_ns; kWaitTimeoutNs by default).
unsigned long long wait_limit_ns();

}  // namespace pa
