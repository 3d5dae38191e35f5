// C ABI entry points (include/pa.h): host-side validation, then kernel launch.
// No device memory is allocated here; every buffer belongs to the caller.
#include <atomic>
#include <chrono>
#include <cmath>
#include <cstdint>
#include <thread>
#include <vector>

#include "pa_trace.h"
#include "pa_common.cuh"
#include "pa_launch.h"

namespace pa {

int num_sms(int device) {
    static int cached[64] = {0};
    if (device >= 0 && device < 64 && cached[device] > 0) return cached[device];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0)
        n = 148;
    if (device >= 0 && device < 64) cached[device] = n;
    return n;
}

namespace {
std::atomic<unsigned long long> g_wait_limit_ns{kWaitTimeoutNs};
}  // namespace

unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pa_status check_cache(const pa_cache_desc *c) {
    if (!c) return PA_ERR_INVALID_ARG;
    if (c->num_blocks < 0 || c->num_kv_heads <= 0) return PA_ERR_INVALID_ARG;
    if (c->block_size != kBlockSize) return PA_ERR_UNSUPPORTED;
    if (c->head_dim != 64 && c->head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (c->dtype == PA_FP8_E4M3) {
        if (!(c->k_scale > 0.f) || !(c->v_scale > 0.f) || !std::isfinite(c->k_scale) ||
            !std::isfinite(c->v_scale))
            return PA_ERR_INVALID_ARG;
        if (c->head_dim != 128) return PA_ERR_UNSUPPORTED;
        return PA_OK;
    }
    if (c->dtype != PA_F32 && c->dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

pa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? PA_OK : PA_ERR_CUDA; }

pa_status check_group(int32_t num_q_heads, int32_t num_kv_heads) {
    if (num_q_heads <= 0 || num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    const int32_t g = num_q_heads / num_kv_heads;
    if (g != 1 && g != 2 && g != 4 && g != 8) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" {

int32_t pa_abi_version(void) { return 3; }

uint64_t pa_set_wait_timeout_ns(uint64_t ns) {
    if (ns == 0) ns = kWaitTimeoutNs;
    return g_wait_limit_ns.exchange(ns);
}

const char *pa_status_string(pa_status s) {
    switch (s) {
        case PA_OK: return "ok";
        case PA_ERR_INVALID_ARG: return "invalid argument";
        case PA_ERR_UNSUPPORTED: return "unsupported configuration";
        case PA_ERR_OOM: return "out of KV blocks";
        case PA_ERR_DEVICE_INDEX: return "device kernel flagged an out-of-range index";
        case PA_ERR_CUDA: return "CUDA runtime error";
        case PA_ERR_TIMEOUT: return "timed out";
        case PA_ERR_NOT_FOUND: return "unknown sequence id";
    }
    return "unknown status";
}

namespace {
pa_status check_cache_write(const void *key, const void *value, const int64_t *slot_mapping,
                            int32_t num_tokens, const void *key_cache, const void *value_cache,
                            const pa_cache_desc *cache) {
    pa_status st = check_cache(cache);
    if (st != PA_OK) return st;
    if (num_tokens < 0) return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !slot_mapping || !key_cache || !value_cache) return PA_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
        return PA_ERR_INVALID_ARG;
    return PA_OK;
}
}  // namespace

pa_status pa_cache_write(const void *key, const void *value, const int64_t *slot_mapping,
                         int32_t num_tokens, void *key_cache, void *value_cache,
                         const pa_cache_desc *cache, int32_t *err_flag, void *stream) {
    const NvtxRange nvtx_range("pa_cache_write");
    const pa_status st = check_cache_write(key, value, slot_mapping, num_tokens, key_cache, value_cache, cache);
    if (st != PA_OK || num_tokens == 0) return st;
    return from_cuda(launch_cache_write(key, value, slot_mapping, num_tokens, key_cache, value_cache,
                                        *cache, err_flag, static_cast<cudaStream_t>(stream)));
}

pa_status pa_check_copy_pairs(const int32_t *src_dst_pairs, int32_t num_pairs, int32_t num_blocks) {
    if (num_pairs < 0 || num_blocks < 0) return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    if (!src_dst_pairs) return PA_ERR_INVALID_ARG;
    // one byte per block: bit 0 = seen as a source, bit 1 = seen as a destination
    std::vector<unsigned char> role;
    try {
        role.assign((size_t)num_blocks, 0);
    } catch (...) {
        return PA_ERR_OOM;  // no exception crosses the C boundary
    }
    for (int32_t p = 0; p < num_pairs; ++p) {
        const int32_t src = src_dst_pairs[2 * p], dst = src_dst_pairs[2 * p + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks || src == dst)
            return PA_ERR_INVALID_ARG;
        if ((role[(size_t)dst] & 2u) || (role[(size_t)dst] & 1u) || (role[(size_t)src] & 2u))
            return PA_ERR_INVALID_ARG;
        role[(size_t)src] |= 1u;
        role[(size_t)dst] |= 2u;
    }
    return PA_OK;
}

pa_status pa_copy_blocks(void *key_cache, void *value_cache, const int32_t *src_dst_pairs,
                         int32_t num_pairs, const pa_cache_desc *cache, int32_t *err_flag,
                         void *stream) {
    const NvtxRange nvtx_range("pa_copy_blocks");
    pa_status st = check_cache(cache);
    if (st != PA_OK) return st;
    if (num_pairs < 0) return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    if (!key_cache || !value_cache || !src_dst_pairs) return PA_ERR_INVALID_ARG;
    if (!aligned16(key_cache) || !aligned16(value_cache)) return PA_ERR_INVALID_ARG;
    return from_cuda(launch_copy_blocks(key_cache, value_cache, src_dst_pairs, num_pairs, *cache,
                                        err_flag, static_cast<cudaStream_t>(stream)));
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t partition_size) {
    if (partition_size <= 0 || num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 ||
        max_context_len <= 0)
        return 0;
    const int64_t parts = ((int64_t)max_context_len + partition_size - 1) / partition_size;
    const int64_t rows = (int64_t)num_seqs * num_q_heads * parts;
    // partials (fp32 acc, then (m, l)), then the shared-prefix group bookkeeping:
    // shared tokens per sequence (16-byte padded), group list (16 bytes each), 32
    // bytes of counts and counters, the table comparison's per-sequence results
    // (16-byte padded) and its blocks' flags (64 x 8 bytes)
    const int64_t partials = rows * head_dim * 4 + rows * 8;
    const int64_t s16 = ((int64_t)num_seqs * 4 + 15) / 16 * 16;
    const int64_t group = s16 + (int64_t)num_seqs * 16 + 32 + s16 + 64 * 8;
    return (size_t)((partials + 15) / 16 * 16 + group);
}

int32_t pa_decode_launches(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                           int32_t dtype, int32_t partition_size) {
    if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0) return 0;
    if (partition_size <= 0) return 1;
    if (head_dim != 128 || num_seqs > kMaxSplitSeqs || dtype != PA_BF16) return 2;
    // detection, group tiles, [group rows: g <= 4], decode, combine
    return num_q_heads / num_kv_heads <= 4 ? 5 : 4;
}

namespace {
// Validate pa_decode's arguments and fill the launch record; launches nothing.
pa_status prepare_decode(const void *query, const void *key_cache, const void *value_cache,
                         const int32_t *block_tables, int32_t max_blocks_per_seq,
                         const int32_t *context_lens, int32_t max_context_len, int32_t num_seqs,
                         int32_t num_q_heads, float scale, int32_t partition_size, void *workspace,
                         size_t workspace_bytes, void *out, const pa_cache_desc *cache,
                         int32_t *err_flag, DecodeLaunch &a) {
    pa_status st = check_cache(cache);
    if (st != PA_OK) return st;
    st = check_group(num_q_heads, cache->num_kv_heads);
    if (st != PA_OK) return st;
    if (num_seqs < 0 || max_blocks_per_seq < 0 || max_context_len < 0 || partition_size < 0)
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    if (num_seqs > 16384) return PA_ERR_UNSUPPORTED;
    if (partition_size % kBlockSize != 0) return PA_ERR_INVALID_ARG;
    if (!query || !key_cache || !value_cache || !block_tables || !context_lens || !out)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) || !aligned16(out))
        return PA_ERR_INVALID_ARG;
    if ((int64_t)max_context_len > (int64_t)max_blocks_per_seq * kBlockSize)
        return PA_ERR_INVALID_ARG;
    a = DecodeLaunch{};
    if (partition_size > 0 && max_context_len > partition_size) {
        if (num_seqs > kMaxSplitSeqs) return PA_ERR_UNSUPPORTED;
        const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, cache->head_dim,
                                                     max_context_len, partition_size);
        if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PA_ERR_INVALID_ARG;
        const int64_t parts = ((int64_t)max_context_len + partition_size - 1) / partition_size;
        a.partition_size = partition_size;
        a.max_partitions = (int32_t)parts;
        a.ws_acc = static_cast<float *>(workspace);
        const size_t rows = (size_t)num_seqs * num_q_heads * parts;
        a.ws_ml = reinterpret_cast<float2 *>(static_cast<char *>(workspace) + rows * cache->head_dim * 4);
        a.ws_group = static_cast<char *>(workspace) + (rows * cache->head_dim * 4 + rows * 8 + 15) / 16 * 16;
    } else {
        // every context fits in one partition: the split would change nothing
        a.partition_size = 0;
        a.max_partitions = 1;
    }
    a.query = query;
    a.key_cache = key_cache;
    a.value_cache = value_cache;
    a.block_tables = block_tables;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.context_lens = context_lens;
    a.max_context_len = max_context_len;
    a.num_seqs = num_seqs;
    a.num_q_heads = num_q_heads;
    a.scale = scale;
    a.out = out;
    a.cache = *cache;
    a.err = err_flag;
    return PA_OK;
}

}  // namespace

pa_status pa_decode(const void *query, const void *key_cache, const void *value_cache,
                    const int32_t *block_tables, int32_t max_blocks_per_seq,
                    const int32_t *context_lens, int32_t max_context_len, int32_t num_seqs,
                    int32_t num_q_heads, float scale, int32_t partition_size, void *workspace,
                    size_t workspace_bytes, void *out, const pa_cache_desc *cache,
                    int32_t *err_flag, void *stream) {
    const NvtxRange nvtx_range("pa_decode");
    DecodeLaunch a;
    const pa_status st = prepare_decode(query, key_cache, value_cache, block_tables, max_blocks_per_seq,
                                        context_lens, max_context_len, num_seqs, num_q_heads, scale,
                                        partition_size, workspace, workspace_bytes, out, cache, err_flag, a);
    if (st != PA_OK || num_seqs == 0) return st;
    return from_cuda(launch_decode(a, static_cast<cudaStream_t>(stream)));
}

pa_status pa_append_decode(const void *key, const void *value, const int64_t *slot_mapping,
                           int32_t num_tokens, const void *query, void *key_cache, void *value_cache,
                           const int32_t *block_tables, int32_t max_blocks_per_seq,
                           const int32_t *context_lens, int32_t max_context_len, int32_t num_seqs,
                           int32_t num_q_heads, float scale, int32_t partition_size, void *workspace,
                           size_t workspace_bytes, void *out, const pa_cache_desc *cache,
                           int32_t *err_flag, void *stream) {
    const NvtxRange nvtx_range("pa_append_decode");
    pa_status st = check_cache_write(key, value, slot_mapping, num_tokens, key_cache, value_cache, cache);
    if (st != PA_OK) return st;
    DecodeLaunch a;
    st = prepare_decode(query, key_cache, value_cache, block_tables, max_blocks_per_seq, context_lens,
                        max_context_len, num_seqs, num_q_heads, scale, partition_size, workspace,
                        workspace_bytes, out, cache, err_flag, a);
    if (st != PA_OK) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (num_seqs == 0) {
        if (num_tokens == 0) return PA_OK;
        return from_cuda(launch_cache_write(key, value, slot_mapping, num_tokens, key_cache, value_cache,
                                            *cache, err_flag, s));
    }
    const StepWrite w{key, value, slot_mapping, num_tokens, key_cache, value_cache};
    return from_cuda(launch_append_decode(w, a, s));
}

pa_status pa_prefill_chunk(const void *query, const void *key_cache, const void *value_cache,
                           const int32_t *block_tables, int32_t max_blocks_per_seq,
                           const int32_t *context_lens, const int32_t *chunk_lens,
                           int32_t num_seqs, int32_t max_chunk, int32_t num_q_heads, float scale,
                           void *out, const pa_cache_desc *cache, int32_t *err_flag,
                           void *stream) {
    const NvtxRange nvtx_range("pa_prefill_chunk");
    pa_status st = check_cache(cache);
    if (st != PA_OK) return st;
    st = check_group(num_q_heads, cache->num_kv_heads);
    if (st != PA_OK) return st;
    if (cache->dtype != PA_BF16 || cache->head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (num_seqs < 0 || max_chunk < 0 || max_blocks_per_seq < 0) return PA_ERR_INVALID_ARG;
    if (num_seqs == 0 || max_chunk == 0) return PA_OK;
    if (!query || !key_cache || !value_cache || !block_tables || !context_lens || !chunk_lens || !out)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) || !aligned16(out))
        return PA_ERR_INVALID_ARG;
    PrefillLaunch a{};
    a.query = query;
    a.key_cache = key_cache;
    a.value_cache = value_cache;
    a.block_tables = block_tables;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.context_lens = context_lens;
    a.chunk_lens = chunk_lens;
    a.num_seqs = num_seqs;
    a.max_chunk = max_chunk;
    a.num_q_heads = num_q_heads;
    a.scale = scale;
    a.out = out;
    a.cache = *cache;
    a.err = err_flag;
    const cudaError_t e = launch_prefill(a, static_cast<cudaStream_t>(stream));
    if (e == cudaErrorNotSupported) return PA_ERR_UNSUPPORTED;
    return from_cuda(e);
}

pa_status pa_wait(void *stream, const int32_t *err_flag, int32_t timeout_ms, int32_t *flag_out) {
    const NvtxRange nvtx_range("pa_wait");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaEvent_t ev = nullptr;
    if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return PA_ERR_CUDA;
    pa_status st = cudaEventRecord(ev, s) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
    // Poll (never block) so a stream that does not finish returns PA_ERR_TIMEOUT.
    const auto t0 = std::chrono::steady_clock::now();
    while (st == PA_OK) {
        const cudaError_t q = cudaEventQuery(ev);
        if (q == cudaSuccess) break;
        if (q != cudaErrorNotReady) {
            st = PA_ERR_CUDA;
            break;
        }
        const auto ms = std::chrono::duration_cast<std::chrono::milliseconds>(
                            std::chrono::steady_clock::now() - t0).count();
        if (timeout_ms >= 0 && ms > timeout_ms) {
            st = PA_ERR_TIMEOUT;
            break;
        }
        std::this_thread::sleep_for(std::chrono::microseconds(50));
    }
    cudaEventDestroy(ev);
    if (st != PA_OK) return st;
    int32_t host_flag = 0;
    if (err_flag) {
        // the stream is idle now, so this copy cannot wait on earlier work
        if (cudaMemcpyAsync(&host_flag, err_flag, sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
                cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return PA_ERR_CUDA;
    }
    if (flag_out) *flag_out = host_flag;
    if (host_flag & PA_DEVERR_TIMEOUT) return PA_ERR_TIMEOUT;
    if (host_flag) return PA_ERR_DEVICE_INDEX;
    return PA_OK;
}

}  // extern "C"
