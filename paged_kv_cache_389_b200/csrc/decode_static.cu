// pa_decode_static_scratch: the split-K decode of pa_decode with its scratch
// taken from a fixed array that lives in the library itself, for callers that
// cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is off limits -- inside a custom
// allocator's own callbacks, in a process whose memory pool is owned and capped
// by another framework, or in plugins that are handed only the tensors of a step
// and no allocator.  Such a caller still passes query, cache, tables, lengths and
// output; only the split-K partials (per-partition running max, running sum and
// unnormalised accumulator) go to the array below.
//
// Set-up: the device address of the array is looked up once per device, with
// that device current, on the first call made on it (cudaGetSymbolAddress);
// make that first call before any stream capture.  Nothing here allocates.
#include <cstdint>
#include <mutex>

#include "pa_trace.h"
#include "pa_common.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_decode_scratch[PA_DECODE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_decode_scratch on the current device (nullptr on failure).
void *scratch_address(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> g(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr) return nullptr;
        g_scratch_addr[dev] = ptr;
    }
    return g_scratch_addr[dev];
}

}  // namespace
}  // namespace pa

extern "C" pa_status pa_decode_static_scratch(
    const void *query, const void *key_cache, const void *value_cache, const int32_t *block_tables,
    int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t max_context_len,
    int32_t num_seqs, int32_t num_q_heads, float scale, int32_t partition_size, void *out,
    const pa_cache_desc *cache, int32_t *err_flag, void *stream) {
    const pa::NvtxRange nvtx_range("pa_decode_static_scratch");
    if (!cache || partition_size < 0) return PA_ERR_INVALID_ARG;
    const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, cache->head_dim,
                                                 max_context_len, partition_size);
    if (need > (size_t)PA_DECODE_STATIC_SCRATCH_BYTES) return PA_ERR_UNSUPPORTED;
    void *ws = nullptr;
    if (need > 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
        ws = pa::scratch_address(dev);
        if (!ws) return PA_ERR_CUDA;
    }
    // Same validation and kernels as pa_decode; only the workspace differs.  No
    // part of the array needs to start at zero: every partial the reduce step
    // reads is written earlier in the same call.
    return pa_decode(query, key_cache, value_cache, block_tables, max_blocks_per_seq, context_lens,
                     max_context_len, num_seqs, num_q_heads, scale, partition_size, ws, need, out,
                     cache, err_flag, stream);
}
