/*
 * pa.h -- C ABI of the B200 (sm_100a) paged-KV-cache attention library.
 *
 * The KV cache of one attention layer lives in a pool of fixed-size physical
 * blocks; a per-sequence block table maps logical block j to a physical block.
 * Sources (page title, section):
 *   "vLLM 深度拆解：当大模型推理学会「分页注意力」" (chenxutan.com), 1.1 and 2.1:
 *       K and V of every past token are kept and attended to; they are split
 *       into fixed 16-token blocks placed anywhere in the pool; a block table
 *       maps logical to physical blocks.  2.3: decode is memory-bandwidth bound,
 *       prefill compute bound.  3.1: every step writes the new token's K/V back.
 *       3.3: shared prefix blocks, copy on write.  5.1: chunked prefill.
 *   devpress.csdn.net/amd vLLM v0.6.x teardown, section 核心代码拆解: tensor
 *       layouts (below), the physical block looked up through the table, the
 *       score scaled by `scale`, softmax and a V-weighted sum.  Section
 *       关键设计二: copy-on-write copies a whole shared block into a new one.
 *
 * Layouts (all row-major, all device pointers 16-byte aligned):
 *   key_cache, value_cache  [num_blocks, num_kv_heads, block_size, head_dim]
 *   query, out (decode)     [num_seqs, num_q_heads, head_dim]
 *   query, out (prefill)    [num_seqs, max_chunk, num_q_heads, head_dim]
 *   block_tables            int32 [num_seqs, max_blocks_per_seq]
 *   context_lens            int32 [num_seqs]
 *   slot_mapping            int64 [num_tokens]; slot = block * block_size + offset
 * Query head h reads kv head h / (num_q_heads / num_kv_heads).
 * Supported: dtype PA_F32 or PA_BF16 (cache, query, key/value and out share it),
 * head_dim 64 or 128, block_size 16, num_q_heads / num_kv_heads in {1,2,4,8}.
 * FP8 KV cache (chenxutan 5.3: FP8 KV is close to lossless and halves the bytes;
 * the devpress teardown's architecture figure puts FP8/INT8 quantisation in the
 * kernel layer): dtype PA_FP8_E4M3 stores the pools as one-byte e4m3 codes (OCP
 * 8-bit floating point: bias 7, largest finite 448, S.1111.111 NaN) with one
 * float scale per pool, code = e4m3(fp32(x) / scale) rounded to nearest even and
 * saturated to +-448, value = e4m3 * scale.  key/value inputs, query and out are
 * then bf16.  pa_cache_write, pa_copy_blocks, pa_decode and pa_append_decode take
 * it with head_dim 128; pa_prefill_chunk returns PA_ERR_UNSUPPORTED.
 *
 * Conventions:
 *   - Ownership: the caller owns every buffer, the decode workspace included.
 *     The library allocates no device memory; its module holds two static device
 *     arrays (the scratch of pa_decode_static_scratch, 32 MiB, and the job
 *     counters of pa_prefill_chunk, 8 KB), set up when the library is loaded.
 *   - Asynchrony: each call validates its arguments on the host and enqueues its
 *     kernels on `stream` (a cudaStream_t; NULL = legacy default stream).
 *     PA_OK means "validated and launched", not "finished".
 *   - Host validation errors (PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED) launch
 *     nothing.  A CUDA launch failure returns PA_ERR_CUDA.
 *   - Device-side index faults (a table entry outside the pool, a slot outside
 *     the pool, a context longer than its table, a copy pair outside the pool)
 *     never trap: the kernel ORs a PA_DEVERR_* bit into *err_flag (when
 *     err_flag is not NULL), skips the offending element and carries on.  The
 *     affected outputs are then unspecified.  Read the flag with pa_wait().
 *   - Every wait inside a kernel is bounded; a wait that runs out sets
 *     PA_DEVERR_TIMEOUT and the kernel returns early.
 *   - CUDA graphs: a captured call replays the values its host side chose at
 *     capture time.  Cache writes, block copies, unsplit decodes, split decodes of
 *     fp32 or fp8 pools or head_dim 64, and prefills with more than 8 jobs per
 *     SM (jobs = num_seqs * num_kv_heads * ceil(max_chunk * g / 256)) replay
 *     correctly.  Issue directly, not from a graph: a split decode (pa_decode,
 *     pa_append_decode, pa_decode_static_scratch) of bf16 pools with head_dim 128,
 *     whose shared-prefix detection tags its flags with a per-call value (a replay
 *     would read the previous replay's table comparison), and a pa_prefill_chunk
 *     with at most 8 jobs per SM, whose work counter is tagged per call (a replay
 *     would find its count spent and skip jobs).
 *   - Programmatic dependent launch: the kernels of a call are chained with it,
 *     and the last kernel of a split decode signals early that a dependent may
 *     launch.  A kernel the caller launches right after a call, with
 *     cudaLaunchAttributeProgrammaticStreamSerialization, must call
 *     cudaGridDependencySynchronize() before it reads the call's outputs (stream
 *     order is unchanged for every other kernel and for copies).  The first
 *     kernel of a split bf16 decode is itself launched that way: until the
 *     kernel before it has finished it only reads block_tables and context_lens,
 *     so the kernel just before the call must not write those two after it has
 *     called cudaTriggerProgrammaticLaunchCompletion() (kernels that never call
 *     it count as finished before the call starts).
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

/* Exported entry points (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer, ... */
    PA_ERR_UNSUPPORTED = 2,   /* valid but not built: dtype, head_dim, group size, ... */
    PA_ERR_OOM = 3,           /* block pool exhausted (host block manager) */
    PA_ERR_DEVICE_INDEX = 4,  /* a kernel flagged an out-of-range index (pa_wait) */
    PA_ERR_CUDA = 5,          /* a CUDA runtime call failed */
    PA_ERR_TIMEOUT = 6,       /* pa_wait gave up, or a kernel's bounded wait ran out */
    PA_ERR_NOT_FOUND = 7      /* unknown sequence id (host block manager) */
} pa_status;

typedef enum pa_dtype { PA_F32 = 0, PA_BF16 = 1, PA_FP8_E4M3 = 2 } pa_dtype;

/* Bits a kernel ORs into *err_flag. */
#define PA_DEVERR_BLOCK_ID 1     /* block table entry outside [0, num_blocks) */
#define PA_DEVERR_SLOT 2         /* slot_mapping entry >= num_blocks * block_size */
#define PA_DEVERR_CONTEXT_LEN 4  /* context_len < 0, > max_context_len or > table capacity */
#define PA_DEVERR_PAIR 8         /* copy pair id outside [0, num_blocks) */
#define PA_DEVERR_TIMEOUT 16     /* a bounded in-kernel wait ran out */
#define PA_DEVERR_CHUNK 32       /* chunk_len < 0, > max_chunk or > context_len */

/* The KV pool one call works on. */
typedef struct pa_cache_desc {
    int32_t num_blocks;
    int32_t num_kv_heads;
    int32_t block_size;   /* must be 16 */
    int32_t head_dim;     /* 64 or 128 */
    int32_t dtype;        /* pa_dtype */
    float k_scale;        /* PA_FP8_E4M3: dequantisation scale of the key pool (finite, > 0) */
    float v_scale;        /* PA_FP8_E4M3: the same for the value pool; both ignored otherwise */
} pa_cache_desc;

/* Version of this ABI (bumped on any signature or layout change). */
PA_API int32_t pa_abi_version(void);

/* Human-readable name of a status code (static storage). */
PA_API const char *pa_status_string(pa_status status);

/*
 * KV append through a slot mapping (reshape-and-cache).
 * For every token i < num_tokens with slot = slot_mapping[i] >= 0 and every kv
 * head h:  key_cache[slot / block_size][h][slot % block_size][:] = key[i][h][:]
 * and the same for value.  key/value: [num_tokens, num_kv_heads, head_dim].
 * slot < 0 is padding (skipped).  slot >= num_blocks * block_size sets
 * PA_DEVERR_SLOT and that token is skipped.  Two tokens with the same slot:
 * unspecified which one lands.  num_tokens == 0 launches nothing.
 * PA_FP8_E4M3 pools: key/value are bf16 and each element is stored as
 * e4m3(fp32(x) / k_scale) (v_scale for value), nearest even, saturated.
 * Source: chenxutan 3.1 (write the new token's K/V back into the cache) and 3.3
 * (append_slot: the token goes into the current block).
 */
PA_API pa_status pa_cache_write(const void *key, const void *value, const int64_t *slot_mapping,
                         int32_t num_tokens, void *key_cache, void *value_cache,
                         const pa_cache_desc *cache, int32_t *err_flag, void *stream);

/*
 * Copy-on-Write block copy.  For each pair p < num_pairs, (src, dst) =
 * (src_dst_pairs[2p], src_dst_pairs[2p+1]): block dst of key_cache and of
 * value_cache becomes a copy of block src (every kv head, slot and dim).
 * Pairs must be independent (no dst repeated, no dst that is also a src); the
 * host block manager only emits such pairs.  An id outside [0, num_blocks) sets
 * PA_DEVERR_PAIR and that pair is skipped.  num_pairs == 0 launches nothing.
 * Source: devpress teardown, 关键设计二 (allocate a new block, copy the shared
 * one into it, drop a reference to the old one).
 */
PA_API pa_status pa_copy_blocks(void *key_cache, void *value_cache, const int32_t *src_dst_pairs,
                         int32_t num_pairs, const pa_cache_desc *cache, int32_t *err_flag,
                         void *stream);

/*
 * Checked mode for copy pairs (host function, host pointer): PA_OK when every id of
 * the num_pairs (src, dst) pairs in src_dst_pairs[2 * num_pairs] lies in
 * [0, num_blocks), src != dst, no dst repeats and no block is both a source and a
 * destination -- the conditions under which pa_copy_blocks's result does not depend
 * on the order its pairs run in; PA_ERR_INVALID_ARG otherwise (also for negative
 * counts or a null pointer with num_pairs > 0); PA_ERR_OOM when the host scratch
 * of num_blocks bytes cannot be allocated.  Reads the pairs only; launches nothing.
 * The host block manager only emits valid pairs.
 */
PA_API pa_status pa_check_copy_pairs(const int32_t *src_dst_pairs, int32_t num_pairs, int32_t num_blocks);

/*
 * Bytes of workspace pa_decode needs for a split (partitioned) context:
 * partials of num_seqs * num_q_heads * ceil(max_context_len / partition_size)
 * partitions (head_dim fp32 accumulators plus a running max and sum each), then
 * the shared-prefix group area (a shared-token count, a 16-byte group record and
 * a table-comparison result per sequence, 32 bytes of counts and 512 bytes of
 * flags).  Returns 0 when partition_size <= 0
 * (no split, no workspace).
 */
PA_API size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t partition_size);

/*
 * Number of kernels one pa_decode call with these arguments launches on its
 * stream (for launch accounting): 1 unsplit; 2 split (the
 * partition kernel and the combine); with a split, dtype PA_BF16, head_dim 128 and
 * num_seqs <= 4096 the shared-prefix detection kernel and the tcgen05 group tiles
 * run first (4), and for g = num_q_heads / num_kv_heads <= 4 also the 16-row
 * group kernel for small sibling groups (5).  0 when num_seqs <= 0 or the head
 * counts are not positive.  Pure host function.
 */
PA_API int32_t pa_decode_launches(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                  int32_t head_dim, int32_t dtype, int32_t partition_size);

/*
 * Decode attention over the paged cache, one query token per sequence:
 *   out[s][h][:] = sum_{t < L_s} softmax_t(scale * <query[s][h], K_s[t]>) V_s[t]
 * with L_s = context_lens[s], K_s[t] = key_cache[block_tables[s][t / 16]][h / g]
 * [t % 16][:] (V alike) and g = num_q_heads / num_kv_heads.  L_s == 0 gives 0.
 * Softmax is computed online in fp32 (running max and sum), products and sums in
 * fp32; bf16 outputs are rounded to nearest even from fp32.
 * partition_size == 0: each (sequence, kv head) is one work unit.
 * partition_size > 0 (a multiple of 16): the context is split into partitions of
 * that many tokens (split-K); each partition keeps its running max m_p, sum
 * l_p and unnormalised accumulator o_p in `workspace`, and a second kernel
 * combines them: out = sum_p e^{m_p - M} o_p / sum_p e^{m_p - M} l_p with
 * M = max_p m_p.  Sequences with a single partition are finished by the first
 * kernel.  With a split, bf16 caches, head_dim 128 and num_seqs <= 4096, adjacent
 * sequences whose block tables begin with the same block ids (forked siblings, a
 * common prompt; at least partition_size tokens of full blocks shared with the
 * previous sequence) read those shared full blocks once per group, with all the
 * group's queries against each K/V tile: for g = num_q_heads / num_kv_heads <= 4,
 * groups of 2 to 16 / g members on 16-row tensor-core tiles; groups of at least 4
 * members (at most 128 / g) on the tcgen05 tile kernel.  The result is the same
 * sum, and the shared blocks cross the memory bus once instead of once per
 * sibling (devpress teardown, 关键设计二: siblings point at the same physical
 * blocks).  workspace_bytes must be >= pa_decode_workspace_size(...) for the same
 * num_seqs, num_q_heads, head_dim, max_context_len and partition_size.
 * max_context_len bounds every context_lens[s] (larger sets PA_DEVERR_CONTEXT_LEN
 * and that sequence's outputs are unspecified).  num_seqs <= 16384.
 * Source: chenxutan 2.3 (one query token per step, bandwidth bound); devpress
 * teardown 核心代码拆解 (table lookup per logical block, scaled scores, softmax,
 * weighted V sum).
 */
PA_API pa_status pa_decode(const void *query, const void *key_cache, const void *value_cache,
                    const int32_t *block_tables, int32_t max_blocks_per_seq,
                    const int32_t *context_lens, int32_t max_context_len, int32_t num_seqs,
                    int32_t num_q_heads, float scale, int32_t partition_size, void *workspace,
                    size_t workspace_bytes, void *out, const pa_cache_desc *cache,
                    int32_t *err_flag, void *stream);

/*
 * One decode step in one call: pa_cache_write(key, value, slot_mapping,
 * num_tokens, ...) followed by pa_decode(...) on the same stream, with the same
 * results (the same kernels run).  The write and the decode's shared-prefix
 * detection run side by side and the decode kernels start without a launch gap
 * (programmatic dependent launch); everything that reads the cache still waits
 * for the write.  Copy-on-write pairs must be applied (pa_copy_blocks) before.
 * Both sets of arguments are validated before anything is launched; argument
 * meaning and errors are those of the two calls.  num_tokens == 0 skips the write.
 * Source: chenxutan 3.1 (each step writes the new token's K/V back into the
 * cache, then attends over it).
 */
PA_API pa_status pa_append_decode(const void *key, const void *value, const int64_t *slot_mapping,
                                  int32_t num_tokens, const void *query, void *key_cache,
                                  void *value_cache, const int32_t *block_tables,
                                  int32_t max_blocks_per_seq, const int32_t *context_lens,
                                  int32_t max_context_len, int32_t num_seqs, int32_t num_q_heads,
                                  float scale, int32_t partition_size, void *workspace,
                                  size_t workspace_bytes, void *out, const pa_cache_desc *cache,
                                  int32_t *err_flag, void *stream);

/*
 * pa_decode with its split-K scratch taken from a fixed array inside the library
 * instead of a caller-provided workspace.  The pages have no counterpart: this
 * exists for callers that cannot allocate device memory -- code running inside an
 * allocator's callbacks, in a process whose device memory is owned and capped by
 * another framework, or in a plugin handed only the step's tensors.  Arguments and
 * results are those of pa_decode without workspace/workspace_bytes.
 * Limit: pa_decode_workspace_size(num_seqs, num_q_heads, head_dim,
 * max_context_len, partition_size) must be <= PA_DECODE_STATIC_SCRATCH_BYTES
 * (32 MiB), else PA_ERR_UNSUPPORTED and nothing is launched.  Every GPU that loads
 * the library holds that array until the process exits.
 * The first call on a device looks up the array's device address (with that
 * device current); make it before any stream capture.  No allocation happens.
 * The address is kept for the life of the process: after cudaDeviceReset (or
 * anything else that destroys the device's primary context) the process must be
 * restarted before this entry point is called again on that device.
 * All calls share the one array and it keeps the last call's contents; nothing in
 * it needs to start at zero.  Calls whose kernels overlap on the GPU (different
 * streams, no ordering between them) race on the array and give wrong results:
 * order them on one stream or with events.
 */
#define PA_DECODE_STATIC_SCRATCH_BYTES (32u << 20)
PA_API pa_status pa_decode_static_scratch(const void *query, const void *key_cache,
                                          const void *value_cache, const int32_t *block_tables,
                                          int32_t max_blocks_per_seq, const int32_t *context_lens,
                                          int32_t max_context_len, int32_t num_seqs,
                                          int32_t num_q_heads, float scale, int32_t partition_size,
                                          void *out, const pa_cache_desc *cache, int32_t *err_flag,
                                          void *stream);

/*
 * Causal chunked prefill against the paged cache.  Sequence s has
 * C_s = chunk_lens[s] new query rows, the last C_s positions of its context of
 * L_s = context_lens[s] tokens (their K/V already written with pa_cache_write).
 * Row i < C_s sits at position p = L_s - C_s + i and
 *   out[s][i][h][:] = sum_{t <= p} softmax_t(scale * <query[s][i][h], K_s[t]>) V_s[t].
 * query/out: [num_seqs, max_chunk, num_q_heads, head_dim]; rows i >= C_s of out
 * are not written.  Requires dtype PA_BF16 and head_dim 128 (tcgen05 tensor-core
 * tiles, bf16 operands, fp32 accumulation in tensor memory).
 * A speculative-decoding verify step is the same operation: each sequence appends
 * its k_s draft tokens (pa_cache_write), then the k_s new positions attend
 * causally with chunk_lens[s] = k_s (chenxutan 5.4, speculative decoding: the
 * target model checks several proposed tokens in one pass).
 * Work distribution (no effect on results): a job is (sequence, kv head, 256
 * packed rows).  With at most 8 jobs per SM they are handed out from a work
 * counter, one of a static pool of 1,024; each call tags its counter with a
 * per-process ticket, so calls need no ordering between them and nothing is
 * reset.  A call whose kernel still runs after 1,024 later pa_prefill_chunk
 * calls of the process have started (impossible on one stream) sets
 * PA_DEVERR_TIMEOUT and its outputs are unspecified.  With more jobs per SM the
 * order is a fixed round robin.
 * Source: chenxutan 2.3 (prefill computes a whole prompt and is compute bound)
 * and 4.3/5.1 (long prompts are cut into chunks that run between decodes).
 */
PA_API pa_status pa_prefill_chunk(const void *query, const void *key_cache, const void *value_cache,
                           const int32_t *block_tables, int32_t max_blocks_per_seq,
                           const int32_t *context_lens, const int32_t *chunk_lens,
                           int32_t num_seqs, int32_t max_chunk, int32_t num_q_heads, float scale,
                           void *out, const pa_cache_desc *cache, int32_t *err_flag,
                           void *stream);

/*
 * Wait for `stream` to finish (polling, at most timeout_ms milliseconds) and read
 * the device error flag.  *flag_out (if not NULL) receives the flag value.
 * Returns PA_OK, PA_ERR_DEVICE_INDEX (flag has an index bit), PA_ERR_TIMEOUT
 * (stream still busy, or the flag has PA_DEVERR_TIMEOUT) or PA_ERR_CUDA.
 * err_flag may be NULL (then only the wait is done).  Not for use during
 * stream capture.
 */
PA_API pa_status pa_wait(void *stream, const int32_t *err_flag, int32_t timeout_ms, int32_t *flag_out);

/*
 * Bound, in nanoseconds, of every wait inside the kernels launched from now on by
 * this process (mbarrier hand-overs between the warps of a CTA); 0 restores the
 * default of one second.  Returns the previous bound.  A wait that runs out sets
 * PA_DEVERR_TIMEOUT in *err_flag, and the kernel stops its work, waits (with the
 * default bound) for the copies and tensor-core operations it has in flight,
 * releases its tensor memory and returns; the outputs of that call are then
 * unspecified and later calls are unaffected.  It exists to exercise that path:
 * a bound of a few nanoseconds makes ordinary waits run out.  Not a per-call or
 * per-thread setting: it applies to launches from every host thread.
 * Source: none on the pages (failure handling of this library).
 */
PA_API uint64_t pa_set_wait_timeout_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
