// Chunked-prefill attention against the paged KV cache on 5th-generation tensor
// cores (tcgen05.mma, accumulators in tensor memory).
//
// What is computed (include/pa.h): sequence s has C_s query rows, the last C_s
// positions of its L_s-token context; row i sits at position p = L_s - C_s + i
// and attends to keys 0..p (causal), K/V read through the block table.
// Sources: "vLLM 深度拆解" (chenxutan) 2.3 (prefill processes a whole prompt and is
// compute bound) and 4.3/5.1 (long prompts are cut into chunks interleaved with
// decode); devpress vLLM v0.6.x teardown, 核心代码拆解 (paged K/V via the table).
//
// Tile: one CTA computes a 128-row query tile of one (sequence, kv head): the g
// query heads of that kv head are packed into the rows (row = chunk row * g +
// head), so every K/V byte staged in shared memory serves all g heads.  The CTA
// walks the keys in tiles of 128 (8 blocks of 16) up to the tile's last position.
//   S   = Q K^T      tcgen05.mma kind::f16, M=128, N=128 keys, K=16 x 8, -> TMEM
//   P   = softmax    online, fp32, one query row per thread (tcgen05.ld from TMEM)
//   O  += P V        tcgen05.mma, A = P (bf16, smem), B = V (MN-major), -> TMEM
// Warp roles: warps 0-3 load (16-byte cp.async into 128-byte-swizzled layouts:
// Q and K K-major, V MN-major, the canonical layouts the MMA descriptors name),
// warps 4-11 run the softmax (warp w: TMEM lanes 32*(w%4)..+31, one 64-column
// half of the tile), warp 12 owns the tensor memory and issues the MMAs from one
// thread.  K and V tiles have separate two-stage rings and loader warps (0-1: Q
// and K, 2-3: V), so a K stage is refilled as soon as its QK is done; the stages
// are handed over with mbarriers; every wait is bounded and an abort still frees
// the tensor memory.
#include <cstring>

#include "pa_common.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kD = 128;              // head_dim (bf16 only)
constexpr int kTileM = 128;          // query rows per CTA
constexpr int kTileN = 128;          // keys per KV tile
constexpr int kThreads = 13 * 32;    // 4 load warps, 8 softmax warps, 1 MMA warp
constexpr int kMmaWarp = 12;
constexpr int kSoftmaxThreads = 256;
constexpr uint32_t kTmemCols = 256;  // S: columns 0..127, O: 128..255

// shared memory (offsets from a 1024-byte aligned base)
constexpr uint32_t kHalf = kTileM * 128;           // one 64-column half of a 128-row tile
constexpr uint32_t kTileBytes = 2 * kHalf;         // 32 KB
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTileBytes;     // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTileBytes; // 2 stages
constexpr uint32_t kOffP = kOffV + 2 * kTileBytes;
constexpr uint32_t kOffBar = kOffP + kTileBytes;
constexpr uint32_t kOffTab = kOffBar + 24 * 8;     // 24 mbarriers
constexpr uint32_t kOffMisc = kOffTab + 2 * 2 * 8 * 4;  // [K, V loader][2 stages][8 table entries]
constexpr uint32_t kOffRed = kOffMisc + 16;          // row-max halves [2 tiles][2 halves][128 rows]
constexpr uint32_t kOffLsum = kOffRed + 2 * 2 * 128 * 4;  // row-sum halves [2][128]
constexpr uint32_t kOffGcum = kOffLsum + 2 * 128 * 4;  // group units: units before each group
constexpr int kMaxGroups = 2048;                     // a group has >= 2 (in fact >= 4) of <= 4096 sequences
constexpr size_t kSmemBytes = 1024 + kOffGcum + kMaxGroups * 4;

struct Params {
    const unsigned char *q;
    const unsigned char *kc;
    const unsigned char *vc;
    const int32_t *tables;
    const int32_t *lens;
    const int32_t *chunks;
    unsigned char *out;
    int32_t *err;
    int32_t max_blocks;
    int32_t num_seqs;
    int32_t max_chunk;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t num_blocks;
    float scale_log2;
    // shared-prefix group units of the split decode
    const int4 *groups;    // (first seq, members, shared partitions, units before)
    const int32_t *meta;   // [0] groups, [1] units
    float *ws_acc;
    float2 *ws_ml;
    int32_t part_tokens;
    int32_t max_parts;
    unsigned long long wait_ns;  // bound of every in-kernel wait
};

// ---- tcgen05 wrappers --------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
          "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
          "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
          "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
          "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
          "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
          "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
          "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
          "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
          "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
          "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: 128-byte swizzle, start/LBO/SBO in 16-byte units,
// descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator, M=128, N=128.
constexpr uint32_t idesc_bf16(bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(kTileN >> 3) << 17) |
           ((uint32_t)(kTileM >> 4) << 24);
}

// Byte offset of 16-byte chunk c (0..15) of row r in a 128-row tile stored as
// two 64-column halves of 128-byte rows with the 128-byte swizzle.
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return (uint32_t)((c >> 3) * kHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Bounded mbarrier wait honouring the CTA abort flag (pa_common.cuh).
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort, int32_t *err,
                                         unsigned long long limit_ns) {
    return mbar_wait_bounded(bar, parity, abort, err, limit_ns);
}

// One 128-row query tile against a run of keys.  Row r (0..127) holds query head
// h*G + r%G of row group r/G; row groups are q_row_stride bytes apart.  Keys are
// 0..nkeys-1 through the table entries starting at trow; row r may see keys
// 0..lim0 + lim_step*(r/G) (lim_step 1: causal prefill; 0: every key).
struct Job {
    const unsigned char *q;  // query row group 0, head h*G
    int64_t q_row_stride;
    int nrows;               // rows r < nrows are real (the rest are zero)
    const int32_t *trow;
    int nkeys;
    int lim0, lim_step;
    int ntiles;
    int h;
    // output: prefill -> normalised bf16 rows at out (same strides as q);
    // group -> fp32 partials of workspace row (first + r/G)*Hq + h*G + r%G, slot part
    unsigned char *out;
    int first, part;
};

template <int G, bool kGroup>
__device__ __forceinline__ Job group_job(const Params &p, const int *gcum, int ngroups, int u) {
    Job jb;
    int lo = 0, hi = ngroups;  // gcum[lo] <= u < gcum[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (gcum[mid] <= u) lo = mid; else hi = mid;
    }
    const int4 gr = __ldg(&p.groups[lo]);  // (first seq, members, shared partitions, units before)
    const int r = u - gr.w;
    jb.h = r % p.num_kv_heads;
    jb.part = r / p.num_kv_heads;  // partition = workspace slot
    jb.first = gr.x;
    const int64_t hs = (int64_t)kD * 2;
    jb.q_row_stride = (int64_t)p.num_q_heads * hs;
    jb.q = p.q + (int64_t)gr.x * jb.q_row_stride + (int64_t)jb.h * G * hs;
    jb.nrows = gr.y * G;
    jb.trow = p.tables + (int64_t)gr.x * p.max_blocks + (int64_t)jb.part * (p.part_tokens / kBlockSize);
    jb.nkeys = p.part_tokens;
    jb.lim0 = p.part_tokens - 1;
    jb.lim_step = 0;
    jb.ntiles = (p.part_tokens + kTileN - 1) / kTileN;
    jb.out = nullptr;
    return jb;
}

// Prefill: one CTA per (query tile, kv head, sequence).  Shared-prefix groups of
// the split decode (kGroup): a persistent CTA loops over the group units (group,
// partition, kv head) listed by the decode's detection kernel; the rows are the
// members' queries, the keys one partition lying inside the blocks all members
// share, and the result is the partition's (m, l, unnormalised O) in workspace
// slot p of every member -- the same partial the per-sequence kernel would write.
// (Units spanning all of a group's partitions were measured: they balance worse
// over the SMs and were slower.)
template <int G, bool kGroup>
__global__ void __launch_bounds__(kThreads, 1) attn_tile_kernel(const __grid_constant__ Params p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const uint32_t sbase = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *q_full = bars + 0;
    uint64_t *k_full = bars + 1;    // [2] K tile landed
    uint64_t *k_empty = bars + 3;   // [2] its QK is done: the K stage may be refilled
    uint64_t *v_full = bars + 5;    // [2] V tile landed
    uint64_t *v_empty = bars + 7;   // [2] its PV is done: the V stage may be refilled
    uint64_t *s_full = bars + 9;
    uint64_t *p_full = bars + 10;
    uint64_t *pv_done = bars + 11;
    uint64_t *mma_idle = bars + 12;
    uint64_t *red_full = bars + 13;  // [2]
    uint64_t *l_full = bars + 15;
    uint64_t *q_empty = bars + 16;  // a unit's last QK is done: Q may be rewritten
    uint64_t *o_free = bars + 17;   // the softmax warps have read a unit's O
    int *tab = reinterpret_cast<int *>(smem + kOffTab);  // [K, V loader][2][8]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
    volatile int *go = reinterpret_cast<volatile int *>(smem + kOffMisc + 8);  // [K, V loader]
    int *gcum = reinterpret_cast<int *>(smem + kOffGcum);
    const int64_t hs = (int64_t)kD * 2;  // bytes per (row, head)

    // ---- the work of this CTA
    int u0 = 0, nunits = 1, ngroups = 0;
    Job jb;
    if constexpr (kGroup) {
        // launched behind the detection kernel: its group list must be complete;
        // then the per-sequence decode may start (it reads only detection output)
        grid_dep_wait();
        grid_dep_launch();
        nunits = __ldg(p.meta + 1);
        ngroups = __ldg(p.meta);
        u0 = blockIdx.x;
        if (u0 >= nunits) return;
    } else {
        constexpr int kRowsPerTile = kTileM / G;
        const int s = blockIdx.z, h = blockIdx.y;
        const int i0 = blockIdx.x * kRowsPerTile;
        const int L = __ldg(p.lens + s), C = __ldg(p.chunks + s);
        // validate once; an invalid sequence is skipped (flagged by its first tile)
        if (C < 0 || C > p.max_chunk || C > L || (int64_t)L > (int64_t)p.max_blocks * kBlockSize) {
            if (blockIdx.x == 0 && h == 0 && threadIdx.x == 0) flag_error(p.err, PA_DEVERR_CHUNK);
            return;
        }
        if (i0 >= C) return;
        const int start = L - C;
        const int last_row = min(C, i0 + kRowsPerTile) - 1;
        jb.h = h;
        jb.q_row_stride = (int64_t)p.num_q_heads * hs;
        jb.q = p.q + ((int64_t)s * p.max_chunk + i0) * jb.q_row_stride + (int64_t)h * G * hs;
        jb.out = p.out + ((int64_t)s * p.max_chunk + i0) * jb.q_row_stride + (int64_t)h * G * hs;
        jb.nrows = (last_row - i0 + 1) * G;
        jb.trow = p.tables + (int64_t)s * p.max_blocks;
        jb.nkeys = L;
        jb.lim0 = start + i0;
        jb.lim_step = 1;
        jb.ntiles = (start + last_row + 1 + kTileN - 1) / kTileN;  // keys 0..start+last_row
        jb.first = jb.part = 0;
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(q_full, 64);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&k_full[i], 64);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_full[i], 64);
            mbar_init(&v_empty[i], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(p_full, kSoftmaxThreads);
        mbar_init(pv_done, 1);
        mbar_init(mma_idle, 1);
        mbar_init(q_empty, 1);
        mbar_init(o_free, kSoftmaxThreads);
        mbar_init(&red_full[0], kSoftmaxThreads);
        mbar_init(&red_full[1], kSoftmaxThreads);
        mbar_init(l_full, kSoftmaxThreads);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if constexpr (kGroup) {
        for (int k = threadIdx.x; k < ngroups; k += kThreads) gcum[k] = __ldg(&p.groups[k].w);
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tO = tmem + 128;

    // Barrier phases run on across units: tile jt = tbase + j of the CTA uses
    // stage jt & 1; q_full, q_empty, l_full and o_free complete once per unit.
    // Units follow one another without a CTA barrier: the loader streams the
    // next unit's Q (after q_empty) and K/V tiles while the current one is
    // still being computed, and the MMA starts the next unit's PV only after
    // o_free.  Every wait is bounded; after an abort the remaining units fall
    // through their (failing) waits.
    int tbase = 0, nu = 0;
    for (int u = u0; u < nunits; u += (kGroup ? gridDim.x : 1), ++nu) {
        if constexpr (kGroup) jb = group_job<G, kGroup>(p, gcum, ngroups, u);
        if (warp < 4) {
            // -------------------------------------------------------- loaders
            // Warps 0-1 stream Q and K, warps 2-3 stream V, each group through
            // its own two-stage ring, two tiles deep.  A K stage comes back as
            // soon as its QK is done, so K runs ahead of V.  Within a group one
            // thread waits and the decision reaches the others through shared
            // memory behind the group's named barrier.
            const bool is_k = warp < 2;
            const int t = threadIdx.x & 63;
            const int gbar = is_k ? 1 : 2;
            volatile int *gw = go + (is_k ? 0 : 1);
            int *gtab = tab + (is_k ? 0 : 16);
            uint64_t *full = is_k ? k_full : v_full;
            uint64_t *empty = is_k ? k_empty : v_empty;
            const uint32_t ring_s = sbase + (is_k ? kOffK : kOffV);
            unsigned char *ring = smem + (is_k ? kOffK : kOffV);
            const unsigned char *src0 = is_k ? p.kc : p.vc;
            bool q_ok = true;
            if (is_k) {
                // the previous unit's QK must be done with Q
                if (t == 0) *gw = (nu == 0 || wait_bar(q_empty, (nu - 1) & 1, abort_flag, p.err, p.wait_ns)) ? 1 : 0;
                named_barrier(gbar, 64);
                q_ok = *gw != 0;
                named_barrier(gbar, 64);  // *gw is rewritten by the first tile issue
                // Q tile: row r = (row group r / G, head r % G); 16 chunks of 16 bytes per row
                for (int idx = t; q_ok && idx < kTileM * 16; idx += 64) {
                    const int r = idx >> 4, c = idx & 15;
                    const uint32_t dst = sbase + kOffQ + swz(r, c);
                    if (r < jb.nrows)
                        cp_async16(dst, jb.q + (int64_t)(r / G) * jb.q_row_stride + (int64_t)(r % G) * hs + c * 16);
                    else
                        *reinterpret_cast<uint4 *>(smem + kOffQ + swz(r, c)) = make_uint4(0, 0, 0, 0);
                }
                cp_async_commit();
            }
            // table entry of block t of tile j (threads t < 8; -1: past the keys),
            // loaded one tile ahead so its latency hides behind the current tile
            auto table_entry = [&](int j) -> int {
                const int b = j * 8 + t;
                return (t < 8 && b * kBlockSize < jb.nkeys) ? __ldg(jb.trow + b) : -1;
            };
            int next_e = table_entry(0);
            auto issue_tile = [&](int j) -> bool {
                const int jt = tbase + j, st = jt & 1;
                if (t == 0) *gw = (jt < 2 || wait_bar(&empty[st], ((jt >> 1) - 1) & 1, abort_flag, p.err, p.wait_ns)) ? 1 : 0;
                if (t < 8) {
                    int e = next_e;
                    if (j * 8 + t < (jb.nkeys + kBlockSize - 1) / kBlockSize && (e < 0 || e >= p.num_blocks)) {
                        flag_error(p.err, PA_DEVERR_BLOCK_ID);
                        e = -1;
                    }
                    gtab[st * 8 + t] = e;
                    next_e = table_entry(j + 1);
                }
                named_barrier(gbar, 64);
                const bool ok = *gw != 0;
                if (ok) {
                    const uint32_t dst0 = ring_s + st * kTileBytes;
                    unsigned char *gen0 = ring + st * kTileBytes;
                    for (int idx = t; idx < kTileN * 16; idx += 64) {
                        const int n = idx >> 4, c = idx & 15;
                        const int key = j * kTileN + n;
                        const int blk = gtab[st * 8 + (n >> 4)];
                        const uint32_t off = swz(n, c);
                        if (blk >= 0 && key < jb.nkeys) {
                            const int64_t src = (((int64_t)blk * p.num_kv_heads + jb.h) * kBlockSize + (n & 15)) * hs + c * 16;
                            cp_async16(dst0 + off, src0 + src);
                        } else {  // past the keys or a bad id: zeros (0 * garbage must not reach the sums)
                            *reinterpret_cast<uint4 *>(gen0 + off) = make_uint4(0, 0, 0, 0);
                        }
                    }
                }
                cp_async_commit();
                named_barrier(gbar, 64);  // gtab and *gw are rewritten by the next issue
                return ok;
            };
            bool ok = q_ok && jb.ntiles > 0 && issue_tile(0);
            for (int j = 0; ok && j < jb.ntiles; ++j) {
                const bool more = j + 1 < jb.ntiles;
                if (more && !issue_tile(j + 1)) break;
                // copy groups so far: (Q,) tiles 0..j (+ j+1): all but the newest are done
                if (more) cp_async_wait<1>(); else cp_async_wait<0>();
                fence_proxy_async_smem();
                if (is_k && j == 0) mbar_arrive(q_full);
                mbar_arrive(&full[(tbase + j) & 1]);
            }
            cp_async_wait<0>();  // nothing may land after an abort
        } else if (warp == kMmaWarp) {
            // -------------------------------------------------------- MMA issuer
            if (lane == 0) {
                constexpr uint32_t kIdQK = idesc_bf16(false), kIdPV = idesc_bf16(true);
                bool ok = wait_bar(q_full, nu & 1, abort_flag, p.err, p.wait_ns);
                for (int j = 0; ok && j < jb.ntiles; ++j) {
                    const int jt = tbase + j, st = jt & 1;
                    if (!wait_bar(&k_full[st], (jt >> 1) & 1, abort_flag, p.err, p.wait_ns)) break;
                    tc_fence_after();
                    const uint32_t qa = sbase + kOffQ, ka = sbase + kOffK + st * kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk) {
                        const uint32_t koff = (kk & 3) * 32 + (kk >> 2) * kHalf;
                        tc_mma(tS, smem_desc(qa + koff, 16, 1024), smem_desc(ka + koff, 16, 1024), kIdQK, kk > 0);
                    }
                    tc_commit(s_full);
                    tc_commit(&k_empty[st]);
                    if (j == jb.ntiles - 1) tc_commit(q_empty);
                    if (!wait_bar(p_full, jt & 1, abort_flag, p.err, p.wait_ns)) break;
                    // the first PV overwrites O: the previous unit's O must have been read
                    if (j == 0 && nu > 0 && !wait_bar(o_free, (nu - 1) & 1, abort_flag, p.err, p.wait_ns)) break;
                    if (!wait_bar(&v_full[st], (jt >> 1) & 1, abort_flag, p.err, p.wait_ns)) break;
                    tc_fence_after();
                    const uint32_t pa_ = sbase + kOffP, va = sbase + kOffV + st * kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < kTileN / 16; ++kk) {
                        const uint32_t poff = (kk & 3) * 32 + (kk >> 2) * kHalf;
                        tc_mma(tO, smem_desc(pa_ + poff, 16, 1024), smem_desc(va + kk * 2048, kHalf, 1024), kIdPV,
                               j > 0 || kk > 0);
                    }
                    tc_commit(pv_done);
                    tc_commit(&v_empty[st]);
                }
            }
            __syncwarp();
        } else {
            // -------------------------------------------------------- softmax
            // Warp w owns TMEM lane quadrant w % 4 (rows 32*(w%4)..+31) and column
            // half hf of S, O and P.  The two halves of a row trade their partial
            // maxima through shared memory each tile (bounded mbarrier) and add
            // their partial sums at the end.
            const int qd = warp & 3, hf = (warp - 4) >> 2;
            const int r = qd * 32 + lane;                // query row = TMEM lane
            const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
            const uint32_t cS = tS + lane_off + hf * 64, cO = tO + lane_off + hf * 64;
            float *red = reinterpret_cast<float *>(smem + kOffRed);    // [2][2][128]
            float *lsum = reinterpret_cast<float *>(smem + kOffLsum);  // [2][128]
            const bool row_ok = r < jb.nrows;
            const bool warp_rows = __any_sync(kFull, row_ok);         // any real row in this warp
            const int lim = jb.lim0 + jb.lim_step * (r / G);          // last key this row may see
            float m = -INFINITY, l = 0.f;
            bool live = true;
            for (int j = 0; j < jb.ntiles; ++j) {
                const int jt = tbase + j;
                const int key0 = j * kTileN + hf * 64;                // first key of this half
                // the whole half is visible to every row of the warp: no per-key test
                const bool open = __all_sync(kFull, row_ok && lim >= key0 + 63);
                live = live && wait_bar(s_full, jt & 1, abort_flag, p.err, p.wait_ns);
                live = __all_sync(kFull, live);
                if (!live) break;
                tc_fence_after();
                // pass 1: partial row max of the scaled, masked scores
                float mx = -INFINITY;
                if (warp_rows) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        float sv[32];
                        tmem_ld32(cS + c * 32, sv);
                        tmem_wait_ld();
                        if (open) {
#pragma unroll
                            for (int k = 0; k < 32; ++k) mx = fmaxf(mx, sv[k] * p.scale_log2);
                        } else {
#pragma unroll
                            for (int k = 0; k < 32; ++k)
                                if (row_ok && key0 + c * 32 + k <= lim) mx = fmaxf(mx, sv[k] * p.scale_log2);
                        }
                    }
                }
                float *rb = red + (jt & 1) * 256;
                rb[hf * 128 + r] = mx;
                mbar_arrive(&red_full[jt & 1]);
                live = wait_bar(&red_full[jt & 1], (jt >> 1) & 1, abort_flag, p.err, p.wait_ns);
                live = __all_sync(kFull, live);
                if (!live) break;
                mx = fmaxf(rb[r], rb[128 + r]);
                const float m_new = fmaxf(m, mx);
                const float m_use = m_new == -INFINITY ? 0.f : m_new;
                const float alpha = fast_exp2(m - m_use);
                if (j > 0) {
                    // P and O are still in use by the previous tile's PV
                    live = wait_bar(pv_done, (jt - 1) & 1, abort_flag, p.err, p.wait_ns);
                    live = __all_sync(kFull, live);
                    if (!live) break;
                    tc_fence_after();
                    if (warp_rows && __any_sync(kFull, alpha != 1.f)) {
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            float ov[32];
                            tmem_ld32(cO + c * 32, ov);
                            tmem_wait_ld();
#pragma unroll
                            for (int k = 0; k < 32; ++k) ov[k] *= alpha;
                            tmem_st32(cO + c * 32, ov);
                        }
                        tmem_wait_st();
                    }
                }
                // pass 2: P = 2^(s - m) as bf16 into this half of the K-major swizzled A tile
                float rs = 0.f;
                if (warp_rows) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        float sv[32];
                        tmem_ld32(cS + c * 32, sv);
                        tmem_wait_ld();
                        if (open) {
#pragma unroll
                            for (int k = 0; k < 32; ++k) {
                                sv[k] = fast_exp2(sv[k] * p.scale_log2 - m_use);
                                rs += sv[k];
                            }
                        } else {
#pragma unroll
                            for (int k = 0; k < 32; ++k) {
                                sv[k] = (row_ok && key0 + c * 32 + k <= lim) ? fast_exp2(sv[k] * p.scale_log2 - m_use) : 0.f;
                                rs += sv[k];
                            }
                        }
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float *x = &sv[q * 8];
                            const uint4 w = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                                                       pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
                            *reinterpret_cast<uint4 *>(smem + kOffP + swz(r, hf * 8 + c * 4 + q)) = w;
                        }
                    }
                }
                l = l * alpha + rs;
                m = m_new;
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(p_full);
            }
            if (live) live = wait_bar(pv_done, (tbase + jb.ntiles - 1) & 1, abort_flag, p.err, p.wait_ns);
            live = __all_sync(kFull, live);
            if (live) {
                lsum[hf * 128 + r] = l;
                mbar_arrive(l_full);
                live = wait_bar(l_full, nu & 1, abort_flag, p.err, p.wait_ns);
                live = __all_sync(kFull, live);
            }
            if (live && warp_rows) {
                tc_fence_after();
                const float lt = lsum[r] + lsum[128 + r];
                if constexpr (kGroup) {
                    const int64_t wrow = ((int64_t)(jb.first + r / G) * p.num_q_heads + jb.h * G + r % G) * p.max_parts + jb.part;
                    float *dst = p.ws_acc + wrow * kD + hf * 64;
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        float ov[32];
                        tmem_ld32(cO + c * 32, ov);
                        tmem_wait_ld();
                        if (row_ok) {
#pragma unroll
                            for (int k = 0; k < 32; k += 4)
                                *reinterpret_cast<float4 *>(dst + c * 32 + k) = make_float4(ov[k], ov[k + 1], ov[k + 2], ov[k + 3]);
                        }
                    }
                    if (row_ok && hf == 0) p.ws_ml[wrow] = make_float2(m, lt);
                } else {
                    const float inv = lt > 0.f ? 1.f / lt : 0.f;
                    unsigned char *dst = jb.out + (int64_t)(r / G) * jb.q_row_stride + (int64_t)(r % G) * hs + hf * 128;
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        float ov[32];
                        tmem_ld32(cO + c * 32, ov);
                        tmem_wait_ld();
                        if (row_ok) {
#pragma unroll
                            for (int k = 0; k < 32; k += 8) {
                                const uint4 w = make_uint4(pack_bf16x2(ov[k] * inv, ov[k + 1] * inv),
                                                           pack_bf16x2(ov[k + 2] * inv, ov[k + 3] * inv),
                                                           pack_bf16x2(ov[k + 4] * inv, ov[k + 5] * inv),
                                                           pack_bf16x2(ov[k + 6] * inv, ov[k + 7] * inv));
                                *reinterpret_cast<uint4 *>(dst + (c * 32 + k) * 2) = w;
                            }
                        }
                    }
                }
            }
            // this unit's O has been read (or was never needed): the MMA may
            // overwrite it with the next unit's first PV
            if (live) {
                tc_fence_before();
                mbar_arrive(o_free);
            }
        }
        tbase += jb.ntiles;
    }
    if (warp == kMmaWarp && lane == 0) {
        // everything issued has completed once this arrives
        tc_commit(mma_idle);
        if (!mbar_wait_drain(mma_idle, 0)) {
            *abort_flag = 1;
            flag_error(p.err, PA_DEVERR_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int G>
cudaError_t launch_g(const PrefillLaunch &a, const Params &prm, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(attn_tile_kernel<G, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    constexpr int rows = kTileM / G;
    dim3 grid((unsigned)((a.max_chunk + rows - 1) / rows), (unsigned)a.cache.num_kv_heads, (unsigned)a.num_seqs);
    attn_tile_kernel<G, false><<<grid, kThreads, kSmemBytes, stream>>>(prm);
    return cudaGetLastError();
}

template <int G>
cudaError_t launch_group_g(const Params &prm, int sms, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(attn_tile_kernel<G, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    return launch_after(attn_tile_kernel<G, true>, dim3((unsigned)sms), dim3(kThreads), kSmemBytes, stream,
                        static_cast<const Params &>(prm));
}

}  // namespace

cudaError_t launch_prefill(const PrefillLaunch &a, cudaStream_t stream) {
    static_assert(kSmemBytes <= 232448, "prefill smem over the sm_100 limit");
    if (a.cache.dtype != PA_BF16 || a.cache.head_dim != kD) return cudaErrorNotSupported;
    if (a.num_seqs > 65535) return cudaErrorNotSupported;
    Params prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.q = static_cast<const unsigned char *>(a.query);
    prm.kc = static_cast<const unsigned char *>(a.key_cache);
    prm.vc = static_cast<const unsigned char *>(a.value_cache);
    prm.tables = a.block_tables;
    prm.lens = a.context_lens;
    prm.chunks = a.chunk_lens;
    prm.out = static_cast<unsigned char *>(a.out);
    prm.err = a.err;
    prm.max_blocks = a.max_blocks_per_seq;
    prm.num_seqs = a.num_seqs;
    prm.max_chunk = a.max_chunk;
    prm.num_q_heads = a.num_q_heads;
    prm.num_kv_heads = a.cache.num_kv_heads;
    prm.num_blocks = a.cache.num_blocks;
    prm.scale_log2 = a.scale * kLog2e;
    prm.wait_ns = wait_limit_ns();
    switch (a.num_q_heads / a.cache.num_kv_heads) {
        case 1: return launch_g<1>(a, prm, stream);
        case 2: return launch_g<2>(a, prm, stream);
        case 4: return launch_g<4>(a, prm, stream);
        case 8: return launch_g<8>(a, prm, stream);
        default: return cudaErrorNotSupported;
    }
}

cudaError_t launch_group_tiles(const GroupTileLaunch &a, int sms, cudaStream_t stream) {
    Params prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.q = static_cast<const unsigned char *>(a.query);
    prm.kc = static_cast<const unsigned char *>(a.key_cache);
    prm.vc = static_cast<const unsigned char *>(a.value_cache);
    prm.tables = a.block_tables;
    prm.err = a.err;
    prm.max_blocks = a.max_blocks_per_seq;
    prm.num_q_heads = a.num_q_heads;
    prm.num_kv_heads = a.num_kv_heads;
    prm.num_blocks = a.num_blocks;
    prm.scale_log2 = a.scale * kLog2e;
    prm.groups = a.groups;
    prm.meta = a.meta;
    prm.ws_acc = a.ws_acc;
    prm.ws_ml = a.ws_ml;
    prm.part_tokens = a.partition_size;
    prm.max_parts = a.max_partitions;
    prm.wait_ns = wait_limit_ns();
    switch (a.num_q_heads / a.num_kv_heads) {
        case 1: return launch_group_g<1>(prm, sms, stream);
        case 2: return launch_group_g<2>(prm, sms, stream);
        case 4: return launch_group_g<4>(prm, sms, stream);
        case 8: return launch_group_g<8>(prm, sms, stream);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace pa
