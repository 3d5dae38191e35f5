// Attention tiles on 5th-generation tensor cores (tcgen05.mma, accumulators and
// probabilities in tensor memory, operands staged by TMA): the chunked prefill,
// and the shared-prefix group units of the split decode.
//
// What is computed (include/pa.h): sequence s has C_s query rows, the last C_s
// positions of its L_s-token context; row i sits at position p = L_s - C_s + i
// and attends to keys 0..p (causal), K/V read through the block table.
// Sources: "vLLM 深度拆解" (chenxutan) 2.3 (prefill processes a whole prompt and is
// compute bound) and 4.3/5.1 (long prompts are cut into chunks interleaved with
// decode); devpress vLLM v0.6.x teardown, 核心代码拆解 (paged K/V via the table).
//
// Rows: the g query heads of one kv head are packed into the rows of a tile
// (row = chunk row * g + head), so every K/V byte staged in shared memory serves
// all g of them.  A persistent CTA runs two row streams over 128-key tiles:
//   S_t = Q_t K^T   tcgen05.mma kind::f16, M = 128, N = 128, K = 16 x 8 -> tensor memory
//   P_t = softmax   online, fp32, one row per thread (tcgen05.ld), written back as
//                   bf16 over the first 64 columns of S_t (tcgen05.st)
//   O_t += P_t V    tcgen05.mma with A = P_t read from tensor memory, B = V (MN-major)
// A job is either two 128-row query tiles sharing every K/V tile (stream t owns
// tile t), or one query tile whose key tiles alternate between the streams (each
// keeps its own running max, sum and O; the two are merged at the end).  Either
// way one stream's softmax runs while the tensor core computes the other's
// products.  The MMA issue order per key tile is PV_t(previous tile of t), then
// QK_t(this tile): S_t being full therefore also means O_t is not being written.
// Tensor memory (512 columns): S0 | S1 | O0 | O1.  The reference point of P and O
// (a running row maximum) moves only when a row's maximum rises by more than 2^8,
// so O is rescaled rarely; the merge and the final division use the same point.
// Warp roles: 0-3 softmax of stream 0, 4-7 softmax of stream 1 (warp w reads
// tensor-memory lanes 32 (w % 4) .. + 31), 8 issues the MMAs from one thread and
// owns the tensor memory, 9 loads Q and K tiles, 10 loads V tiles (11 only
// completes the third warpgroup): TMA with the 128-byte swizzle (the canonical
// layouts the MMA descriptors name) into separate two-stage K and V rings of
// 32 KB stages, one TMA box per (16-token block, 64-column half).  With rings and
// warps of their own, K loads run ahead of the V stages that PVs still hold.
// Every wait is bounded; an abort drains the copies and MMAs in flight
// and still frees the tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cstring>
#include <mutex>

#include "pa_common.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kD = 128;              // head_dim (bf16 only)
constexpr int kTileM = 128;          // query rows per stream tile
constexpr int kTileN = 128;          // keys per K/V tile
constexpr int kKStages = 2;          // K tile ring
constexpr int kVStages = 2;          // V tile ring
constexpr int kThreads = 12 * 32;    // 8 softmax warps, 1 MMA warp, 2 load warps, 1 idle
constexpr int kMmaWarp = 8, kLoadWarp = 9, kVLoadWarp = 10;
// Registers per thread after the split (setmaxnreg, per warpgroup of 4 warps): the
// launch gives 384 threads x 168; the softmax warpgroups take 200 (a row of S in
// registers), the MMA / load warpgroup 96: 256 x 200 + 128 x 96 <= 384 x 168, and
// each SM sub-partition (warps w, w + 4, w + 8) holds 2 x 200 + 96 <= 512 per lane.
constexpr int kRegsSoftmax = 200, kRegsOther = 96;
static_assert(256 * kRegsSoftmax + 128 * kRegsOther <= kThreads * 168, "register split over the launch's total");
constexpr int kSoftmaxThreads = 256;
constexpr uint32_t kTmemCols = 512;  // S0, S1, O0, O1
constexpr float kRescaleLog2 = 8.f;  // the reference point moves when a row max rises by more (log2 units)

// shared memory (offsets from a 1024-byte aligned base inside the dynamic area)
constexpr uint32_t kHalf = kTileM * 128;            // one 64-column half of a 128-row tile
constexpr uint32_t kTileBytes = 2 * kHalf;          // 32 KB
constexpr uint32_t kBlockBytes = kBlockSize * 128;  // one block's rows in one half
constexpr uint32_t kOffQ = 0;                       // Q buffers 0 and 1
constexpr uint32_t kOffRing = 2 * kTileBytes;
constexpr uint32_t kOffVRing = kOffRing + kKStages * kTileBytes;
constexpr uint32_t kOffBar = kOffVRing + kVStages * kTileBytes;
// barriers
constexpr int kBarKFull = 0;                      // [kKStages] K stage landed (TMA bytes)
constexpr int kBarKEmpty = kBarKFull + kKStages;  // [kKStages] its QKs done (MMA commit)
constexpr int kBarVFull = kBarKEmpty + kKStages;  // [kVStages] V stage landed: TMA bytes + the V loader's 2nd arrival
constexpr int kBarVEmpty = kBarVFull + kVStages;  // [kVStages] its PVs done (MMA commit)
constexpr int kBarQFull = kBarVEmpty + kVStages;  // [2] Q buffer landed
constexpr int kBarQEmpty = kBarQFull + 2;       // [2] last QK reading a Q buffer done
constexpr int kBarSFull = kBarQEmpty + 2;       // [2] S_t written
constexpr int kBarPFull = kBarSFull + 2;        // [2] P_t written (the 128 softmax threads of stream t)
constexpr int kBarOFull = kBarPFull + 2;        // [2] last PV_t of a job done
constexpr int kBarOFree = kBarOFull + 2;        // the job's O read by every softmax thread
constexpr int kBarMl = kBarOFree + 1;           // both streams' (m, l) rows published
constexpr int kBarIdle = kBarMl + 1;            // every MMA issued has completed
constexpr int kNumBars = kBarIdle + 1;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;  // tmem slot, abort flag
constexpr uint32_t kOffMl = kOffMisc + 16;             // float2 (m, l) [2 streams][128 rows]
constexpr uint32_t kOffJobs = kOffMl + 2 * 128 * 8;  // job records [8] (int4) and tags [8] (group units)
constexpr uint32_t kOffGroups = (kOffJobs + 8 * 16 + 8 * 4 + 15) / 16 * 16;  // int4 group records
constexpr int kMaxGroups = 1024;                      // >= 4 members each, <= 4096 sequences
constexpr size_t kSmemUsed = kOffGroups + kMaxGroups * 16;
static_assert(kOffQ % 1024 == 0 && kOffRing % 1024 == 0 && kOffVRing % 1024 == 0 && kTileBytes % 1024 == 0,
              "swizzled tiles: 1024-byte aligned");
static_assert(kOffBar % 8 == 0 && kOffMisc % 4 == 0 && kOffMl % 8 == 0 && kOffJobs % 4 == 0 && kOffGroups % 16 == 0,
              "shared-memory fields aligned to their types");
constexpr size_t kSmemBytes = kSmemUsed + 1024;       // slack to align the base

struct Params {
    CUtensorMap qmap;  // query rows: {head_dim, Hq, rows of Hq heads}, box {64, G, 128 / G}
    CUtensorMap kmap;  // pool: {head_dim, 16 tokens, blocks x kv heads}, box {64, 16, 1}
    CUtensorMap vmap;
    const unsigned char *vc;  // value pool (rows of a partly filled last block are copied by hand)
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
    int32_t pairs;     // prefill: 256-row jobs per (sequence, kv head)
    float scale_log2;
    // shared-prefix group units of the split decode
    const int4 *groups;    // (first seq, members, shared tokens, units before)
    const int32_t *meta;   // [0] groups, [1] units, [3] work counter, [4] CTAs that take units
    float *ws_acc;
    float2 *ws_ml;
    int32_t max_parts;
    unsigned long long wait_ns;  // bound of every in-kernel wait
    uint32_t ticket;   // prefill with dynamic jobs: this call's tag on its work counter (nonzero)
};

// ---- tcgen05 and TMA wrappers -------------------------------------------------
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

// D (tensor memory) (+)= A (shared-memory descriptor) * B (shared-memory descriptor)
__device__ __forceinline__ void tc_mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}
// D (tensor memory) (+)= A (tensor memory: rows = lanes, K packed two bf16 per
// column) * B (shared-memory descriptor)
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// 32 lanes x 32 columns of 32 bits: thread i gets columns c..c+31 of lane base + i
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
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
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 3-D tiled TMA load of one box into shared memory; completion as transaction
// bytes on `bar`.  x (the innermost coordinate) is 0 or 64 here: 16-byte aligned.
// A box reaching outside the tensor (z = -1 included) reads zeros there.
__device__ __forceinline__ void tma_load_3d(uint32_t dst_smem, const CUtensorMap *map, int x, int y, int z,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst_smem),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Shared-memory matrix descriptor: 128-byte swizzle, start/LBO/SBO in 16-byte
// units, descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator, M = 128,
// N = 128, A K-major; B K-major (QK) or MN-major (PV).
constexpr uint32_t idesc_bf16(bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(kTileN >> 3) << 17) |
           ((uint32_t)(kTileM >> 4) << 24);
}

// max of three (the sm_100 three-input max)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort, const Params &p) {
    return mbar_wait_bounded(bar, parity, abort, p.err, p.wait_ns);
}

// One job of a CTA.  Packed row r (0..127) of query tile t holds query head
// h*G + r%G of row group qz[t] + r/G.  two: both tiles hold rows and share every
// key tile; otherwise one tile (t = 0) whose key tile j goes to stream j & 1.
// Row r of tile t may see keys 0..lim0[t] + lim_step * (r / G) (all < nkeys).
struct Job {
    bool two;
    int nrows[2];
    int qz[2];         // TMA z coordinate of the tile's first row group
    int lim0[2];
    int lim_step;
    int nkeys, ntiles;
    int h;             // kv head
    const int32_t *trow;
    // output: prefill -> bf16 rows of row group out_row0 + ..; group -> fp32
    // partials of workspace row (first + r/G)*Hq + h*G + r%G, slot part
    int64_t out_row0;
    int first, part;
};

// Group unit u's record (first seq, members, shared tokens, kv head), from
// the group list copied to shared memory.
__device__ __forceinline__ int4 group_record(int u, const int4 *sgroups, int ngroups) {
    int lo = 0, hi = ngroups;  // groups[lo].w <= u < groups[hi].w
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (sgroups[mid].w <= u) lo = mid; else hi = mid;
    }
    const int4 gr = sgroups[lo];  // (first seq, members, shared tokens, units before)
    return make_int4(gr.x, gr.y, gr.z, u - gr.w);
}

// The job: a group unit from its record (u unused), a prefill job from its index u
// (rec unused).  False: a prefill job with no rows, or an invalid chunk.
template <int G, bool kGroup>
__device__ __forceinline__ bool make_job(const Params &p, int u, int4 rec, Job &jb) {
    if constexpr (kGroup) {
        const int4 gr = rec;
        jb.h = gr.w;                   // one unit per kv head
        jb.part = 0;                   // workspace slot 0 holds the shared tokens' partial
        jb.first = gr.x;
        jb.two = false;
        jb.nrows[0] = gr.y * G;
        jb.nrows[1] = 0;
        jb.qz[0] = jb.qz[1] = gr.x;
        jb.trow = p.tables + (int64_t)gr.x * p.max_blocks;
        jb.nkeys = gr.z;               // the group's shared tokens (whole blocks)
        jb.lim0[0] = jb.lim0[1] = jb.nkeys - 1;
        jb.lim_step = 0;
        jb.ntiles = (jb.nkeys + kTileN - 1) / kTileN;
        jb.out_row0 = 0;
        return true;
    } else {
        const int jp = u % p.pairs;
        const int rem = u / p.pairs;
        const int h = rem % p.num_kv_heads, s = rem / p.num_kv_heads;
        const int L = __ldg(p.lens + s), C = __ldg(p.chunks + s);
        if (C < 0 || C > p.max_chunk || C > L || (int64_t)L > (int64_t)p.max_blocks * kBlockSize) return false;
        const int rows = C * G, r0 = jp * 2 * kTileM;
        if (r0 >= rows) return false;
        const int start = L - C;
        jb.h = h;
        jb.nrows[0] = min(kTileM, rows - r0);
        jb.nrows[1] = min(kTileM, max(0, rows - r0 - kTileM));
        jb.two = jb.nrows[1] > 0;
        const int i0 = r0 / G;  // chunk row of the job's first packed row
        jb.qz[0] = s * p.max_chunk + i0;
        jb.qz[1] = jb.qz[0] + kTileM / G;
        jb.lim0[0] = start + i0;
        jb.lim0[1] = jb.two ? start + i0 + kTileM / G : jb.lim0[0];
        jb.lim_step = 1;
        const int last_row = (r0 + jb.nrows[0] + jb.nrows[1] - 1) / G;
        jb.nkeys = start + last_row + 1;  // keys 0..start + last_row
        jb.ntiles = (jb.nkeys + kTileN - 1) / kTileN;
        jb.trow = p.tables + (int64_t)s * p.max_blocks;
        jb.out_row0 = (int64_t)s * p.max_chunk + i0;
        jb.first = jb.part = 0;
        return true;
    }
}

// Prefill jobs with few per CTA are handed out dynamically (measured on B200: a
// 32K-token chunk of 3.5 jobs per CTA 9% faster; with 14 short jobs per CTA the
// static round robin evens out by itself and the hand-off costs 3.5%): a CTA's
// first job is blockIdx.x, the next ones gridDim.x + values drawn from a work
// counter, so that the CTAs that finish early take the last jobs.  The counters are a static pool; a call
// uses slot ticket % kCtrSlots, whose 64-bit word holds (ticket << 32 | jobs drawn).
// A draw is one atomic add; the one that finds an earlier call's tag there
// installs this call's tag with a count of 1 (its job 0), so no counter needs
// zeroing between calls.  A later call's tag means kCtrSlots later calls have
// started while this one still runs (never on one stream): the CTA then stops
// taking jobs and flags a timeout.
constexpr int kCtrSlots = 1024;
constexpr int kDynJobsPerCta = 8;  // dynamic when njobs <= this x the grid
__device__ unsigned long long g_job_ctr[kCtrSlots];

__device__ __forceinline__ unsigned long long *job_ctr(const Params &p) { return &g_job_ctr[p.ticket % kCtrSlots]; }
__device__ __forceinline__ unsigned long long draw_add(const Params &p) { return atomicAdd(job_ctr(p), 1ull); }

// The job index (from 0) of a draw whose add returned `old`, or -1 (see above).
__device__ __forceinline__ int64_t job_claim(const Params &p, unsigned long long old) {
    unsigned long long *w = job_ctr(p);
    unsigned long long guess = old + 1;  // the word after this draw's add
    for (int i = 0; i < 4096; ++i) {
        const uint32_t tag = (uint32_t)(old >> 32);
        if (tag == p.ticket) return (int64_t)(uint32_t)old;
        if ((int32_t)(tag - p.ticket) > 0) return -1;
        // an earlier call's word: install this call's tag, counting this draw as job 0
        const unsigned long long o = atomicCAS(w, guess, ((unsigned long long)p.ticket << 32) | 1ull);
        if (o == guess) return 0;
        if ((uint32_t)(o >> 32) == (uint32_t)(guess >> 32)) {
            guess = o;  // still the earlier call's word (other stale adds): retry on it
        } else {
            old = draw_add(p);  // another draw installed a tag first: draw again
            guess = old + 1;
        }
    }
    return -1;
}

// An invalid prefill chunk is flagged once, by its sequence's first job.
__device__ __forceinline__ void flag_bad_chunk(const Params &p, int u) {
    if (u % p.pairs != 0 || (u / p.pairs) % p.num_kv_heads != 0) return;
    const int s = u / p.pairs / p.num_kv_heads;
    const int L = __ldg(p.lens + s), C = __ldg(p.chunks + s);
    if (C < 0 || C > p.max_chunk || C > L || (int64_t)L > (int64_t)p.max_blocks * kBlockSize)
        flag_error(p.err, PA_DEVERR_CHUNK);
}

// Streams that consume key tile j of a job (bit t = stream t).
__device__ __forceinline__ unsigned consumers(const Job &jb, int j) { return jb.two ? 3u : (1u << (j & 1)); }
// Does stream t take part in the job (it has at least one key tile)?
__device__ __forceinline__ bool stream_used(const Job &jb, int t) { return jb.two || jb.ntiles > t; }
// Q buffer of stream t: a two-tile job uses both; a one-tile job alternates
// buffers with the job count, so the next job's Q loads during this one.
__device__ __forceinline__ int q_buffer(const Job &jb, int t, int njob) { return jb.two ? t : (njob & 1); }

template <int G, bool kGroup, bool kDyn>
__global__ void __launch_bounds__(kThreads, 1) attn_tile_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const uint32_t sbase = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
    float2 *mlx = reinterpret_cast<float2 *>(smem + kOffMl);  // [2][128]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    int4 *sgroups = reinterpret_cast<int4 *>(smem + kOffGroups);
    // Group units are handed out dynamically: unit 0 of a CTA is blockIdx.x, the
    // next ones gridDim.x + values drawn from a counter (zeroed by the detection
    // kernel).  The K loader (warp 9), the only warp that waits for the detection
    // kernel, draws them and publishes job k's record (first seq, members, shared
    // partitions, kv head; members 0 = no more jobs) in slot k & 7; the other
    // warps read it there.  So the set-up below (barriers, tensor memory,
    // register split) overlaps the detection kernel.  Dynamic prefill jobs go the
    // same way, their ids drawn from this call's counter (job_claim); the K loader
    // skips the jobs with nothing to do, so every job published has at least one
    // key tile.  Static prefill jobs are computed by every warp itself.
    volatile int *job_rec = reinterpret_cast<volatile int *>(smem + kOffJobs);  // [8][4]
    volatile int *job_tag = job_rec + 32;
    int njobs = 0;
    if constexpr (!kGroup) {
        njobs = p.num_seqs * p.num_kv_heads * p.pairs;
        if ((int)blockIdx.x >= njobs) return;
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < 8; ++i) job_tag[i] = -1;
        for (int i = 0; i < kKStages; ++i) {
            mbar_init(&bars[kBarKFull + i], 1);
            mbar_init(&bars[kBarKEmpty + i], 1);
        }
        for (int i = 0; i < kVStages; ++i) {
            mbar_init(&bars[kBarVFull + i], 2);
            mbar_init(&bars[kBarVEmpty + i], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars[kBarQFull + t], 1);
            mbar_init(&bars[kBarQEmpty + t], 1);
            mbar_init(&bars[kBarSFull + t], 1);
            mbar_init(&bars[kBarPFull + t], kSoftmaxThreads / 2);
            mbar_init(&bars[kBarOFull + t], 1);
        }
        mbar_init(&bars[kBarOFree], kSoftmaxThreads);
        mbar_init(&bars[kBarMl], kSoftmaxThreads);
        mbar_init(&bars[kBarIdle], 1);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == kLoadWarp && lane == 0) {
        prefetch_tensormap(&p.qmap);
        prefetch_tensormap(&p.kmap);
        prefetch_tensormap(&p.vmap);
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // This CTA's job k as seen by the calling thread: 1 = jb filled, 0 = a prefill
    // job with nothing to do, -1 = no more jobs (or the wait gave up).
    // (a prefill record is (job id, 1, 0, 0); members 0 ends the work there too)
    auto job_from = [&](int4 rec, Job &jb) {
        if constexpr (kGroup) make_job<G, true>(p, 0, rec, jb);
        else make_job<G, false>(p, rec.x, rec, jb);
    };
    auto job_of_thread = [&](int k, Job &jb) -> int {
        if constexpr (!kGroup && !kDyn) {
            const int u = (int)blockIdx.x + k * (int)gridDim.x;
            if (u >= njobs) return -1;
            return make_job<G, false>(p, u, make_int4(0, 0, 0, 0), jb) ? 1 : 0;
        } else {
            const unsigned long long t0 = global_ns();
            while (job_tag[k & 7] != k) {
                if (*abort_flag || global_ns() - t0 > p.wait_ns) {
                    if (!*abort_flag) flag_error(p.err, PA_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                    return -1;
                }
            }
            __threadfence_block();
            const int4 rec = make_int4(job_rec[(k & 7) * 4], job_rec[(k & 7) * 4 + 1], job_rec[(k & 7) * 4 + 2],
                                       job_rec[(k & 7) * 4 + 3]);
            if (rec.y <= 0) return -1;
            job_from(rec, jb);
            return 1;
        }
    };
    // the same for a whole warp: lane 0 reads the record, the others take it
    auto job_of_warp = [&](int k, Job &jb) -> int {
        if constexpr (!kGroup && !kDyn) {
            return job_of_thread(k, jb);
        } else {
            int4 rec = make_int4(0, -1, 0, 0);
            if (lane == 0) {
                const unsigned long long t0 = global_ns();
                bool okw = true;
                while (job_tag[k & 7] != k) {
                    if (*abort_flag || global_ns() - t0 > p.wait_ns) {
                        if (!*abort_flag) flag_error(p.err, PA_DEVERR_TIMEOUT);
                        *abort_flag = 1;
                        okw = false;
                        break;
                    }
                }
                __threadfence_block();
                if (okw)
                    rec = make_int4(job_rec[(k & 7) * 4], job_rec[(k & 7) * 4 + 1], job_rec[(k & 7) * 4 + 2],
                                    job_rec[(k & 7) * 4 + 3]);
            }
            rec.x = __shfl_sync(kFull, rec.x, 0);
            rec.y = __shfl_sync(kFull, rec.y, 0);
            rec.z = __shfl_sync(kFull, rec.z, 0);
            rec.w = __shfl_sync(kFull, rec.w, 0);
            if (rec.y <= 0) return -1;
            job_from(rec, jb);
            return 1;
        }
    };
    // the K loader's lane 0 publishes job k's record in slot k & 7
    auto publish = [&](int k, int4 rec) {
        if (lane == 0) {
            job_rec[(k & 7) * 4] = rec.x;
            job_rec[(k & 7) * 4 + 1] = rec.y;
            job_rec[(k & 7) * 4 + 2] = rec.z;
            job_rec[(k & 7) * 4 + 3] = rec.w;
            __threadfence_block();
            job_tag[k & 7] = k;
        }
    };

    // each warpgroup sets its register count at one instruction that dominates
    // all of its code
    if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
    if (warp == kLoadWarp || warp == kVLoadWarp) {
        // ------------------------------------------------------------ loaders
        // Warp 9 loads Q and the K tiles and hands out the group units' ids; warp
        // 10 loads the V tiles.  Lane 0 issues Q and arms the barriers; lanes 0..15
        // each issue one of a key tile's 16 TMA boxes (block lane / 2, 64-column
        // half lane % 2): a TMA instruction holds its issuing thread for a while,
        // so the boxes of a tile go out from 16 threads at once.  A V stage completes on the TMA bytes plus a second arrival of
        // lane 0, made once the warp has filled by hand the block that holds the
        // last keys of a job when they end inside it (its rows past the keys become
        // zeros: 0 * (NaN or Inf) would poison the sums).
        const bool is_v = warp == kVLoadWarp;
        const int nst = is_v ? kVStages : kKStages;
        uint64_t *full = &bars[is_v ? kBarVFull : kBarKFull];
        uint64_t *empty = &bars[is_v ? kBarVEmpty : kBarKEmpty];
        const uint32_t ring = sbase + (is_v ? kOffVRing : kOffRing);
        const CUtensorMap *map = is_v ? &p.vmap : &p.kmap;
        int it = 0;                 // tiles issued into this warp's ring (jobs in order)
        int qn[2] = {0, 0};         // loads issued per Q buffer (warp 9)
        bool ok = true;
        int njob = 0;
        int ngroups = 0, active = (int)gridDim.x;
        if constexpr (kGroup) {
            if (!is_v) {
                // launched behind the detection kernel: its group list must be
                // complete; then the per-sequence decode may start (it reads only
                // detection output)
                grid_dep_wait();
                grid_dep_launch();
                njobs = __ldg(p.meta + 1);
                ngroups = min(__ldg(p.meta), kMaxGroups);
                active = min((int)gridDim.x, __ldg(p.meta + 4));
                for (int i = lane; i < ngroups; i += 32) sgroups[i] = __ldg(&p.groups[i]);
                __syncwarp();
            }
        }
        int u = blockIdx.x;
        // prefill (K loader, lane 0): the add of the next job's draw, issued three
        // tiles before the end of the current job so its latency is hidden
        unsigned long long pend = 0;
        bool pend_ok = false;
        for (int k = 0; ok; ++k) {
            int u_next = 0;
            Job jb;
            if constexpr (kGroup) {
                if (!is_v) {
                    // publish job k (members 0: no more jobs); CTAs past the number
                    // the detection kernel chose take none and leave their SM
                    if (k == 0 && (int)blockIdx.x >= active) u = njobs;
                    const int4 rec = u < njobs ? group_record(u, sgroups, ngroups) : make_int4(0, 0, 0, 0);
                    publish(k, rec);
                    if (u >= njobs) break;
                    // the next job's id (drawn now, read at the end of this one)
                    if (lane == 0) u_next = active + atomicAdd(const_cast<int32_t *>(p.meta) + 3, 1);
                    make_job<G, true>(p, 0, rec, jb);
                } else if (job_of_warp(k, jb) < 0) {
                    break;
                }
            } else if (kDyn && !is_v) {
                // dynamic prefill: job k is the next drawn job with work; an empty job
                // (chunk shorter than its pair's rows) or an invalid chunk is skipped.
                // A draw made during the previous job (pend) is used first.
                auto next_job = [&]() -> int {
                    int v = njobs;
                    if (lane == 0) {
                        const unsigned long long old = pend_ok ? pend : draw_add(p);
                        pend_ok = false;
                        const int64_t id = job_claim(p, old);
                        if (id < 0) flag_error(p.err, PA_DEVERR_TIMEOUT);
                        else v = (int)min((int64_t)njobs, (int64_t)gridDim.x + id);
                    }
                    return __shfl_sync(kFull, v, 0);
                };
                int uj = k == 0 ? (int)blockIdx.x : next_job();
                while (uj < njobs && !make_job<G, false>(p, uj, make_int4(0, 0, 0, 0), jb)) {
                    if (lane == 0) flag_bad_chunk(p, uj);
                    uj = next_job();
                }
                publish(k, uj < njobs ? make_int4(uj, 1, 0, 0) : make_int4(0, 0, 0, 0));
                if (uj >= njobs) break;
            } else {
                // static prefill (every warp computes job k), or the V loader of a
                // dynamic one (reads the K loader's record: never an empty job)
                const int have = job_of_warp(k, jb);
                if (have < 0) break;
                if (have == 0) {
                    if (lane == 0 && !is_v) flag_bad_chunk(p, (int)blockIdx.x + k * (int)gridDim.x);
                    continue;
                }
            }
            // Q tiles: a buffer is rewritten once the QKs of its previous use are done
            const int nq = jb.two ? 2 : 1;
            for (int t = 0; !is_v && ok && t < nq; ++t) {
                const int b = q_buffer(jb, t, njob);
                if (lane == 0) {
                    ok = qn[b] == 0 || wait_bar(&bars[kBarQEmpty + b], (qn[b] - 1) & 1, abort_flag, p);
                    if (ok) {
                        mbar_arrive_expect_tx(&bars[kBarQFull + b], kTileBytes);
                        const uint32_t dst = sbase + kOffQ + b * kTileBytes;
                        tma_load_3d(dst, &p.qmap, 0, jb.h * G, jb.qz[t], &bars[kBarQFull + b]);
                        tma_load_3d(dst + kHalf, &p.qmap, 64, jb.h * G, jb.qz[t], &bars[kBarQFull + b]);
                    }
                }
                ok = __shfl_sync(kFull, ok, 0);
                if (ok) ++qn[b];
            }
            const int nblk = (jb.nkeys + kBlockSize - 1) / kBlockSize;
            const int tail = jb.nkeys % kBlockSize;  // tokens in a partly filled last block (0: none)
            // table entries 32 at a time (four key tiles), one group ahead: lane i
            // holds block 32 q + i of group q (-1: past the keys or invalid; flagged
            // by the K loader)
            auto entries = [&](int q) -> int {
                const int b = q * 32 + lane;
                if (b >= nblk) return -1;
                const int e = __ldg(jb.trow + b);
                if (e < 0 || e >= p.num_blocks) {
                    if (!is_v) flag_error(p.err, PA_DEVERR_BLOCK_ID);
                    return -1;
                }
                return e;
            };
            int ent = entries(0);
            int ent_next = jb.ntiles > 4 ? entries(1) : -1;
            for (int j = 0; ok && j < jb.ntiles; ++j) {
                if (j > 0 && (j & 3) == 0) {
                    ent = ent_next;
                    ent_next = j + 4 < jb.ntiles ? entries((j >> 2) + 1) : -1;
                }
                // the block of tile j whose box this lane issues (lanes 0..15)
                const int cur_e = __shfl_sync(kFull, ent, ((j & 3) << 3) | ((lane >> 1) & 7));
                // invalid or past the keys: a coordinate outside the map reads zeros
                const int z = cur_e >= 0 ? cur_e * p.num_kv_heads + jb.h : -1;
                // block of this V tile filled by hand, or -1
                const int hand = (is_v && tail != 0 && (jb.nkeys - 1) / kTileN == j)
                                     ? (jb.nkeys - 1) / kBlockSize - j * 8 : -1;
                const int st = it % nst;
                if constexpr (kDyn) {
                    if (!is_v && lane == 0 && !pend_ok && j == max(0, jb.ntiles - 3)) {
                        pend = draw_add(p);
                        pend_ok = true;
                    }
                }
                if (lane == 0) {
                    ok = it < nst || wait_bar(&empty[st], ((it / nst) - 1) & 1, abort_flag, p);
                    if (ok) mbar_arrive_expect_tx(&full[st], hand >= 0 ? kTileBytes - 2 * kBlockBytes : kTileBytes);
                }
                ok = __shfl_sync(kFull, ok, 0);
                if (!ok) break;
                if (lane < 16 && (lane >> 1) != hand) {
                    const int hf = lane & 1;
                    tma_load_3d(ring + st * kTileBytes + hf * kHalf + (lane >> 1) * kBlockBytes, map, hf * 64, 0, z,
                                &full[st]);
                }
                if (hand >= 0) {
                    const int e = __shfl_sync(kFull, cur_e, 2 * hand);
                    unsigned char *base = smem + (is_v ? kOffVRing : kOffRing) + st * kTileBytes;
                    const unsigned char *src =
                        e >= 0 ? p.vc + ((int64_t)e * p.num_kv_heads + jb.h) * kBlockSize * (kD * 2) : nullptr;
                    // 16 rows x 16 chunks of 16 bytes, stored as TMA would (128-byte swizzle)
                    for (int idx = lane; idx < kBlockSize * 16; idx += 32) {
                        const int rr = idx >> 4, c = idx & 15;
                        uint4 v = make_uint4(0, 0, 0, 0);
                        if (src && rr < tail) v = *reinterpret_cast<const uint4 *>(src + rr * (kD * 2) + c * 16);
                        const int row = hand * kBlockSize + rr;  // row inside the 128-row tile
                        *reinterpret_cast<uint4 *>(base + (c >> 3) * kHalf + row * 128 + (((c & 7) ^ (row & 7)) << 4)) = v;
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                if (is_v && lane == 0) mbar_arrive(&full[st]);
                ++it;
            }
            ++njob;
            if constexpr (kGroup) u = __shfl_sync(kFull, u_next, 0);
        }
        // nothing may land after the CTA exits: wait for every stage still in flight
        if (lane == 0) {
            for (int k = std::max(0, it - nst); k < it; ++k) mbar_wait_drain(&full[k % nst], (k / nst) & 1);
            for (int b = 0; b < 2; ++b)
                if (qn[b] > 0) mbar_wait_drain(&bars[kBarQFull + b], (qn[b] - 1) & 1);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdQK = idesc_bf16(false), kIdPV = idesc_bf16(true);
            int itk = 0, itv = 0;        // K and V tiles consumed
            int qn[2] = {0, 0};          // uses per Q buffer
            int npf[2] = {0, 0};         // P_t tiles consumed
            int njob = 0;
            bool ok = true;
            for (int k = 0; ok; ++k) {
                Job jb;
                const int have = job_of_thread(k, jb);  // this MMA thread runs alone
                if (have < 0) break;
                if (have == 0) continue;
                const int nq = jb.two ? 2 : 1;
                int qb[2];
                for (int t = 0; t < 2; ++t) qb[t] = q_buffer(jb, t, njob);
                for (int t = 0; ok && t < nq; ++t) {
                    ok = wait_bar(&bars[kBarQFull + qb[t]], qn[qb[t]] & 1, abort_flag, p);
                    ++qn[qb[t]];
                }
                if (!ok) break;
                int pend[2] = {-1, -1};     // key tile whose PV is still to be issued, per stream
                bool first_pv[2] = {true, true};
                bool o_ready = njob == 0;   // the previous job's O has been read
                const int itk0 = itk, itv0 = itv;
                // PV_t of key tile jp
                auto issue_pv = [&](int t, int jp) -> bool {
                    if (!o_ready) {
                        if (!wait_bar(&bars[kBarOFree], (njob - 1) & 1, abort_flag, p)) return false;
                        o_ready = true;
                    }
                    if (!wait_bar(&bars[kBarPFull + t], npf[t] & 1, abort_flag, p)) return false;
                    ++npf[t];
                    const int iv = itv0 + jp, st = iv % kVStages;
                    if (!wait_bar(&bars[kBarVFull + st], (iv / kVStages) & 1, abort_flag, p)) return false;
                    tc_fence_after();
                    const uint32_t va = sbase + kOffVRing + st * kTileBytes;
                    const uint32_t tP = tmem + t * 128, tO = tmem + 256 + t * 128;
#pragma unroll
                    for (int kk = 0; kk < kTileN / 16; ++kk)
                        tc_mma_ts(tO, tP + kk * 8, smem_desc(va + kk * 2048, kHalf, 1024), kIdPV,
                                  !first_pv[t] || kk > 0);
                    first_pv[t] = false;
                    // V(jp) is free once its last consumer's PV is done
                    if (!jb.two || t == 1) tc_commit(&bars[kBarVEmpty + st]);
                    return true;
                };
                for (int j = 0; ok && j < jb.ntiles; ++j) {
                    const int ik = itk0 + j, sk = ik % kKStages;
                    const unsigned cons = consumers(jb, j);
                    bool k_ready = false;
                    for (int t = 0; t < 2; ++t) {
                        if (!(cons >> t & 1u)) continue;
                        if (pend[t] >= 0 && !issue_pv(t, pend[t])) {
                            ok = false;
                            break;
                        }
                        if (!k_ready) {
                            if (!wait_bar(&bars[kBarKFull + sk], (ik / kKStages) & 1, abort_flag, p)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            k_ready = true;
                        }
                        const uint32_t qa = sbase + kOffQ + qb[t] * kTileBytes;
                        const uint32_t ka = sbase + kOffRing + sk * kTileBytes;
                        const uint32_t tS = tmem + t * 128;
#pragma unroll
                        for (int kk = 0; kk < kD / 16; ++kk) {
                            const uint32_t koff = (kk & 3) * 32 + (kk >> 2) * kHalf;
                            tc_mma_ss(tS, smem_desc(qa + koff, 16, 1024), smem_desc(ka + koff, 16, 1024), kIdQK,
                                      kk > 0);
                        }
                        tc_commit(&bars[kBarSFull + t]);
                        pend[t] = j;
                    }
                    if (!ok) break;
                    tc_commit(&bars[kBarKEmpty + sk]);  // K(j) is free once its QKs are done
                    if (j == jb.ntiles - 1) {          // the job's last QKs: its Q buffers are free
                        tc_commit(&bars[kBarQEmpty + qb[0]]);
                        if (jb.two) tc_commit(&bars[kBarQEmpty + qb[1]]);
                    }
                }
                for (int t = 0; ok && t < 2; ++t) {
                    if (pend[t] < 0) continue;
                    if (!issue_pv(t, pend[t])) {
                        ok = false;
                        break;
                    }
                    tc_commit(&bars[kBarOFull + t]);
                }
                itk = itk0 + jb.ntiles;
                itv = itv0 + jb.ntiles;
                ++njob;
            }
            // everything issued has completed once this arrives
            tc_commit(&bars[kBarIdle]);
            if (!mbar_wait_drain(&bars[kBarIdle], 0)) {
                *abort_flag = 1;
                flag_error(p.err, PA_DEVERR_TIMEOUT);
            }
        }
        __syncwarp();
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        // ------------------------------------------------------------ softmax
        // Stream t = warp / 4; one row per thread (tensor-memory lane 32 (warp % 4) + lane).
        const int t = warp >> 2, qd = warp & 3;
        const int r = qd * 32 + lane;
        const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
        const uint32_t tS = tmem + lane_off + t * 128;
        const float sl2 = p.scale_log2;
        int ns = 0;             // S_t fills seen
        int no[2] = {0, 0};     // O_t completions, both streams
        int njob = 0;
        bool live = true;
        for (int k = 0; live; ++k) {
            Job jb;
            const int have = job_of_warp(k, jb);
            if (have < 0) break;
            if (have == 0) continue;
            const int tile = jb.two ? t : 0;  // query tile whose rows this thread's lane holds
            const bool row_ok = r < jb.nrows[tile];
            const bool warp_rows = __any_sync(kFull, row_ok);
            // last key this row may see; a padding row (never written out) is left
            // unmasked, so that it does not force the masked path on its warp
            const int lim = row_ok ? jb.lim0[tile] + jb.lim_step * (r / G) : INT_MAX;
            float m = -INFINITY, l = 0.f;
            bool first = true;
            if (stream_used(jb, t)) {
                for (int j = 0; j < jb.ntiles; ++j) {
                    if (!(consumers(jb, j) >> t & 1u)) continue;
                    live = live && wait_bar(&bars[kBarSFull + t], ns & 1, abort_flag, p);
                    live = __all_sync(kFull, live);
                    if (!live) break;
                    ++ns;
                    tc_fence_after();
                    if (warp_rows) {
                        const int key0 = j * kTileN;
                        float sv[kTileN];
#pragma unroll
                        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sv + c * 32);
                        tmem_wait_ld();
                        // every key of the tile visible to every row of the warp: no per-key test
                        const bool open = __all_sync(kFull, lim >= key0 + kTileN - 1);
                        // row max of the scaled visible scores
                        float mx = -INFINITY;
                        if (sl2 >= 0.f) {
                            float a = -INFINITY;
                            if (open) {
#pragma unroll
                                for (int k = 0; k < kTileN; k += 2) a = fmax3(a, sv[k], sv[k + 1]);
                            } else {  // a causal edge or the keys' end
#pragma unroll
                                for (int k = 0; k < kTileN; ++k) a = key0 + k <= lim ? fmaxf(a, sv[k]) : a;
                            }
                            mx = a == -INFINITY ? -INFINITY : a * sl2;
                        } else {
                            float a = INFINITY;
#pragma unroll
                            for (int k = 0; k < kTileN; ++k) a = key0 + k <= lim ? fminf(a, sv[k]) : a;
                            mx = a == INFINITY ? -INFINITY : a * sl2;
                        }
                        if (mx != mx) mx = -INFINITY;
                        const float m_new = fmaxf(m, mx);
                        float alpha = 1.f;
                        bool resc = false;
                        if (first) {
                            m = m_new;
                        } else if (row_ok && m_new > m + kRescaleLog2) {
                            alpha = fast_exp2(m - m_new);  // m = -inf: O holds zeros, alpha 0
                            m = m_new;
                            resc = true;
                        }
                        if (__any_sync(kFull, resc)) {
                            // O_t is idle: its last PV completed before this S was written
                            const uint32_t tO = tmem + lane_off + 256 + t * 128;
#pragma unroll 1
                            for (int c = 0; c < 8; ++c) {
                                float ov[16];
                                tmem_ld16(tO + c * 16, ov);
                                tmem_wait_ld();
                                uint32_t w[16];
#pragma unroll
                                for (int k = 0; k < 16; ++k) w[k] = __float_as_uint(ov[k] * alpha);
                                tmem_st16(tO + c * 16, w);
                            }
                        }
                        l *= alpha;
                        const float m_use = m == -INFINITY ? 0.f : m;
                        // P = 2^(s * scale - m) as bf16 pairs over columns 0..63 of S_t
                        float2 acc = make_float2(0.f, 0.f);
                        const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-m_use, -m_use);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            uint32_t w[16];
#pragma unroll
                            for (int k = 0; k < 16; ++k) {
                                const int e = c * 32 + 2 * k;
                                float2 x = __ffma2_rn(make_float2(sv[e], sv[e + 1]), sc2, nm2);
                                x.x = fast_exp2(x.x);
                                x.y = fast_exp2(x.y);
                                if (!open) {
                                    if (key0 + e > lim) x.x = 0.f;
                                    if (key0 + e + 1 > lim) x.y = 0.f;
                                }
                                acc = __fadd2_rn(acc, x);
                                w[k] = pack_bf16x2(x.x, x.y);
                            }
                            tmem_st16(tS + c * 16, w);
                        }
                        l += acc.x + acc.y;
                        tmem_wait_st();
                    }
                    first = false;
                    tc_fence_before();
                    mbar_arrive(&bars[kBarPFull + t]);
                }
            }
            if (!live) break;
            // ---- epilogue: publish this stream's (m, l), then the output rows
            mlx[t * 128 + r] = make_float2(m, l);
            mbar_arrive(&bars[kBarMl]);
            live = wait_bar(&bars[kBarMl], njob & 1, abort_flag, p);
            live = __all_sync(kFull, live);
            const bool used1 = stream_used(jb, 1);
            if (live) {
                for (int s2 = 0; s2 < 2; ++s2) {
                    if (!stream_used(jb, s2) || (jb.two && s2 != t)) continue;
                    live = live && wait_bar(&bars[kBarOFull + s2], no[s2] & 1, abort_flag, p);
                }
                live = __all_sync(kFull, live);
            }
            ++no[0];
            if (used1) ++no[1];
            if (live && warp_rows) {
                tc_fence_after();
                // columns of this thread: a two-tile job -> all 128 of its own tile;
                // a one-tile job -> stream t takes columns 64t..64t+63 of the merge
                const int c0 = jb.two ? 0 : t * 64, ncol = jb.two ? 128 : 64;
                float f0 = 0.f, f1 = 0.f, M = -INFINITY, lt = 0.f;
                if (jb.two) {
                    M = m;
                    f0 = 1.f;
                    lt = l;
                } else {
                    const float2 a = mlx[r], b = used1 ? mlx[128 + r] : make_float2(-INFINITY, 0.f);
                    M = fmaxf(a.x, b.x);
                    if (M != -INFINITY) {
                        f0 = a.x == -INFINITY ? 0.f : fast_exp2(a.x - M);
                        f1 = b.x == -INFINITY ? 0.f : fast_exp2(b.x - M);
                    }
                    lt = a.y * f0 + b.y * f1;
                }
                const uint32_t tO0 = tmem + lane_off + 256 + (jb.two ? t * 128 : 0);
                const uint32_t tO1 = tmem + lane_off + 384;
                const bool any0 = __any_sync(kFull, f0 != 0.f);
                const bool any1 = __any_sync(kFull, f1 != 0.f);
                const float inv = kGroup ? 1.f : (lt > 0.f ? 1.f / lt : 0.f);
                for (int c = c0; c < c0 + ncol; c += 32) {
                    float o[32], o1[32];
#pragma unroll
                    for (int k = 0; k < 32; ++k) o[k] = o1[k] = 0.f;
                    if (any0) tmem_ld32(tO0 + c, o);
                    if (any1) tmem_ld32(tO1 + c, o1);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        float v = f0 != 0.f ? o[k] * f0 : 0.f;
                        if (f1 != 0.f) v = fmaf(o1[k], f1, v);
                        o[k] = v * inv;
                    }
                    if (!row_ok) continue;
                    if constexpr (kGroup) {
                        const int64_t wrow =
                            ((int64_t)(jb.first + r / G) * p.num_q_heads + jb.h * G + r % G) * p.max_parts + jb.part;
                        float *dst = p.ws_acc + wrow * kD + c;
#pragma unroll
                        for (int k = 0; k < 32; k += 4)
                            *reinterpret_cast<float4 *>(dst + k) = make_float4(o[k], o[k + 1], o[k + 2], o[k + 3]);
                        if (c == c0 && t == 0) p.ws_ml[wrow] = make_float2(M, lt);
                    } else {
                        const int64_t hs = (int64_t)kD * 2;
                        const int rr = (jb.two ? t * kTileM : 0) + r;  // packed row inside the job
                        unsigned char *dst = p.out + (jb.out_row0 + rr / G) * (int64_t)p.num_q_heads * hs +
                                             (int64_t)(jb.h * G + rr % G) * hs + c * 2;
#pragma unroll
                        for (int k = 0; k < 32; k += 8) {
                            const uint4 w = make_uint4(pack_bf16x2(o[k], o[k + 1]), pack_bf16x2(o[k + 2], o[k + 3]),
                                                       pack_bf16x2(o[k + 4], o[k + 5]), pack_bf16x2(o[k + 6], o[k + 7]));
                            *reinterpret_cast<uint4 *>(dst + k * 2) = w;
                        }
                    }
                }
            }
            // this job's O has been read (or was never needed): the MMA may overwrite it
            if (live) {
                tc_fence_before();
                mbar_arrive(&bars[kBarOFree]);
            }
            ++njob;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---- tensor maps (host) -------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// bf16 rows of 128 elements seen as {128, n1, n2} with byte strides {256,
// stride2}, box {64, b1, b2}, 128-byte swizzle; coordinates outside read zeros.
bool encode_map(CUtensorMap *m, const void *base, uint64_t n1, uint64_t n2, uint64_t stride2, uint32_t b1,
                uint32_t b2) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)n1, (cuuint64_t)(n2 > 0 ? n2 : 1)};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)stride2};
    const cuuint32_t box[3] = {64, b1, b2};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K/V pools [num_blocks, Hkv, 16, 128] as {128, 16, num_blocks * Hkv}, box {64, 16, 1}.
bool encode_cache_maps(Params &prm, const void *kc, const void *vc) {
    const uint64_t n2 = (uint64_t)prm.num_blocks * prm.num_kv_heads;
    prm.vc = static_cast<const unsigned char *>(vc);
    return encode_map(&prm.kmap, kc, kBlockSize, n2, (uint64_t)kBlockSize * kD * 2, kBlockSize, 1) &&
           encode_map(&prm.vmap, vc, kBlockSize, n2, (uint64_t)kBlockSize * kD * 2, kBlockSize, 1);
}

// Tag of a prefill call's work counter: nonzero, one per call in this process.
uint32_t next_ticket() {
    static std::atomic<uint32_t> ticket{0};
    uint32_t t = ticket.fetch_add(1, std::memory_order_relaxed) + 1;
    while (t == 0) t = ticket.fetch_add(1, std::memory_order_relaxed) + 1;
    return t;
}

template <int G, bool kGroup, bool kDyn = false>
cudaError_t launch_tiles(const Params &prm, int grid, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(attn_tile_kernel<G, kGroup, kDyn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    if constexpr (kGroup) {
        return launch_after(attn_tile_kernel<G, true, false>, dim3((unsigned)grid), dim3(kThreads), kSmemBytes,
                            stream, static_cast<const Params &>(prm));
    } else {
        attn_tile_kernel<G, false, kDyn><<<(unsigned)grid, kThreads, kSmemBytes, stream>>>(prm);
        return cudaGetLastError();
    }
}

template <int G>
cudaError_t launch_prefill_tiles(const Params &prm, int grid, bool dyn, cudaStream_t stream) {
    return dyn ? launch_tiles<G, false, true>(prm, grid, stream) : launch_tiles<G, false, false>(prm, grid, stream);
}

}  // namespace

cudaError_t launch_prefill(const PrefillLaunch &a, cudaStream_t stream) {
    static_assert(kSmemBytes <= 232448, "tile kernel shared memory over the sm_100 limit");
    if (a.cache.dtype != PA_BF16 || a.cache.head_dim != kD) return cudaErrorNotSupported;
    const int G = a.num_q_heads / a.cache.num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return cudaErrorNotSupported;
    Params prm;
    std::memset(&prm, 0, sizeof(prm));
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
    prm.pairs = (a.max_chunk * G + 2 * kTileM - 1) / (2 * kTileM);
    prm.scale_log2 = a.scale * kLog2e;
    prm.wait_ns = wait_limit_ns();
    prm.ticket = next_ticket();
    const int64_t njobs = (int64_t)a.num_seqs * a.cache.num_kv_heads * prm.pairs;
    if (njobs <= 0) return cudaSuccess;
    if (njobs > INT32_MAX) return cudaErrorNotSupported;
    const uint64_t qrows = (uint64_t)a.num_seqs * a.max_chunk;
    if (!encode_map(&prm.qmap, a.query, (uint64_t)a.num_q_heads, qrows, (uint64_t)a.num_q_heads * kD * 2, G,
                    kTileM / G) ||
        !encode_cache_maps(prm, a.key_cache, a.value_cache))
        return cudaErrorInvalidValue;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<int64_t>(njobs, num_sms(dev));
    const bool dyn = njobs <= (int64_t)kDynJobsPerCta * grid;
    switch (G) {
        case 1: return launch_prefill_tiles<1>(prm, grid, dyn, stream);
        case 2: return launch_prefill_tiles<2>(prm, grid, dyn, stream);
        case 4: return launch_prefill_tiles<4>(prm, grid, dyn, stream);
        default: return launch_prefill_tiles<8>(prm, grid, dyn, stream);
    }
}

cudaError_t launch_group_tiles(const GroupTileLaunch &a, int sms, cudaStream_t stream) {
    const int G = a.num_q_heads / a.num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return cudaErrorNotSupported;
    Params prm;
    std::memset(&prm, 0, sizeof(prm));
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
    prm.max_parts = a.max_partitions;
    prm.wait_ns = wait_limit_ns();
    if (!encode_map(&prm.qmap, a.query, (uint64_t)a.num_q_heads, (uint64_t)a.num_seqs,
                    (uint64_t)a.num_q_heads * kD * 2, G, kTileM / G) ||
        !encode_cache_maps(prm, a.key_cache, a.value_cache))
        return cudaErrorInvalidValue;
    switch (G) {
        case 1: return launch_tiles<1, true>(prm, sms, stream);
        case 2: return launch_tiles<2, true>(prm, sms, stream);
        case 4: return launch_tiles<4, true>(prm, sms, stream);
        default: return launch_tiles<8, true>(prm, sms, stream);
    }
}

}  // namespace pa
