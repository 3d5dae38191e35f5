// Decode attention over the paged KV cache (one query token per sequence) and
// the log-sum-exp reduce of its split-K variant.
//
// What is computed (see include/pa.h): for sequence s and query head h,
//   out = sum_{t < L_s} softmax_t(scale * <q, K_s[t]>) V_s[t],
// K_s[t] / V_s[t] read through the block table of s, kv head h / g.
// Sources: "vLLM 深度拆解" (chenxutan) 2.1/2.3 and the devpress vLLM v0.6.x
// teardown, section 核心代码拆解 (table lookup per logical block, scaled scores,
// softmax, V-weighted sum).
//
// Design (B200, HBM bound):
//  * Work unit = (sequence, kv head, partition of the context).  One CTA serves
//    all g = Hq/Hkv query heads of its kv head, so every K/V byte is read once
//    per unit.  The grid is persistent (one CTA per SM).  CTA c's first unit
//    is c; after it, CTA c takes c + gridDim, ... or, when a work counter is
//    given (the shared-prefix path), draws unit ids from it, so CTAs that start
//    early or get short units take more.  Units are ordered "further partitions
//    of long sequences, sequence-major, kv head innermost" then "first
//    partition of every sequence, kv head innermost": the further partitions
//    are all full length, and the first partitions (often shorter) even out
//    the CTAs' finish; sibling sequences' first partitions are read by CTAs
//    running at the same time, so blocks they share come from L2.
//  * Each of the CTA's 8 warps takes logical blocks w, w+8, ... of a unit and
//    streams them itself: the (block, kv head) slabs of K and V (4 KB each in
//    bf16) are fetched with 16-byte cp.async, all 32 lanes issuing, into a
//    per-warp ring of stages, the next block (across unit boundaries) always in
//    flight while the current one is computed.  Measured on B200: random 4 KB
//    slabs stream at ~6.6-7 TB/s this way, while bulk copies issued by a single
//    thread per SM cap near 0.9 TB/s (each copy costs the issuing thread
//    ~0.65 us), so there is no producer warp.  Each warp keeps its own
//    online-softmax state (running max m, running sum l, unnormalised
//    accumulator).  The 8 states of a unit are merged without a CTA barrier:
//    each warp leaves its state in one of two merge slots and arrives on an
//    mbarrier, streams the next unit, then merges its 1/8 share of the
//    previous one.
//  * bf16: QK and PV run on warp-level tensor-core tiles (mma.sync m16n8k16, bf16
//    operands, fp32 accumulation).  QK puts the block's 16 tokens in M and the g
//    heads in N (S^T = K Q^T); PV computes O^T = V^T P^T with head_dim in M, so no
//    tile rows are padding.  movmatrix turns S^T's fragments into P^T's operand
//    fragments in registers.  Slab rows are stored with an XOR swizzle of their
//    16-byte chunks so the ldmatrix reads are bank-conflict free.  A CUDA-core
//    version of this path (packed fp32 FMAs, shuffle reductions) measured issue
//    bound: 63 warp instructions per (token, kv head) against ~6 here.
//  * fp8 (e4m3 codes, head_dim 128): the slabs are 2 KB, half of bf16.  Each
//    thread reads whole 16-byte chunks of them and turns the codes into f16
//    (exact: e4m3 is a subset of f16) right before f16 tensor-core tiles; the
//    query goes to f16 once per unit.  k_scale is folded into the softmax scale,
//    v_scale into the merge.  Four stages per warp keep as many bytes in flight
//    as bf16's two.
//  * fp32: CUDA-core path (tensor cores would round fp32 inputs to tf32): 8 lanes
//    per token for QK with a transposing shuffle reduction, packed FFMA2 for QK
//    and PV.
//  * Split-K (partition_size > 0): a sequence with several partitions writes
//    (m, l, acc) per partition to the workspace and reduce_kernel combines them;
//    single-partition sequences are finished directly.
//  * Every wait that depends on another warp or kernel (the merge slots' mbarrier,
//    the ring of unit ids) is bounded by %globaltimer; on a timeout the CTA sets
//    PA_DEVERR_TIMEOUT, raises its abort flag and every warp leaves its loop.
#include <atomic>
#include <cfloat>
#include <chrono>
#include <climits>
#include <cstring>
#include <type_traits>

#include <cuda_fp8.h>

#include "cache_write.cuh"
#include "pa_common.cuh"
#include "pa_launch.h"

namespace pa {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

template <typename T>
struct ElemBytes;
template <>
struct ElemBytes<float> {
    static constexpr int value = 4;
};
template <>
struct ElemBytes<__nv_bfloat16> {
    static constexpr int value = 2;
};
// One e4m3 code of an FP8 pool (queries and outputs are bf16 then).
struct e4m3_t {
    unsigned char bits;
};
template <>
struct ElemBytes<e4m3_t> {
    static constexpr int value = 1;
};
template <typename T>
constexpr bool kIsFp8 = std::is_same<T, e4m3_t>::value;
// element type of queries and outputs
template <typename T>
using IoT = typename std::conditional<kIsFp8<T>, __nv_bfloat16, T>::type;

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

// Query rows of one unit of the group-rows mode (decode_kernel<T, D, kRowTile>):
// the members x g query heads of a small sibling group, two 8-column tensor-core
// tiles.
constexpr int kRowTile = 16;
// Longest private tail (blocks past the shared ones) a group-rows unit takes per
// member, so that its members need no per-sequence unit.
constexpr int kTailBlocks = 4;
constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Shared-memory carve-up (byte offsets from the dynamic shared memory base).
// Each warp owns kStagesPerWarp ring stages (K slab + V slab each): two, or one
// when a stage is too large (fp32, head_dim 128).  Two merge slots let the
// merge of a unit run while the next unit streams (mbarrier hand-over).  The
// group-rows mode (G == kRowTile: 16 rows per warp state) has room for one merge
// slot only and keeps no per-sequence prefix sums.
template <typename T, int D, int G>
struct Layout {
    static constexpr bool kRows = G == kRowTile;
    static constexpr int kElem = ElemBytes<T>::value;
    static constexpr int kRowBytes = D * kElem;                 // one token of one head
    static constexpr int kQRowBytes = D * (int)sizeof(IoT<T>);  // one query head
    static constexpr int kSlabBytes = kBlockSize * kRowBytes;   // one (block, kv head) slab
    static constexpr int kStageBytes = 2 * kSlabBytes;          // K slab + V slab
    static constexpr size_t kLimit = 232448;                    // sm_100 max dynamic smem per CTA
    static constexpr size_t kPBytes = sizeof(T) == 4 ? (size_t)kWarps * (16 * G + G) * 4 : 64;
    static constexpr size_t kMergeBytes = (size_t)kWarps * G * (D * 4 + 8);
    // prefix sums of the split path: the extra units per sequence, and on the
    // shared-prefix path (bf16, head_dim 128) also the first units
    static constexpr int kCumArrays = kRows ? 0 : (sizeof(T) == 2 && D == 128 ? 2 : 1);
    static constexpr size_t kFixed = kPBytes + 16 + 48 + 96 + (size_t)kCumArrays * (kMaxSplitSeqs + 1) * 4 + 64;
    static constexpr int stages_fit(int bufs) {
        return (int)((kLimit - kFixed - bufs * kMergeBytes) / ((size_t)kWarps * kStageBytes));
    }
    static constexpr int kWantStages = kIsFp8<T> ? 4 : 2;
    static constexpr int kStagesPerWarp =
        kRows ? kWantStages : (stages_fit(2) >= kWantStages ? kWantStages : (stages_fit(2) >= 2 ? 2 : 1));
    static constexpr int kMergeBufs = kRows ? 1 : (stages_fit(2) >= kStagesPerWarp ? 2 : 1);
    static constexpr size_t kPWarpFloats = 16 * G + G;          // fp32 path: p[16][G], alpha[G]
    static constexpr size_t kOffRing = 0;
    static constexpr size_t kOffP = kOffRing + (size_t)kWarps * kStagesPerWarp * kStageBytes;
    static constexpr size_t kOffMacc = align_up(kOffP + kPBytes, 16);
    static constexpr size_t kOffMml = kOffMacc + (size_t)kMergeBufs * kWarps * G * D * 4;
    static constexpr size_t kOffBar = align_up(kOffMml + (size_t)kMergeBufs * kWarps * G * 8, 16);
    static constexpr size_t kOffRingIds = kOffBar + 48;  // after 4 mbarriers + abort word
    static constexpr size_t kOffCum = kOffRingIds + 96;    // unit-id ring: ids, tags, claims [8] each
    static constexpr size_t smem_bytes(int cum_entries) { return kOffCum + (size_t)cum_entries * 4; }
};

struct Params {
    const unsigned char *q;
    const unsigned char *kc;
    const unsigned char *vc;
    const int32_t *tables;
    const int32_t *lens;
    float *ws_acc;
    float2 *ws_ml;
    void *out;
    int32_t *err;
    int32_t max_blocks;
    int32_t max_context;
    int32_t num_seqs;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t num_blocks;
    int32_t part_tokens;  // 0 = whole context is one unit
    int32_t max_parts;
    int32_t seq_tokens;   // split: tokens per per-sequence unit (a multiple of part_tokens)
    float scale_log2;
    // shared-prefix groups (split contexts only; nullptr = none): first_t[s] is the
    // number of leading tokens of s computed by its group's unit (the shared full
    // blocks, at least part_tokens; all of s when the group-rows unit also takes
    // the members' tails; 0 outside a group)
    const int32_t *first_t;
    const int4 *groups;     // (first seq, members, shared tokens, units before: tile groups;
                            //  1 when the unit takes the members' tails: row groups)
    const int32_t *meta;    // [0] tile groups, [1] their units, [2] / [3] work counters of the
                            // per-sequence and tile kernels, [4] tile CTAs, [5] row groups,
                            // [6] group-rows work counter, [7] group-rows CTAs
    int32_t max_members;    // sequences per tile group: query rows members x g <= 128
    int32_t row_groups;     // detection may form row groups (the group-rows kernel runs)
    int32_t wait_first;     // launched right behind a cache write: wait for it first
    float v_scale;          // fp8 pools: value dequantisation scale (1 otherwise)
    unsigned long long wait_ns;  // bound of every in-kernel wait
    int32_t *work_ctr;      // units handed out beyond the first gridDim.x (zeroed by the
                            // detection kernel of this call), or nullptr: static order
    int32_t num_sms;        // SMs of the device (the detection kernel splits them)
    // detection: blocks 1..lcp_blocks compare the tables of a slice of sequences
    // each, write lcp_g[s] and then lflags[block - 1] = epoch (a 64-bit value unique
    // to the call, so stale workspace contents never match); block 0 waits for those
    // flags (0 blocks: block 0 compares all)
    int32_t *lcp_g;
    unsigned long long *lflags;
    unsigned long long epoch;
    int32_t lcp_blocks;
};

// Context length, or -1 when outside [0, max_context] or longer than its table.
__device__ __forceinline__ int check_len(const Params &p, int L) {
    if (L < 0 || L > p.max_context || (int64_t)L > (int64_t)p.max_blocks * kBlockSize) return -1;
    return L;
}
__device__ __forceinline__ int checked_len(const Params &p, int s) {
    return check_len(p, __ldg(p.lens + s));
}

// Split contexts: the first ft tokens (shared with the other members of a
// group; one partial in slot 0, written by the group's unit) are followed by
// per-sequence units of seq_tokens each; unit k writes slot slot_base(ft) + k.
// Returns the number of per-sequence units (1 unsplit).  With ft >= part_tokens
// and seq_tokens >= part_tokens the slots never exceed ceil(L / part_tokens).
__device__ __forceinline__ int seq_units(const Params &p, int L, int ft) {
    if (p.part_tokens <= 0) return 1;
    const int rem = L - ft;
    if (ft == 0 && rem <= 0) return 1;  // empty context: one unit, finished as 0
    return rem > 0 ? (rem + p.seq_tokens - 1) / p.seq_tokens : 0;
}

struct Unit {
    int s, part, h;  // part: the workspace slot the unit writes
    int ft;          // first_tok(s): leading tokens of s computed by its group's unit
};

// Workspace slot of a sequence's first per-sequence unit: its shared leading
// tokens are computed together by one group unit per kv head, which writes one
// partial into slot 0.
__device__ __forceinline__ int slot_base(int ft) { return ft > 0 ? 1 : 0; }

// first_t[s] carries kDoneBit for the members of a group-rows unit that takes the
// tails: that unit covers all of s and writes s's output itself.
constexpr int kDoneBit = 1 << 30;
__device__ __forceinline__ int first_tok(const Params &p, int s) {
    return p.first_t ? (__ldg(p.first_t + s) & (kDoneBit - 1)) : 0;
}

// Unit u -> (sequence, slot, kv head).  Units [0, n_extra) are the further
// units of long sequences (slots after their first unit's), sequence-major, kv
// head innermost, using cum[s] = sum_{s' < s} (seq_units(s') - 1)^+; after them
// comes the first per-sequence unit (slot slot_base(ft)) of every sequence that
// has one, using cum[S + 1 + s] (their count before s).  Most sequences have a
// first unit only, often short, so the queue tends to end on short units (a strict
// longest-first order of the first units was measured slower on B200).
__device__ __forceinline__ Unit unit_of(const Params &p, int64_t u, int64_t n_extra, int hkv,
                                        const int *cum, int S) {
    if (u >= n_extra) {
        const int64_t f = u - n_extra;
        const int fi = (int)(f / hkv);
        int s = fi;  // identity when every sequence has a first unit
        if (p.first_t != nullptr && cum[2 * S + 1] != S) {
            const int *cumf = cum + S + 1;
            int lo = 0, hi = S;  // cumf[lo] <= fi < cumf[hi]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (cumf[mid] <= fi) lo = mid; else hi = mid;
            }
            s = lo;
        }
        const int ft = first_tok(p, s);
        return Unit{s, slot_base(ft), (int)(f % hkv), ft};
    }
    const int64_t v = u;
    const int e = (int)(v / hkv), h = (int)(v % hkv);
    int lo = 0, hi = S;  // cum[lo] <= e < cum[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cum[mid] <= e) lo = mid; else hi = mid;
    }
    const int ft = first_tok(p, lo);
    return Unit{lo, slot_base(ft) + 1 + e - cum[lo], h, ft};
}

// What one warp needs to know about a unit.  `tab` holds, in lane i, the table
// entry of the unit's logical block i (for i < 32).
struct WarpUnit {
    Unit un;
    int L;    // validated context length (0 when invalid)
    int t0;   // first token of the partition
    int nt;   // tokens in the partition
    int nb;   // blocks in the partition
    int tab;
    const int32_t *trow;
    bool skip;  // partition past the end (every partition was covered by a group unit)
    int nrow;   // group-rows mode: query rows in use (members x g)
    int nsh;    // group-rows mode: shared blocks (items [0, nsh)); items after them are the
                // members' tails, kTailBlocks slots per member (empty past a member's tail)
    int mlen;   // group-rows mode with tails: lane m holds member m's context length
    bool full;  // group-rows mode: the unit covers its members entirely (writes the output)
};

// A tail slot past its member's tail: no block to load (not an error).
constexpr int kEmptyItem = -2;

// Group-rows mode: unit v = (row group v / Hkv, kv head v % Hkv).  Its keys are
// the group's shared tokens (whole blocks of the first member's table); its rows
// are members x g query heads, member-major.
__device__ __forceinline__ void load_unit_rows(const Params &p, int64_t v, int gbase, WarpUnit &w, int lane) {
    const int hkv = p.num_kv_heads;
    const int4 gr = __ldg(p.groups + gbase + (int)(v / hkv));  // (first seq, members, shared tokens, tails)
    w.un = Unit{gr.x, 0, (int)(v % hkv), gr.z};
    w.L = gr.z;
    w.t0 = 0;
    w.nt = gr.z;
    w.nsh = gr.z / kBlockSize;
    w.nb = w.nsh + (gr.w ? gr.y * kTailBlocks : 0);
    w.mlen = gr.w && lane < gr.y ? max(checked_len(p, gr.x + lane), 0) : 0;
    w.full = gr.w != 0;
    w.trow = p.tables + (int64_t)gr.x * p.max_blocks;
    w.tab = lane < p.max_blocks ? __ldg(w.trow + lane) : -1;
    w.skip = false;
    w.nrow = gr.y * (p.num_q_heads / hkv);
}

__device__ __forceinline__ void load_unit(const Params &p, int64_t u, int64_t n_extra,
                                          const int *cum, WarpUnit &w, int lane, bool flagger) {
    w.un = unit_of(p, u, n_extra, p.num_kv_heads, cum, p.num_seqs);
    const int k = w.un.part - slot_base(w.un.ft);  // per-sequence unit index
    const int t_first = p.part_tokens > 0 ? w.un.ft + k * p.seq_tokens : 0;
    const int b0 = t_first / kBlockSize;
    w.trow = p.tables + (int64_t)w.un.s * p.max_blocks + b0;
    // both loads issued before either value is needed
    const int raw = __ldg(p.lens + w.un.s);
    w.tab = lane < p.max_blocks - b0 ? __ldg(w.trow + lane) : -1;
    int L = check_len(p, raw);
    if (L < 0) {
        if (flagger && lane == 0 && w.un.part == 0 && w.un.h == 0) flag_error(p.err, PA_DEVERR_CONTEXT_LEN);
        L = 0;
    }
    w.L = L;
    if (p.part_tokens <= 0) {
        w.t0 = 0;
        w.nt = L;
    } else {
        w.t0 = t_first;
        w.nt = max(0, min(L, w.t0 + p.seq_tokens) - w.t0);
    }
    w.skip = k >= seq_units(p, L, w.un.ft);
    if (w.skip) w.nt = 0;
    w.nb = (w.nt + kBlockSize - 1) / kBlockSize;
}

// Prologue (split contexts): cum[s] = sum_{s' < s} (seq_units(s') - 1)^+ and, at
// cum[S + 1 + s], the number of s' < s with seq_units(s') >= 1 (sequences whose
// every token is covered by a group unit have no per-sequence unit at all);
// exclusive scans, one chunk of sequences per thread.  Ends with __syncthreads.
__device__ __forceinline__ void prologue(const Params &p, int *cum, int *scratch) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (p.part_tokens > 0) {
        const int S = p.num_seqs;
        int *cumf = cum + S + 1;  // written only on the shared-prefix path (first_t set)
        const bool wf = p.first_t != nullptr;
        const int per = (S + kThreads - 1) / kThreads;
        const int beg = min(S, (int)threadIdx.x * per), end = min(S, beg + per);
        int local = 0, localf = 0;
        for (int s = beg; s < end; ++s) {
            const int L = checked_len(p, s);
            const int su = seq_units(p, L < 0 ? 0 : L, first_tok(p, s));
            local += max(0, su - 1);
            localf += su > 0 ? 1 : 0;
        }
        int incl = local, inclf = localf;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, incl, o), yf = __shfl_up_sync(kFull, inclf, o);
            if (lane >= o) {
                incl += y;
                inclf += yf;
            }
        }
        if (lane == 31) {
            scratch[warp] = incl;
            scratch[kWarps + warp] = inclf;
        }
        __syncthreads();
        int off = 0, offf = 0;
        for (int w = 0; w < warp; ++w) {
            off += scratch[w];
            offf += scratch[kWarps + w];
        }
        int run = off + incl - local, runf = offf + inclf - localf;
        for (int s = beg; s < end; ++s) {
            cum[s] = run;
            if (wf) cumf[s] = runf;
            const int L = checked_len(p, s);
            const int su = seq_units(p, L < 0 ? 0 : L, first_tok(p, s));
            run += max(0, su - 1);
            runf += su > 0 ? 1 : 0;
        }
        if ((int)threadIdx.x == kThreads - 1) {
            cum[S] = run;
            if (wf) cumf[S] = runf;
        }
    }
    __syncthreads();
}

// Issue the cp.async copies of one (block, kv head) slab pair into a stage.
// bf16 rows are 2*D bytes (fp8: D); chunk c of row r goes to chunk position
// (c & ~7) | ((c ^ r) & 7), which keeps 8 consecutive rows of any column in 8
// different bank groups.  fp32 rows keep their natural order.
template <typename T, int D, int G>
__device__ __forceinline__ void issue_slabs(const Params &p, uint32_t stage, int blk, int h,
                                            int lane) {
    using Lay = Layout<T, D, G>;
    constexpr int kChunksPerRow = Lay::kRowBytes / 16;
    constexpr int kChunks = Lay::kSlabBytes / 16;
    const int64_t off = ((int64_t)blk * p.num_kv_heads + h) * Lay::kSlabBytes;
    const unsigned char *ks = p.kc + off;
    const unsigned char *vs = p.vc + off;
#pragma unroll
    for (int i = lane; i < kChunks; i += 32) {
        const int r = i / kChunksPerRow, c = i % kChunksPerRow;
        const int pc = sizeof(T) <= 2 ? ((c & ~7) | ((c ^ r) & 7)) : c;
        const uint32_t d = stage + r * Lay::kRowBytes + pc * 16;
        cp_async16(d, ks + i * 16);
        cp_async16(d + Lay::kSlabBytes, vs + i * 16);
    }
}

template <typename T>
__device__ __forceinline__ void store_out(void *out, int64_t idx, float v);
template <>
__device__ __forceinline__ void store_out<float>(void *out, int64_t idx, float v) {
    static_cast<float *>(out)[idx] = v;
}
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(void *out, int64_t idx, float v) {
    static_cast<__nv_bfloat16 *>(out)[idx] = __float2bfloat16_rn(v);
}

// After the warps' states of a unit are in macc/mml: combine them and write the
// output (single partition) or the partition's (m, l, acc) to the workspace.
template <typename T, int D, int G>
__device__ __forceinline__ void finish_unit(const Params &p, const WarpUnit &w, const float *uacc,
                                            const float2 *uml) {
    if (w.skip) return;
    const bool single = w.un.ft == 0 && seq_units(p, w.L, 0) == 1;
    const int64_t head0 = (int64_t)w.un.s * p.num_q_heads + (int64_t)w.un.h * G;
    for (int e = threadIdx.x; e < G * D; e += kThreads) {
        const int h = e / D, dd = e - h * D;
        float M = -INFINITY;
#pragma unroll
        for (int k = 0; k < kWarps; ++k) M = fmaxf(M, uml[k * G + h].x);
        float lsum = 0.f, o = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int k = 0; k < kWarps; ++k) {
                const float2 ml = uml[k * G + h];
                if (ml.x != -INFINITY) {
                    const float f = fast_exp2(ml.x - M);
                    lsum = fmaf(ml.y, f, lsum);
                    o = fmaf(uacc[(k * G + h) * D + dd], f, o);
                }
            }
        }
        if constexpr (kIsFp8<T>) o *= p.v_scale;
        if (single) {
            store_out<IoT<T>>(p.out, (head0 + h) * D + dd, lsum > 0.f ? o * (1.f / lsum) : 0.f);
        } else {
            const int64_t row = (head0 + h) * p.max_parts + w.un.part;
            p.ws_acc[row * D + dd] = o;
            if (dd == 0) p.ws_ml[row] = make_float2(M, lsum);
        }
    }
}

// Group-rows mode: combine the warps' states of a unit (rows r < w.nrow) and
// write the partial of its shared tokens into workspace slot 0 of every member:
// row r is query head h g + r % g of sequence first + r / g.
template <typename T, int D>
__device__ __forceinline__ void finish_unit_rows(const Params &p, const WarpUnit &w, const float *uacc,
                                                 const float2 *uml) {
    const int g = p.num_q_heads / p.num_kv_heads;
    for (int e = threadIdx.x; e < kRowTile * D; e += kThreads) {
        const int r = e / D, dd = e - r * D;
        if (r >= w.nrow) break;  // rows only grow with e
        float M = -INFINITY;
#pragma unroll
        for (int k = 0; k < kWarps; ++k) M = fmaxf(M, uml[k * kRowTile + r].x);
        float lsum = 0.f, o = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int k = 0; k < kWarps; ++k) {
                const float2 ml = uml[k * kRowTile + r];
                if (ml.x != -INFINITY) {
                    const float f = fast_exp2(ml.x - M);
                    lsum = fmaf(ml.y, f, lsum);
                    o = fmaf(uacc[(k * kRowTile + r) * D + dd], f, o);
                }
            }
        }
        if constexpr (kIsFp8<T>) o *= p.v_scale;
        const int64_t qrow = (int64_t)(w.un.s + r / g) * p.num_q_heads + (int64_t)w.un.h * g + r % g;
        if (w.full) {  // the unit covered every key of its members: the output itself
            store_out<IoT<T>>(p.out, qrow * D + dd, lsum > 0.f ? o * (1.f / lsum) : 0.f);
        } else {
            const int64_t row = qrow * p.max_parts;
            p.ws_acc[row * D + dd] = o;
            if (dd == 0) p.ws_ml[row] = make_float2(M, lsum);
        }
    }
}

// ------------------------------------------------------------- bf16 block
// Per-warp state of the tensor-core path.  m, l: online-softmax state of this
// thread's two head columns 2*(lane%4) and 2*(lane%4)+1; o: O^T accumulator
// fragments (rows = head dims, cols = heads); qb: Q^T operand fragments.
template <int D>
struct MmaState {
    float m[2], l[2];
    float o[D / 16][4];
    uint32_t qb[D / 16][2];
};

// Online-softmax step over NT 16-token tiles.  s[i]: tile i's scores in log2
// units as S^T fragments (tokens lane/4 and lane/4 + 8, head columns 2(lane%4)
// and 2(lane%4)+1).  Masks tokens at or past ntok[i] (ntok 0: the whole tile),
// updates m and l, rescales the O^T accumulators and leaves the unnormalised
// probabilities in s.  At least one tile must hold a token.
template <int D, int NT>
__device__ __forceinline__ void softmax_tiles(float (&s)[NT][4], const int (&ntok)[NT], MmaState<D> &st,
                                              int lane) {
    constexpr int KS = D / 16;
    const int t0 = lane >> 2;
#pragma unroll
    for (int i = 0; i < NT; ++i) {
        if (t0 >= ntok[i]) s[i][0] = s[i][1] = -INFINITY;
        if (t0 + 8 >= ntok[i]) s[i][2] = s[i][3] = -INFINITY;
    }
    float c0 = fmaxf(s[0][0], s[0][2]), c1 = fmaxf(s[0][1], s[0][3]);
#pragma unroll
    for (int i = 1; i < NT; ++i) {
        c0 = fmaxf(c0, fmaxf(s[i][0], s[i][2]));
        c1 = fmaxf(c1, fmaxf(s[i][1], s[i][3]));
    }
    // online softmax per head column over the tiles' tokens
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        c0 = fmaxf(c0, __shfl_xor_sync(kFull, c0, off));
        c1 = fmaxf(c1, __shfl_xor_sync(kFull, c1, off));
    }
    const float mn0 = fmaxf(st.m[0], c0), mn1 = fmaxf(st.m[1], c1);
    const float al0 = fast_exp2(st.m[0] - mn0), al1 = fast_exp2(st.m[1] - mn1);
#pragma unroll
    for (int i = 0; i < NT; ++i) {
        s[i][0] = fast_exp2(s[i][0] - mn0);
        s[i][1] = fast_exp2(s[i][1] - mn1);
        s[i][2] = fast_exp2(s[i][2] - mn0);
        s[i][3] = fast_exp2(s[i][3] - mn1);
    }
    float r0 = s[0][0] + s[0][2], r1 = s[0][1] + s[0][3];
#pragma unroll
    for (int i = 1; i < NT; ++i) {
        r0 += s[i][0] + s[i][2];
        r1 += s[i][1] + s[i][3];
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        r0 += __shfl_xor_sync(kFull, r0, off);
        r1 += __shfl_xor_sync(kFull, r1, off);
    }
    st.l[0] = st.l[0] * al0 + r0;
    st.l[1] = st.l[1] * al1 + r1;
    st.m[0] = mn0;
    st.m[1] = mn1;
    if (__any_sync(kFull, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
            st.o[mt][0] *= al0;
            st.o[mt][1] *= al1;
            st.o[mt][2] *= al0;
            st.o[mt][3] *= al1;
        }
    }
}

template <int D>
__device__ __forceinline__ void softmax_block(float (&s)[4], int ntok, MmaState<D> &st, int lane) {
    float t[1][4] = {{s[0], s[1], s[2], s[3]}};
    const int n[1] = {ntok};
    softmax_tiles<D, 1>(t, n, st, lane);
#pragma unroll
    for (int k = 0; k < 4; ++k) s[k] = t[0][k];
}

// One 16-token block on tensor-core tiles.  kb: shared address of the K slab
// (V slab follows), rows of 2*D bytes with swizzled 16-byte chunks.
template <int D>
__device__ __forceinline__ void mma_block(uint32_t kb, unsigned char *vgen, int ntok,
                                          MmaState<D> &st, float sl2, int lane) {
    constexpr int KS = D / 16;
    constexpr int kRow = 2 * D;
    const uint32_t vb = kb + kBlockSize * kRow;
    const int mat = lane >> 3, r8 = lane & 7;
    auto addr = [&](uint32_t base, int row, int chunk) {
        return base + row * kRow + ((((chunk & ~7) | ((chunk ^ row) & 7))) << 4);
    };
    // S^T = K Q^T: rows = tokens, cols = heads (two accumulators halve the chain)
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
    const int krow = ((mat & 1) << 3) + r8;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
        uint32_t a[4];
        ldsm_x4(a, addr(kb, krow, kk * 2 + (mat >> 1)));
        if (kk & 1) mma_bf16_16816(sb, a, st.qb[kk][0], st.qb[kk][1]);
        else mma_bf16_16816(sa, a, st.qb[kk][0], st.qb[kk][1]);
    }
    float s[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) s[k] = (sa[k] + sb[k]) * sl2;
    softmax_block<D>(s, ntok, st, lane);
    const float p0 = s[0], p1 = s[1], p2 = s[2], p3 = s[3];
    // P^T operand fragments: rows 0-7 / 8-15 of S^T, transposed in registers
    const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0, p1));
    const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2, p3));
    if (ntok < kBlockSize) {
        // zero the V rows past the context: 0 * (NaN or Inf) would poison the sums
        for (int idx = lane; idx < (kBlockSize - ntok) * (kRow / 16); idx += 32)
            *reinterpret_cast<uint4 *>(vgen + (ntok + idx / (kRow / 16)) * kRow + (idx % (kRow / 16)) * 16) =
                make_uint4(0, 0, 0, 0);
        __syncwarp();
    }
    // O^T += V^T P^T: rows = head dims, cols = heads
    const int vrow = ((mat >> 1) << 3) + r8;
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) {
        uint32_t a[4];
        ldsm_x4_trans(a, addr(vb, vrow, mt * 2 + (mat & 1)));
        mma_bf16_16816(st.o[mt], a, pb0, pb1);
    }
}

// Group-rows mode: the state of 16 query rows, two 8-column tiles (n = 0, 1).
// m, l: columns 2(lane%4), 2(lane%4)+1 of tile 0, then of tile 1; o: O^T
// accumulators per (head-dim tile, column tile); qb: Q^T operand fragments.
template <int D>
struct MmaRows {
    float m[4], l[4];
    float o[D / 16][2][4];
    uint32_t qb[D / 16][2][2];
};

// Group-rows mode: one online-softmax step per column over one 16-token block.
// s[n]: column tile n's scores in log2 units as S^T fragments (tokens lane/4 and
// lane/4 + 8, columns 2(lane%4) and 2(lane%4)+1), -inf where a column does not
// see the block.  Masks tokens at or past ntok (>= 1), updates m and l, rescales
// the O^T accumulators and leaves the unnormalised probabilities in s.  A column
// that has seen no key yet keeps m = -inf and contributes nothing (its reference
// point is taken as 0, so no -inf - -inf arises).
template <int D>
__device__ __forceinline__ void softmax_rows(float (&s)[2][4], int ntok, MmaRows<D> &st, int lane) {
    constexpr int KS = D / 16;
    const int t0 = lane >> 2;
    float c[4], al[4];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
        if (t0 >= ntok) s[n][0] = s[n][1] = -INFINITY;
        if (t0 + 8 >= ntok) s[n][2] = s[n][3] = -INFINITY;
        c[2 * n] = fmaxf(s[n][0], s[n][2]);
        c[2 * n + 1] = fmaxf(s[n][1], s[n][3]);
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1)
#pragma unroll
        for (int i = 0; i < 4; ++i) c[i] = fmaxf(c[i], __shfl_xor_sync(kFull, c[i], off));
    float ref[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float mn = fmaxf(st.m[i], c[i]);
        ref[i] = mn == -INFINITY ? 0.f : mn;
        al[i] = fast_exp2(st.m[i] - ref[i]);
        st.m[i] = mn;
    }
    float r[4];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
        s[n][0] = fast_exp2(s[n][0] - ref[2 * n]);
        s[n][1] = fast_exp2(s[n][1] - ref[2 * n + 1]);
        s[n][2] = fast_exp2(s[n][2] - ref[2 * n]);
        s[n][3] = fast_exp2(s[n][3] - ref[2 * n + 1]);
        r[2 * n] = s[n][0] + s[n][2];
        r[2 * n + 1] = s[n][1] + s[n][3];
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1)
#pragma unroll
        for (int i = 0; i < 4; ++i) r[i] += __shfl_xor_sync(kFull, r[i], off);
#pragma unroll
    for (int i = 0; i < 4; ++i) st.l[i] = st.l[i] * al[i] + r[i];
    if (__any_sync(kFull, al[0] != 1.f || al[1] != 1.f || al[2] != 1.f || al[3] != 1.f)) {
#pragma unroll
        for (int mt = 0; mt < KS; ++mt)
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                st.o[mt][n][0] *= al[2 * n];
                st.o[mt][n][1] *= al[2 * n + 1];
                st.o[mt][n][2] *= al[2 * n];
                st.o[mt][n][3] *= al[2 * n + 1];
            }
    }
}

// One 16-token block against 16 query rows: S^T = K Q^T as two 16 x 8 tiles
// sharing every K fragment, one online-softmax step per column, then
// O^T += V^T P^T with every V fragment feeding both column tiles.
template <int D>
__device__ __forceinline__ void mma_block_rows(uint32_t kb, unsigned char *vgen, int ntok, int c_lo, int c_hi,
                                               MmaRows<D> &st, float sl2, int lane) {
    constexpr int KS = D / 16;
    constexpr int kRow = 2 * D;
    const uint32_t vb = kb + kBlockSize * kRow;
    const int mat = lane >> 3, r8 = lane & 7;
    auto addr = [&](uint32_t base, int row, int chunk) {
        return base + row * kRow + ((((chunk & ~7) | ((chunk ^ row) & 7))) << 4);
    };
    // two accumulators per column tile (even / odd k steps) halve the MMA chains
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float s2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const int krow = ((mat & 1) << 3) + r8;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
        uint32_t a[4];
        ldsm_x4(a, addr(kb, krow, kk * 2 + (mat >> 1)));
        float(&d0)[4] = (kk & 1) ? s2[0] : s[0];
        float(&d1)[4] = (kk & 1) ? s2[1] : s[1];
        mma_bf16_16816(d0, a, st.qb[kk][0][0], st.qb[kk][0][1]);
        mma_bf16_16816(d1, a, st.qb[kk][1][0], st.qb[kk][1][1]);
    }
#pragma unroll
    for (int n = 0; n < 2; ++n) {
#pragma unroll
        for (int k = 0; k < 4; ++k) s[n][k] = (s[n][k] + s2[n][k]) * sl2;
        // columns (query rows) outside [c_lo, c_hi) do not see this block
        const int c0 = 8 * n + 2 * (lane & 3);
        if (c0 < c_lo || c0 >= c_hi) s[n][0] = s[n][2] = -INFINITY;
        if (c0 + 1 < c_lo || c0 + 1 >= c_hi) s[n][1] = s[n][3] = -INFINITY;
    }
    softmax_rows<D>(s, ntok, st, lane);
    // P^T operand fragments of both column tiles, transposed in registers
    uint32_t pb[2][2];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
        pb[n][0] = movmatrix_trans(pack_bf16x2(s[n][0], s[n][1]));
        pb[n][1] = movmatrix_trans(pack_bf16x2(s[n][2], s[n][3]));
    }
    if (ntok < kBlockSize) {
        // zero the V rows past the keys: 0 * (NaN or Inf) would poison the sums
        for (int idx = lane; idx < (kBlockSize - ntok) * (kRow / 16); idx += 32)
            *reinterpret_cast<uint4 *>(vgen + (ntok + idx / (kRow / 16)) * kRow + (idx % (kRow / 16)) * 16) =
                make_uint4(0, 0, 0, 0);
        __syncwarp();
    }
    const int vrow = ((mat >> 1) << 3) + r8;
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) {
        uint32_t a[4];
        ldsm_x4_trans(a, addr(vb, vrow, mt * 2 + (mat & 1)));
        mma_bf16_16816(st.o[mt][0], a, pb[0][0], pb[0][1]);
        mma_bf16_16816(st.o[mt][1], a, pb[1][0], pb[1][1]);
    }
}

// ------------------------------------------------------------- fp8 block
// Four e4m3 codes (bytes 0..3 of w) -> two f16x2 registers (exact): lo holds
// bytes 0, 1 and hi bytes 2, 3, the lower byte in the lower half of each.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t &lo, uint32_t &hi) {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

// NT (1 or 2) 16-token blocks of an fp8 pool on f16 tensor-core tiles, with one
// softmax step for all of them: two blocks per step interleave their QK chains
// and halve the shuffle reductions per token.  kb[i]: block i's stage (K slab,
// V slab behind it), rows of D = 128 bytes, 16-byte chunk c of row r stored at
// chunk position c ^ (r & 7); ntok[i]: its tokens (0: skip the block).  Head
// dims are laid on the mma slots so that each thread reads whole chunks,
// conflict free:
//   S^T = K Q^T: at k step kk = 4j + i, thread (g, t) = (lane/4, lane%4) holds
//     dims 32t + 16j + 4i + {0,1} in k slots 2t, 2t+1 and + {2,3} in 2t+8, 2t+9
//     (its query fragments follow the same map);
//   O^T = V^T P^T: accumulator row g of m tile mt is dim 16g + 2mt, row g + 8 is
//     dim 16g + 2mt + 1, so thread (g, t) reads chunk g of token rows 2t, 2t+1,
//     2t+8, 2t+9.
template <int D, int NT>
__device__ __forceinline__ void mma_tiles_fp8(unsigned char *const (&kb)[NT], const int (&ntok)[NT],
                                              MmaState<D> &st, float sl2, int lane) {
    static_assert(D == 128, "the fp8 fragment map assumes 128-byte rows");
    constexpr int kSlab = kBlockSize * D;
    const int g = lane >> 2, t = lane & 3;
    auto chunk = [&](const unsigned char *base, int row, int c) {
        return *reinterpret_cast<const uint4 *>(base + row * D + ((c ^ (row & 7)) << 4));
    };
    float s[NT][4];
#pragma unroll
    for (int b = 0; b < NT; ++b) {
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint4 lo = chunk(kb[b], g, 2 * t + j), hi = chunk(kb[b], g + 8, 2 * t + j);
            const uint32_t wl[4] = {lo.x, lo.y, lo.z, lo.w}, wh[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int kk = 4 * j + i;
                uint32_t a[4];
                e4m3x4_to_f16x2x2(wl[i], a[0], a[2]);
                e4m3x4_to_f16x2x2(wh[i], a[1], a[3]);
                if (kk & 1) mma_f16_16816(sb, a, st.qb[kk][0], st.qb[kk][1]);
                else mma_f16_16816(sa, a, st.qb[kk][0], st.qb[kk][1]);
            }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) s[b][k] = (sa[k] + sb[k]) * sl2;
    }
    softmax_tiles<D, NT>(s, ntok, st, lane);
    uint32_t pb0[NT], pb1[NT];
    bool zero = false;
#pragma unroll
    for (int b = 0; b < NT; ++b) {
        pb0[b] = movmatrix_trans(pack_f16x2(s[b][0], s[b][1]));
        pb1[b] = movmatrix_trans(pack_f16x2(s[b][2], s[b][3]));
        if (ntok[b] < kBlockSize) {
            // codes past the context (or of a skipped block) may be NaN: zero those V rows
            unsigned char *vb = kb[b] + kSlab;
            for (int idx = lane; idx < (kBlockSize - ntok[b]) * (D / 16); idx += 32)
                *reinterpret_cast<uint4 *>(vb + (ntok[b] + idx / (D / 16)) * D + (idx % (D / 16)) * 16) =
                    make_uint4(0, 0, 0, 0);
            zero = true;
        }
    }
    if (zero) __syncwarp();
#pragma unroll
    for (int b = 0; b < NT; ++b) {
        const unsigned char *vb = kb[b] + kSlab;
        const uint4 v0 = chunk(vb, 2 * t, g), v1 = chunk(vb, 2 * t + 1, g);
        const uint4 v2 = chunk(vb, 2 * t + 8, g), v3 = chunk(vb, 2 * t + 9, g);
        const uint32_t r0[4] = {v0.x, v0.y, v0.z, v0.w}, r1[4] = {v1.x, v1.y, v1.z, v1.w};
        const uint32_t r2[4] = {v2.x, v2.y, v2.z, v2.w}, r3[4] = {v3.x, v3.y, v3.z, v3.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            // interleave token pairs (2t, 2t+1) and (2t+8, 2t+9) of dims 4w+{0,1}, 4w+{2,3}
            const uint32_t e01 = __byte_perm(r0[w], r1[w], 0x5140), f01 = __byte_perm(r0[w], r1[w], 0x7362);
            const uint32_t e23 = __byte_perm(r2[w], r3[w], 0x5140), f23 = __byte_perm(r2[w], r3[w], 0x7362);
            uint32_t a[4];
            e4m3x4_to_f16x2x2(e01, a[0], a[1]);
            e4m3x4_to_f16x2x2(e23, a[2], a[3]);
            mma_f16_16816(st.o[2 * w], a, pb0[b], pb1[b]);
            e4m3x4_to_f16x2x2(f01, a[0], a[1]);
            e4m3x4_to_f16x2x2(f23, a[2], a[3]);
            mma_f16_16816(st.o[2 * w + 1], a, pb0[b], pb1[b]);
        }
    }
}

// ------------------------------------------------------------- fp32 block
template <int D, int G>
struct F32Cfg {
    static constexpr int kRowBytes = D * 4;
    static constexpr int kQkChunks = kRowBytes / 128;   // 16-byte chunks per lane (8 lanes/token)
    static constexpr int kQkPairs = kQkChunks * 2;      // float2 of q per head per lane
    static constexpr int kDpl = D / 32;                 // PV dims per lane
    static constexpr int kPvPairs = kDpl / 2;
    static constexpr int kLogG = ilog2(G);
    static constexpr int kDupMask = (8 >> kLogG) - 1;  // lanes holding the same score
};

template <int D, int G>
struct F32State {
    float m, l;
    float2 acc[G][F32Cfg<D, G>::kPvPairs];
    float2 qreg[G][F32Cfg<D, G>::kQkPairs];
};

// Transposing reduction over the 8 lanes of one token (lanes differing in bits
// 0..2).  Lane holds N partial sums (one per head); each level halves the set,
// keeping the upper or lower half according to the lane's bit, and adds the
// partner's copy of the kept half.  When one value is left the remaining levels
// are plain butterflies.  Result: lane `part` holds head part >> (3 - log2 N).
template <int N, int BIT>
__device__ __forceinline__ float reduce8(float *w, int part) {
    if constexpr (BIT < 0) {
        return w[0];
    } else if constexpr (N > 1) {
        constexpr int H = N / 2;
        const bool up = (part >> BIT) & 1;
#pragma unroll
        for (int k = 0; k < H; ++k) {
            const float keep = up ? w[k + H] : w[k];
            const float send = up ? w[k] : w[k + H];
            w[k] = keep + __shfl_xor_sync(kFull, send, 1 << BIT);
        }
        return reduce8<H, BIT - 1>(w, part);
    } else {
        w[0] += __shfl_xor_sync(kFull, w[0], 1 << BIT);
        return reduce8<1, BIT - 1>(w, part);
    }
}

template <int D, int G>
__device__ __forceinline__ void f32_block(const unsigned char *kb, const unsigned char *vb, int ntok,
                                          F32State<D, G> &st, float *pw, int lane) {
    using C = F32Cfg<D, G>;
    const int tq = lane >> 3, part = lane & 7;
    const int hd = part >> (3 - C::kLogG);
    float sc[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int t = tq + 4 * r;
        float2 a[G];
#pragma unroll
        for (int h = 0; h < G; ++h) a[h] = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < C::kQkChunks; ++i) {
            const float4 kv = *reinterpret_cast<const float4 *>(kb + t * C::kRowBytes + (part + 8 * i) * 16);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                a[h] = ffma2(st.qreg[h][2 * i], make_float2(kv.x, kv.y), a[h]);
                a[h] = ffma2(st.qreg[h][2 * i + 1], make_float2(kv.z, kv.w), a[h]);
            }
        }
        float v[G];
#pragma unroll
        for (int h = 0; h < G; ++h) v[h] = a[h].x + a[h].y;
        const float s = reduce8<G, 2>(v, part);
        sc[r] = t < ntok ? s : -INFINITY;
    }
    float bm = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    bm = fmaxf(bm, __shfl_xor_sync(kFull, bm, 8));
    bm = fmaxf(bm, __shfl_xor_sync(kFull, bm, 16));
    const float m_new = fmaxf(st.m, bm);
    const float alpha = fast_exp2(st.m - m_new);
    float ps = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        sc[r] = fast_exp2(sc[r] - m_new);
        ps += sc[r];
    }
    ps += __shfl_xor_sync(kFull, ps, 8);
    ps += __shfl_xor_sync(kFull, ps, 16);
    st.l = st.l * alpha + ps;
    st.m = m_new;
    if ((part & C::kDupMask) == 0) {
#pragma unroll
        for (int r = 0; r < 4; ++r) pw[(tq + 4 * r) * G + hd] = sc[r];
        if (tq == 0) pw[16 * G + hd] = alpha;
    }
    __syncwarp();
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float al = pw[16 * G + h];
#pragma unroll
        for (int k = 0; k < C::kPvPairs; ++k) {
            st.acc[h][k].x *= al;
            st.acc[h][k].y *= al;
        }
    }
    const unsigned char *vrow = vb + lane * C::kDpl * 4;
#pragma unroll
    for (int t = 0; t < kBlockSize; ++t) {
        if (t < ntok) {
            float2 vv[C::kPvPairs];
            if constexpr (C::kPvPairs == 2) {
                const float4 x = *reinterpret_cast<const float4 *>(vrow + t * C::kRowBytes);
                vv[0] = make_float2(x.x, x.y);
                vv[1] = make_float2(x.z, x.w);
            } else {
                vv[0] = *reinterpret_cast<const float2 *>(vrow + t * C::kRowBytes);
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float pt = pw[t * G + h];
#pragma unroll
                for (int k = 0; k < C::kPvPairs; ++k)
                    st.acc[h][k] = ffma2(make_float2(pt, pt), vv[k], st.acc[h][k]);
            }
        }
    }
    __syncwarp();  // pw is rewritten by the next block
}

// ------------------------------------------------------------- the kernel
// Blocks of the warp's work, one after another: blocks w, w+8, ... of the current
// unit, then of the next one.  Each is fetched with cp.async up to NS items before
// it is computed.  (An extra prefetch.global.L2 a few items further ahead measured
// slower on B200 at every distance tried, as did a third stage per warp.)

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ Params p) {
    using Lay = Layout<T, D, G>;
    constexpr bool kFp8 = kIsFp8<T>;
    constexpr bool kMma = sizeof(T) <= 2;  // bf16 and fp8 run on tensor-core tiles
    constexpr int NS = Lay::kStagesPerWarp;
    extern __shared__ __align__(128) unsigned char smem[];
    float *pbuf = reinterpret_cast<float *>(smem + Lay::kOffP);
    float *macc = reinterpret_cast<float *>(smem + Lay::kOffMacc);
    float2 *mml = reinterpret_cast<float2 *>(smem + Lay::kOffMml);
    int *cum = reinterpret_cast<int *>(smem + Lay::kOffCum);

    constexpr bool kRows = Lay::kRows;
    static_assert(Lay::kMergeBufs == 2 || kRows, "the deferred merge needs two slots");
    static_assert(!kRows || (kMma && !kFp8), "group-rows mode runs on bf16 tensor-core tiles");
    // The combine may start launching now; it waits for this grid to finish.
    // When launched behind the group tiles, this grid reads only what the
    // detection wrote (complete before the tiles let it start) and writes other
    // partitions; it waits for the tiles only before exiting, so that its
    // completion implies theirs.  Launched right behind a cache write instead
    // (pa_append_decode without groups), it waits for the write first.
    grid_dep_launch();
    if (p.wait_first) grid_dep_wait();
    // Group-rows mode: the detection kernel chose how many CTAs take row-group
    // units (ids from the counter meta[6]); the others leave their SM at once.
    // CTA 0 always stays until the previous kernel of the call has finished, so
    // that this grid's completion implies it (the next kernel waits for this grid).
    int dyn_base = (int)gridDim.x;
    if constexpr (kRows) {
        dyn_base = min((int)gridDim.x, __ldg(p.meta + 7));
        if ((int)blockIdx.x >= dyn_base) {
            if (blockIdx.x == 0) grid_dep_wait();
            return;
        }
    }
    // merge slot hand-over: full[b] when all warps wrote their state of the
    // slot's unit, freed[b] when all warps finished their share of its merge
    uint64_t *mfull = reinterpret_cast<uint64_t *>(smem + Lay::kOffBar);
    uint64_t *mfreed = mfull + 2;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::kOffBar + 32);
    if (threadIdx.x == 0) {
        mbar_init(&mfull[0], kWarps);
        mbar_init(&mfull[1], kWarps);
        mbar_init(&mfreed[0], kWarps);
        mbar_init(&mfreed[1], kWarps);
        *abort_flag = 0;
        mbar_init_fence();
    }
    // This CTA's units, in order: unit 0 is blockIdx.x.  With a work counter,
    // unit k >= 1 is gridDim.x + a value drawn from it, so CTAs that start early
    // (beside the group tiles) or get short units take more of them; without one
    // it is blockIdx.x + k * gridDim.x.  Ids are drawn two units ahead, in order,
    // by the first warp to start a unit, and published in a ring of 8 slots.
    volatile int *ring_id = reinterpret_cast<volatile int *>(smem + Lay::kOffRingIds);
    volatile int *ring_tag = ring_id + 8;      // unit index whose id the slot holds
    int *ring_claim = const_cast<int *>(ring_id) + 16;  // unit index last claimed for the slot
    const bool dyn = p.work_ctr != nullptr;
    if (threadIdx.x == 0) {
        for (int i = 0; i < 8; ++i) {
            ring_tag[i] = -1;
            ring_claim[i] = i - 8;
        }
        ring_tag[0] = ring_claim[0] = 0;
        if (dyn) {
            const int v = dyn_base + atomicAdd(p.work_ctr, 2);
            ring_id[1] = v;
            ring_id[2] = v + 1;
            ring_tag[1] = ring_claim[1] = 1;
            ring_tag[2] = ring_claim[2] = 2;
        }
    }
    if constexpr (kRows) __syncthreads();  // barriers and ring initialised
    else prologue(p, cum, reinterpret_cast<int *>(macc));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.num_seqs, hkv = p.num_kv_heads;
    const int64_t n_extra = !kRows && p.part_tokens > 0 ? (int64_t)cum[S] * hkv : 0;
    const int gbase = kRows ? __ldg(p.meta) : 0;  // row groups follow the tile groups
    const int64_t total = kRows ? (int64_t)__ldg(p.meta + 5) * hkv
                                : (p.first_t != nullptr ? (int64_t)cum[2 * S + 1] : (int64_t)S) * hkv + n_extra;
    auto load_any = [&](int64_t u, WarpUnit &w) {
        if constexpr (kRows) load_unit_rows(p, u, gbase, w, lane);
        else load_unit(p, u, n_extra, cum, w, lane, warp == 0);
    };
    unsigned char *wring = smem + Lay::kOffRing + (size_t)warp * NS * Lay::kStageBytes;
    const uint32_t wring_s = smem_u32(wring);
    float *pw = pbuf + warp * Lay::kPWarpFloats;
    const int q4 = lane & 3, dr = lane >> 2;

    // id of this CTA's unit k (whole warp; bounded wait for a dynamic id; INT64_MAX
    // ends the work)
    auto unit_id = [&](int k) -> int64_t {
        if (k == 0) return blockIdx.x;
        if (!dyn) return (int64_t)blockIdx.x + (int64_t)k * gridDim.x;
        int v = INT_MAX;
        if (lane == 0) {
            const unsigned long long t0 = global_ns();
            bool ok = true;
            while (ring_tag[k & 7] != k) {
                if (*abort_flag || global_ns() - t0 > p.wait_ns) {
                    if (!*abort_flag) flag_error(p.err, PA_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                    ok = false;
                    break;
                }
            }
            __threadfence_block();
            if (ok) v = ring_id[k & 7];
        }
        v = __shfl_sync(kFull, v, 0);
        return v == INT_MAX ? INT64_MAX : (int64_t)v;
    };
    // near the end of unit k (the first warp to finish its share of it): draw the
    // id of unit k + 2, after the id of unit k + 1 is out, so that a CTA's ids only
    // grow; drawn this late, a CTA holds at most one unit beyond the one it works on
    auto claim_ahead = [&](int k) {
        if (!dyn || lane != 0 || k < 1) return;
        const int k2 = k + 2, sl = k2 & 7;
        if (atomicCAS(&ring_claim[sl], k2 - 8, k2) != k2 - 8) return;
        const unsigned long long t0 = global_ns();
        while (ring_tag[(k2 - 1) & 7] != k2 - 1) {
            if (*abort_flag || global_ns() - t0 > p.wait_ns) break;
        }
        ring_id[sl] = dyn_base + atomicAdd(p.work_ctr, 1);
        __threadfence_block();
        ring_tag[sl] = k2;
    };

    WarpUnit cur, nxt;
    int64_t u = unit_id(0);
    if (u >= total) {
        grid_dep_wait();
        return;
    }
    load_any(u, cur);
    int64_t u_nxt = unit_id(1);
    bool have_nxt = u_nxt < total;
    if (have_nxt) load_any(u_nxt, nxt);

    // table entry of logical block j of a unit (the first 32 come from registers);
    // a group-rows unit's items past its shared blocks are its members' tail blocks
    auto phys_of = [&](const WarpUnit &w, int j) {
        const int v = __shfl_sync(kFull, w.tab, j & 31);
        if constexpr (kRows) {
            if (j >= w.nsh) {
                const int m = (j - w.nsh) / kTailBlocks, i = (j - w.nsh) % kTailBlocks;
                const int Lm = __shfl_sync(kFull, w.mlen, m & 31);
                if (i >= (Lm + kBlockSize - 1) / kBlockSize - w.nsh) return kEmptyItem;
                return __ldg(p.tables + (int64_t)(w.un.s + m) * p.max_blocks + w.nsh + i);
            }
        }
        return j < 32 ? v : __ldg(w.trow + j);
    };
    // normalise a cursor (iu: 0 = cur, 1 = nxt) onto an existing item, skipping
    // `steps` items; false when it runs past the next unit
    auto walk = [&](int &iu, int &ij, int steps) {
        for (;;) {
            if (iu > 1 || (iu == 1 && !have_nxt)) return false;
            const WarpUnit &w = iu ? nxt : cur;
            if (ij >= w.nb) {
                ++iu;
                ij = warp;
                continue;
            }
            if (steps == 0) return true;
            ij += kWarps;
            --steps;
        }
    };
    int iss_u = 0, iss_j = warp;  // next item to fetch
    int n_iss = 0, n_cmp = 0;     // items fetched / computed so far
    uint32_t okmask = 0;          // per stage: block id was valid
    auto fetch_one = [&]() {
        if (!walk(iss_u, iss_j, 0)) return false;
        const WarpUnit &w = iss_u ? nxt : cur;
        const int stage = n_iss % NS;
        const int blk = phys_of(w, iss_j);
        const bool ok = blk >= 0 && blk < p.num_blocks;
        if (ok) issue_slabs<T, D, G>(p, wring_s + stage * Lay::kStageBytes, blk, w.un.h, lane);
        else if (lane == 0 && blk != kEmptyItem) flag_error(p.err, PA_DEVERR_BLOCK_ID);
        cp_async_commit();
        okmask = (okmask & ~(1u << stage)) | ((ok ? 1u : 0u) << stage);
        iss_j += kWarps;
        ++n_iss;
        return true;
    };

    WarpUnit prv;            // unit whose merge is still to be finished
    bool dead = false;       // a hand-over wait timed out
    int uc = 0;
    for (;; ++uc) {
        // ---- q operands of this unit (tiny, L2 resident)
        MmaState<D> ms;
        MmaRows<D> mr;
        F32State<D, (G > 8 ? 8 : G)> fs;
        const unsigned char *qg =
            p.q + ((int64_t)cur.un.s * p.num_q_heads + (int64_t)cur.un.h * G) * Lay::kQRowBytes;
        if constexpr (kRows) {
            // row r = 8 n + lane / 4 of column tile n: head h g + r % g of member r / g
            const int g = p.num_q_heads / hkv;
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                const int r = 8 * n + dr;
                const bool rv = r < cur.nrow;
                const unsigned char *qr =
                    p.q + ((int64_t)(cur.un.s + r / g) * p.num_q_heads + (int64_t)cur.un.h * g + r % g) *
                              Lay::kQRowBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int d0 = kk * 16 + 2 * q4;
                    mr.qb[kk][n][0] = rv ? __ldg(reinterpret_cast<const uint32_t *>(qr + d0 * 2)) : 0u;
                    mr.qb[kk][n][1] = rv ? __ldg(reinterpret_cast<const uint32_t *>(qr + (d0 + 8) * 2)) : 0u;
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                mr.m[i] = -INFINITY;
                mr.l[i] = 0.f;
            }
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
                for (int n = 0; n < 2; ++n) mr.o[mt][n][0] = mr.o[mt][n][1] = mr.o[mt][n][2] = mr.o[mt][n][3] = 0.f;
        } else if constexpr (kFp8) {
            // bf16 -> f16 in the k-slot map of mma_block_fp8; clamped to the f16 range
            const bool hv = dr < G;
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int d0 = 32 * q4 + 16 * j + 4 * i;
                    uint2 x = make_uint2(0u, 0u);
                    if (hv) x = __ldg(reinterpret_cast<const uint2 *>(qg + dr * Lay::kQRowBytes + d0 * 2));
                    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&x.x));
                    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&x.y));
                    auto c = [](float v) { return fminf(fmaxf(v, -65504.f), 65504.f); };
                    ms.qb[4 * j + i][0] = pack_f16x2(c(a.x), c(a.y));
                    ms.qb[4 * j + i][1] = pack_f16x2(c(b.x), c(b.y));
                }
            ms.m[0] = ms.m[1] = -INFINITY;
            ms.l[0] = ms.l[1] = 0.f;
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt) ms.o[mt][0] = ms.o[mt][1] = ms.o[mt][2] = ms.o[mt][3] = 0.f;
        } else if constexpr (kMma) {
            const bool hv = dr < G;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int d0 = kk * 16 + 2 * q4;
                ms.qb[kk][0] = hv ? __ldg(reinterpret_cast<const uint32_t *>(qg + dr * Lay::kQRowBytes + d0 * 2)) : 0u;
                ms.qb[kk][1] = hv ? __ldg(reinterpret_cast<const uint32_t *>(qg + dr * Lay::kQRowBytes + (d0 + 8) * 2)) : 0u;
            }
            ms.m[0] = ms.m[1] = -INFINITY;
            ms.l[0] = ms.l[1] = 0.f;
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt) ms.o[mt][0] = ms.o[mt][1] = ms.o[mt][2] = ms.o[mt][3] = 0.f;
        } else {
            using C = F32Cfg<D, G>;
            const int part = lane & 7;
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int i = 0; i < C::kQkChunks; ++i) {
                    const float4 x = __ldg(reinterpret_cast<const float4 *>(qg + h * C::kRowBytes + (part + 8 * i) * 16));
                    fs.qreg[h][2 * i] = make_float2(x.x * p.scale_log2, x.y * p.scale_log2);
                    fs.qreg[h][2 * i + 1] = make_float2(x.z * p.scale_log2, x.w * p.scale_log2);
                }
            fs.m = -INFINITY;
            fs.l = 0.f;
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int k = 0; k < C::kPvPairs; ++k) fs.acc[h][k] = make_float2(0.f, 0.f);
        }

        // ---- this warp's blocks of the unit, up to NS fetched ahead (fp8: two
        // blocks per step, the pair's stages both landed before it is computed)
        if constexpr (kFp8 && !kRows) {
            static_assert(NS >= 2, "paired fp8 blocks need two stages");
            for (int j = warp; j < cur.nb; j += 2 * kWarps) {
                const bool two = j + kWarps < cur.nb;
                while (n_iss - n_cmp < NS && fetch_one()) {
                }
                cp_async_wait_dyn(n_iss - n_cmp - (two ? 2 : 1));
                __syncwarp();
                const int s0 = n_cmp % NS, s1 = (n_cmp + 1) % NS;
                const bool ok0 = (okmask >> s0) & 1u, ok1 = two && ((okmask >> s1) & 1u);
                const int nt0 = ok0 ? min(kBlockSize, cur.nt - j * kBlockSize) : 0;
                if (two) {
                    if (ok0 || ok1) {
                        unsigned char *const kb2[2] = {wring + s0 * Lay::kStageBytes, wring + s1 * Lay::kStageBytes};
                        const int n2[2] = {nt0, ok1 ? min(kBlockSize, cur.nt - (j + kWarps) * kBlockSize) : 0};
                        mma_tiles_fp8<D, 2>(kb2, n2, ms, p.scale_log2, lane);
                    }
                } else if (ok0) {
                    unsigned char *const kb1[1] = {wring + s0 * Lay::kStageBytes};
                    const int n1[1] = {nt0};
                    mma_tiles_fp8<D, 1>(kb1, n1, ms, p.scale_log2, lane);
                }
                __syncwarp();  // the stages may be refilled by the next fetch
                n_cmp += two ? 2 : 1;
            }
        } else
        for (int j = warp; j < cur.nb; j += kWarps) {
            while (n_iss - n_cmp < NS && fetch_one()) {
            }
            cp_async_wait_dyn(n_iss - n_cmp - 1);
            __syncwarp();
            const int stage = n_cmp % NS;
            if ((okmask >> stage) & 1u) {
                int ntok = min(kBlockSize, cur.nt - j * kBlockSize);
                if constexpr (kRows) {
                    // a tail block counts for its member's g rows only
                    int c_lo = 0, c_hi = kRowTile;
                    if (j >= cur.nsh) {
                        const int m = (j - cur.nsh) / kTailBlocks, i = (j - cur.nsh) % kTailBlocks;
                        const int Lm = __shfl_sync(kFull, cur.mlen, m & 31);
                        const int g = p.num_q_heads / hkv;
                        ntok = min(kBlockSize, Lm - (cur.nsh + i) * kBlockSize);
                        c_lo = m * g;
                        c_hi = c_lo + g;
                    }
                    mma_block_rows<D>(wring_s + stage * Lay::kStageBytes,
                                      wring + stage * Lay::kStageBytes + Lay::kSlabBytes, ntok, c_lo, c_hi, mr,
                                      p.scale_log2, lane);
                }
                else if constexpr (kMma)
                    mma_block<D>(wring_s + stage * Lay::kStageBytes,
                                 wring + stage * Lay::kStageBytes + Lay::kSlabBytes, ntok, ms,
                                 p.scale_log2, lane);
                else
                    f32_block<D, G>(wring + stage * Lay::kStageBytes,
                                    wring + stage * Lay::kStageBytes + Lay::kSlabBytes, ntok, fs, pw, lane);
            }
            __syncwarp();  // the stage may be refilled by the next fetch
            ++n_cmp;
        }
        // keep the pipeline full across the merge
        while (n_iss - n_cmp < NS && fetch_one()) {
        }
        claim_ahead(uc);

        if constexpr (kRows) {
            // ---- one merge slot: this warp's state goes in once every warp has
            // finished its share of the previous unit's merge; then all warps meet
            // and each merges its share of this unit
            if (uc >= 1 && !mbar_wait_bounded(&mfreed[0], (uc - 1) & 1, abort_flag, p.err, p.wait_ns)) {
                dead = true;
                break;
            }
            float *wacc = macc + (size_t)warp * kRowTile * D;
            float2 *wml = mml + (size_t)warp * kRowTile;
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int d = mt * 16 + dr + 8 * half;  // accumulator row dr + 8 half of tile mt
#pragma unroll
                    for (int n = 0; n < 2; ++n) {
                        wacc[(8 * n + 2 * q4) * D + d] = mr.o[mt][n][2 * half];
                        wacc[(8 * n + 2 * q4 + 1) * D + d] = mr.o[mt][n][2 * half + 1];
                    }
                }
            if (dr == 0) {
#pragma unroll
                for (int n = 0; n < 2; ++n) {
                    wml[8 * n + 2 * q4] = make_float2(mr.m[2 * n], mr.l[2 * n]);
                    wml[8 * n + 2 * q4 + 1] = make_float2(mr.m[2 * n + 1], mr.l[2 * n + 1]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&mfull[0]);
            if (!mbar_wait_bounded(&mfull[0], uc & 1, abort_flag, p.err, p.wait_ns)) {
                dead = true;
                break;
            }
            finish_unit_rows<T, D>(p, cur, macc, mml);
            __syncwarp();
            if (lane == 0) mbar_arrive(&mfreed[0]);
        } else {
        // ---- this warp's state into merge slot uc & 1, once the slot's previous
        // unit (uc - 2) has been merged by every warp
        const int b = uc & 1;
        if (uc >= 2 && !mbar_wait_bounded(&mfreed[b], ((uc - 2) >> 1) & 1, abort_flag, p.err, p.wait_ns)) {
            dead = true;
            break;
        }
        float *wacc = macc + ((size_t)b * kWarps + warp) * G * D;
        float2 *wml = mml + ((size_t)b * kWarps + warp) * G;
        if constexpr (kMma) {
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    // accumulator row dr + 8 half of tile mt (fp8: the dim map of mma_block_fp8)
                    const int d = kFp8 ? 16 * dr + 2 * mt + half : mt * 16 + dr + 8 * half;
                    if (2 * q4 < G) wacc[(2 * q4) * D + d] = ms.o[mt][2 * half];
                    if (2 * q4 + 1 < G) wacc[(2 * q4 + 1) * D + d] = ms.o[mt][2 * half + 1];
                }
            if (dr == 0) {
                if (2 * q4 < G) wml[2 * q4] = make_float2(ms.m[0], ms.l[0]);
                if (2 * q4 + 1 < G) wml[2 * q4 + 1] = make_float2(ms.m[1], ms.l[1]);
            }
        } else {
            using C = F32Cfg<D, G>;
            const int tq = lane >> 3, part = lane & 7;
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int k = 0; k < C::kPvPairs; ++k)
                    *reinterpret_cast<float2 *>(wacc + h * D + lane * C::kDpl + 2 * k) = fs.acc[h][k];
            if (tq == 0 && (part & C::kDupMask) == 0) wml[part >> (3 - C::kLogG)] = make_float2(fs.m, fs.l);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&mfull[b]);
        // ---- this warp's share of the previous unit's merge (its states are
        // all in by now unless a warp is a whole unit behind)
        if (uc >= 1) {
            const int pb = b ^ 1;
            if (!mbar_wait_bounded(&mfull[pb], ((uc - 1) >> 1) & 1, abort_flag, p.err, p.wait_ns)) {
                dead = true;
                break;
            }
            finish_unit<T, D, G>(p, prv, macc + (size_t)pb * kWarps * G * D, mml + (size_t)pb * kWarps * G);
            __syncwarp();
            if (lane == 0) mbar_arrive(&mfreed[pb]);
        }
        }
        prv = cur;

        // ---- advance: the fetch cursor moves down one unit with the window
        if (!have_nxt) break;
        walk(iss_u, iss_j, 0);
        cur = nxt;
        iss_u = iss_u > 0 ? iss_u - 1 : 0;
        u_nxt = unit_id(uc + 2);
        have_nxt = u_nxt < total;
        if (have_nxt) load_any(u_nxt, nxt);
    }
    // the last unit's merge (group-rows mode: done in the loop)
    if (!kRows && !dead && mbar_wait_bounded(&mfull[uc & 1], (uc >> 1) & 1, abort_flag, p.err, p.wait_ns))
        finish_unit<T, D, G>(p, prv, macc + (size_t)(uc & 1) * kWarps * G * D, mml + (size_t)(uc & 1) * kWarps * G);
    cp_async_wait<0>();
    grid_dep_wait();
}

// ------------------------------------------------------------- shared prefixes
// Sequences next to each other in the batch whose tables start with the same
// physical blocks (forks, a shared system prompt: chenxutan 2.1 / 3.3, devpress
// 关键设计二) read those blocks once: the shared leading full blocks are computed
// by group units (group, kv head) whose query rows are members x heads and whose
// keys are all the group's shared tokens, and the per-sequence units start after
// them.  The result is the same sum -- the group partial lands in slot 0 of
// every member, the per-sequence units in the slots after it, and the LSE
// reduce combines them.
//
// Detection (block 0 of group_detect_kernel): each sequence's count of leading
// full blocks shared with its predecessor, then the cut of the batch into
// groups.  The group units -- a dense (members x g) x shared tokens x head_dim
// attention each -- run on the tcgen05 tile kernel of prefill.cu
// (launch_group_tiles).

constexpr int kDetectThreads = 1024;
constexpr int kLcpBlocksMax = 64;  // detection blocks that compare tables (flags in the workspace)

// A 64-bit value unique to each call of this process (the high half drawn from
// the clock once per process), so that detection flags left in a reused
// workspace by an earlier call -- or by another process -- never match.
unsigned long long next_epoch() {
    static std::atomic<unsigned long long> ctr{
        (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count() << 20};
    unsigned long long e = ++ctr;
    return e == 0 ? ++ctr : e;
}
constexpr int kMaxGroupSeqs = 4096;  // == kMaxSplitSeqs
constexpr int kMaxGroupBlocks = (1 << 21) - 1;  // fits info's packing (nb << 10)
// Groups of fewer members do not pay for the group unit's fixed cost (its rows
// pad a 128-row tensor-core tile).
constexpr int kMinGroupMembers = 4;
constexpr int kLcpBatch = 8;         // sequences a warp compares at once

// lcp[s] = leading entries of s's table equal to those of s-1, counted over the
// blocks both contexts fill completely (0 for s = 0).  A warp takes kLcpBatch
// sequences at a time and compares 64 entries of each per round.
__device__ __forceinline__ void shared_prefix_lengths(const Params &p, int *lcp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int S = p.num_seqs;
    for (int base = warp * kLcpBatch; base < S; base += (kDetectThreads / 32) * kLcpBatch) {
        int n[kLcpBatch], res[kLcpBatch], la[kLcpBatch], lb[kLcpBatch];
        int va[kLcpBatch][2], vb[kLcpBatch][2];
        // the first 64 entries of both tables are loaded together with the
        // lengths (not behind them): one memory round trip for most pairs
#pragma unroll
        for (int b = 0; b < kLcpBatch; ++b) {
            const int s = base + b;
            const bool pair = s > 0 && s < S;
            la[b] = pair ? __ldg(p.lens + s) : 0;
            lb[b] = pair ? __ldg(p.lens + s - 1) : 0;
            const int32_t *ta = p.tables + (int64_t)s * p.max_blocks;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int i = 32 * k + lane;
                const bool act = pair && i < p.max_blocks;
                va[b][k] = act ? __ldg(ta + i) : 0;
                vb[b][k] = act ? __ldg(ta - p.max_blocks + i) : 0;
            }
        }
#pragma unroll
        for (int b = 0; b < kLcpBatch; ++b) {
            const int La = check_len(p, la[b]), Lb = check_len(p, lb[b]);
            n[b] = (base + b > 0 && base + b < S) ? min(max(La, 0), max(Lb, 0)) / kBlockSize : 0;
            res[b] = n[b];  // == n: no difference found yet
        }
        for (int c0 = 0;; c0 += 64) {
            if (c0 > 0) {
#pragma unroll
                for (int b = 0; b < kLcpBatch; ++b) {
                    const int32_t *ta = p.tables + (int64_t)(base + b) * p.max_blocks;
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const int i = c0 + 32 * k + lane;
                        const bool act = res[b] == n[b] && i < n[b];  // implies 0 < s < S
                        va[b][k] = act ? __ldg(ta + i) : 0;
                        vb[b][k] = act ? __ldg(ta - p.max_blocks + i) : 0;
                    }
                }
            }
            bool more = false;
#pragma unroll
            for (int b = 0; b < kLcpBatch; ++b) {
                if (res[b] != n[b] || c0 >= n[b]) continue;  // warp-uniform
                int mis = n[b];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int i = c0 + 32 * k + lane;
                    if (i < n[b] && va[b][k] != vb[b][k]) mis = min(mis, i);
                }
                mis = __reduce_min_sync(kFull, mis);
                if (mis < n[b]) res[b] = mis;
                else more = more || c0 + 64 < n[b];
            }
            if (!more) break;
        }
#pragma unroll
        for (int b = 0; b < kLcpBatch; ++b)
            if (lane == 0 && base + b < S) lcp[base + b] = res[b];
    }
}

// lcp of the pair (s - 1, s) (s > 0) by one warp: leading entries of s's table
// equal to those of s - 1, over the blocks both contexts fill completely.  Rounds
// of 256 entries (8 loads per lane and table); the first round's loads go out
// together with the lengths'.
__device__ __forceinline__ int pair_lcp(const Params &p, int s, int lane) {
    const int32_t *ta = p.tables + (int64_t)s * p.max_blocks;
    const int32_t *tb = ta - p.max_blocks;
    const int la = __ldg(p.lens + s), lb = __ldg(p.lens + s - 1);
    int va[8], vb[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int i = 32 * k + lane;
        va[k] = i < p.max_blocks ? __ldg(ta + i) : 0;
        vb[k] = i < p.max_blocks ? __ldg(tb + i) : 0;
    }
    const int La = check_len(p, la), Lb = check_len(p, lb);
    const int n = min(max(La, 0), max(Lb, 0)) / kBlockSize;
    for (int c0 = 0;; c0 += 256) {
        if (c0 > 0) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int i = c0 + 32 * k + lane;
                va[k] = i < n ? __ldg(ta + i) : 0;
                vb[k] = i < n ? __ldg(tb + i) : 0;
            }
        }
        int mis = n;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int i = c0 + 32 * k + lane;
            if (i < n && va[k] != vb[k]) mis = min(mis, i);
        }
        mis = __reduce_min_sync(kFull, mis);
        if (mis < n || c0 + 256 >= n) return mis;
    }
}

// Warp-wide exclusive scan (sum, or max when kMax) of one int per lane.
template <bool kMax>
__device__ __forceinline__ int warp_exclusive_scan(int x, int identity) {
    const int lane = threadIdx.x & 31;
    int inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, inc, o);
        if (lane >= o) inc = kMax ? max(inc, y) : inc + y;
    }
    const int exc = __shfl_up_sync(kFull, inc, 1);
    return lane == 0 ? identity : exc;
}

// Detection.  lcp[s] = leading full blocks of s's table equal to those of s - 1
// (compared by blocks 1.. of the grid for more than 64 sequences, else by block
// 0); then block 0 forms the groups block-parallel.  A run is a maximal stretch of
// sequences each sharing at least part_tokens tokens of full blocks with its
// predecessor.  With row groups, a run of n sequences with n x g <= 16 query rows
// stays whole; other runs are cut into chunks of max_members (128 / g) sequences
// counted from their start.  A chunk shares its nb = min(lcp over its members
// after the first) leading blocks; it becomes a row group when 2 <= n and
// n x g <= 16 (one group-rows unit per kv head, on decode_kernel<T, D, kRowTile>),
// else a tile group when n >= kMinGroupMembers (one tcgen05 tile unit per kv head);
// each unit covers the 16 nb shared tokens, a row group's unit also its members'
// private tails when none is longer than kTailBlocks.  first_t[s] = 16 nb of s's
// group, or s's length with kDoneBit for a row group with tails (0 outside one).
// The one-call step's cache write, done by blocks 1.. of the detection grid.
struct StepWriteArgs {
    const uint4 *key;
    const uint4 *value;
    const int64_t *slot_mapping;
    int32_t num_tokens;
    uint4 *key_cache;
    uint4 *value_cache;
    int32_t num_kv_heads;
    int32_t chunks_per_row;
    int64_t num_slots;
    int64_t chunks;  // num_tokens * num_kv_heads * chunks_per_row (0: no write)
};

__global__ void __launch_bounds__(kDetectThreads) group_detect_kernel(const __grid_constant__ Params p,
                                                                      int32_t *first_t, int4 *groups,
                                                                      int32_t *meta,
                                                                      const __grid_constant__ StepWriteArgs w) {
    __shared__ int lcp[kMaxGroupSeqs];
    __shared__ int info[kMaxGroupSeqs];  // at a chunk head: its size, then nb << 10 |
                                         // tails << 9 | row group << 8 | size (size <= 128)
    // Launched with programmatic serialization: this grid may start while the
    // kernel before it in the stream (the previous call's combine, say) is still
    // running.  Until grid_dep_wait() it only reads the block tables and lengths
    // (inputs no kernel of this library writes) and works in shared memory (the
    // whole grouping); every global write comes after it.
    grid_dep_launch();  // the group tiles set up while this runs, then wait for it
    if (blockIdx.x > 0) {
        if ((int)blockIdx.x <= p.lcp_blocks) {
            // this block's slice of the table comparison, one pair per warp
            const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
            const int per = (p.num_seqs + p.lcp_blocks - 1) / p.lcp_blocks;
            const int b0 = ((int)blockIdx.x - 1) * per, b1 = min(p.num_seqs, b0 + per);
            for (int s = b0 + warp; s < b1; s += kDetectThreads / 32) {
                const int v = s > 0 ? pair_lcp(p, s, lane) : 0;
                if (lane == 0) p.lcp_g[s] = v;
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                __threadfence();
                *reinterpret_cast<volatile unsigned long long *>(p.lflags + blockIdx.x - 1) = p.epoch;
            }
        }
        // the step's new K/V (pa_append_decode): the tiles and the decode wait for
        // this whole grid, so they see it; detection reads no cache bytes
        grid_dep_wait();
        for (int64_t i = (int64_t)(blockIdx.x - 1) * kDetectThreads + threadIdx.x; i < w.chunks;
             i += (int64_t)(gridDim.x - 1) * kDetectThreads)
            write_chunk(i, w.key, w.value, w.slot_mapping, w.num_tokens, w.key_cache, w.value_cache,
                        w.num_kv_heads, w.chunks_per_row, w.num_slots, p.err);
        return;
    }
    const int S = p.num_seqs;
    __shared__ int lcp_ok;  // 0: the wait for the other blocks' comparisons ran out
    if (threadIdx.x == 0) lcp_ok = 1;
    if (p.lcp_blocks > 0) {
        // the other blocks compare the tables; wait (bounded) for their flags.  On a
        // timeout no sequence is grouped (lcp 0): slower, the same result.
        __syncthreads();
        if ((int)threadIdx.x < p.lcp_blocks) {
            const volatile unsigned long long *f =
                reinterpret_cast<const volatile unsigned long long *>(p.lflags + threadIdx.x);
            const unsigned long long t0 = global_ns();
            while (*f != p.epoch) {
                if (global_ns() - t0 > p.wait_ns) {
                    lcp_ok = 0;
                    break;
                }
            }
        }
        __syncthreads();
        __threadfence();
        for (int s = threadIdx.x; s < S; s += kDetectThreads) lcp[s] = lcp_ok ? __ldcg(p.lcp_g + s) : 0;
    } else {
        shared_prefix_lengths(p, lcp);
    }
    __syncthreads();
    // Every thread owns a contiguous run of at most 4 sequences [s0, s1).
    __shared__ int wtot[kDetectThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int bpp = p.part_tokens / kBlockSize;
    const int M = p.max_members;  // 128 / g: a power of two
    const int per = (S + kDetectThreads - 1) / kDetectThreads;
    const int s0 = min(S, (int)threadIdx.x * per), s1 = min(S, s0 + per);
    // this thread's context lengths, loaded now for the work estimate at the end
    // (their latency hides behind the grouping's scans)
    int len_of[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) len_of[i] = s0 + i < s1 ? __ldg(p.lens + s0 + i) : 0;
    // block-wide exclusive scan of one value per thread (sum, or max when kMax)
    auto block_scan = [&](int x, int identity, bool is_max) -> int {
        const int wex = is_max ? warp_exclusive_scan<true>(x, identity) : warp_exclusive_scan<false>(x, identity);
        const int winc = is_max ? max(wex, x) : wex + x;
        if (lane == 31) wtot[warp] = winc;
        __syncthreads();
        if (warp == 0) {
            const int v = wtot[lane];
            const int e = is_max ? warp_exclusive_scan<true>(v, identity) : warp_exclusive_scan<false>(v, identity);
            __syncwarp();
            wtot[lane] = e;
        }
        __syncthreads();
        const int r = is_max ? max(wtot[warp], wex) : wtot[warp] + wex;
        __syncthreads();  // wtot is reused by the next scan
        return r;
    };
    // run starts (a sequence sharing fewer than part_tokens tokens of full blocks
    // with its predecessor), then each sequence's run start rs by a max-scan
    int mx = -1;
    for (int s = s0; s < s1; ++s)
        if (s == 0 || lcp[s] < bpp) mx = s;
    int rs = block_scan(mx, -1, true);
    // With row groups, a run of at most K = kRowTile / g sequences (its rows fit
    // one group-rows unit) stays whole: its next run start lies within K after its
    // start.  Other runs are cut, from their start, into chunks of M.
    const int g = p.num_q_heads / p.num_kv_heads;
    const int K = kRowTile / g;
    int head_of[4];
    int short_rs = -1, short_ok = 0;  // the last run start tested, and its result
    for (int s = s0; s < s1; ++s) {
        if (s == 0 || lcp[s] < bpp) rs = s;
        if (p.row_groups && rs != short_rs) {
            short_rs = rs;
            short_ok = rs + K >= S;
            for (int k = 1; k <= K && !short_ok; ++k) short_ok = lcp[rs + k] < bpp;
        }
        head_of[s - s0] = short_ok ? rs : rs + ((s - rs) & ~(M - 1));
    }
    __syncthreads();  // every lcp read; heads' entries are reset below
    // chunk heads collect their size and the smallest shared length of the
    // members after them (a head's own lcp is no longer needed)
    for (int s = s0; s < s1; ++s)
        if (head_of[s - s0] == s) {
            info[s] = 0;
            lcp[s] = INT_MAX;
        }
    __syncthreads();
    for (int s = s0; s < s1; ++s) {
        const int hd = head_of[s - s0];
        atomicAdd(&info[hd], 1);
        if (hd != s) atomicMin(&lcp[hd], lcp[s]);
    }
    __syncthreads();
    // a chunk of n members is a row group when n x g <= kRowTile (n >= 2), else a
    // tile group when n >= kMinGroupMembers.  A row group whose members' private
    // tails (blocks past the shared ones) are all at most kTailBlocks long takes
    // the tails too (its unit masks each tail block to its member's rows), so its
    // members need no per-sequence unit.  info = nb << 10 | tails << 9 | row << 8 | n
    int nt_heads = 0, nr_heads = 0;  // this thread's tile / row groups
    for (int s = s0; s < s1; ++s) {
        if (head_of[s - s0] != s) continue;
        const int n = info[s], mn = lcp[s];
        const bool row = p.row_groups && n >= 2 && n * g <= kRowTile;
        const bool tile = !row && n >= kMinGroupMembers;
        const int nb = (row || tile) && mn >= bpp ? min(mn, kMaxGroupBlocks) : 0;
        bool tails = false;
        if (row && nb > 0) {
            int tmax = 0;
            for (int k = 0; k < n; ++k) {
                const int L = max(checked_len(p, s + k), 0);
                tmax = max(tmax, (L + kBlockSize - 1) / kBlockSize - nb);
            }
            tails = tmax <= kTailBlocks;
            for (int k = 0; k < n && tails; ++k) tails = checked_len(p, s + k) < kDoneBit;
        }
        info[s] = (nb << 10) | ((tails ? 1 : 0) << 9) | ((row ? 1 : 0) << 8) | n;
        if (nb > 0) {
            if (row) ++nr_heads;
            else ++nt_heads;
        }
    }
    // both counts in one scan (each total <= 4096 fits 16 bits)
    __shared__ int tot_groups;
    const int mine = nt_heads + (nr_heads << 16);
    const int ex = block_scan(mine, 0, false);  // (the scan's barriers publish info)
    if (threadIdx.x == kDetectThreads - 1) tot_groups = ex + mine;
    // work estimate in (token, kv head) units: group keys (measured on B200 to
    // cost about 1.5 times a per-sequence key: a tile group's rows pad a 128-row
    // tensor-core tile, a row group's 16 rows double the tiles of a block) against
    // the per-sequence kernel's keys
    __shared__ unsigned long long work[3];
    if (threadIdx.x == 0) work[0] = work[1] = work[2] = 0ull;
    __syncthreads();
    const int n_tile = tot_groups & 0xffff, n_row = tot_groups >> 16;
    // Everything so far ran in shared memory and registers.  The previous kernel
    // must be complete before this grid writes anything; behind a cache write
    // (pa_decode after pa_cache_write) this also means that this kernel finishes
    // only after the write, and the group tiles, which wait for this kernel, see
    // the new tokens' K/V.
    grid_dep_wait();
    if (threadIdx.x == 0 && !lcp_ok) flag_error(p.err, PA_DEVERR_TIMEOUT);
    unsigned long long tw = 0, rw = 0, dw = 0;
    for (int s = s0; s < s1; ++s) {
        const int inf = info[head_of[s - s0]];
        const int L = max(check_len(p, len_of[s - s0]), 0);
        const int fs = (inf >> 10) * kBlockSize;                // shared tokens
        const int ft = ((inf >> 9) & 1) ? max(L, fs) : fs;      // tails: all of it
        first_t[s] = ((inf >> 9) & 1) ? (ft | kDoneBit) : ft;
        dw += (unsigned long long)max(0, L - ft);
        if ((inf >> 8) & 1) rw += (unsigned long long)(max(0, ft - fs) + (head_of[s - s0] == s ? fs : 0));
        else if (head_of[s - s0] == s) tw += (unsigned long long)fs;
    }
    // one shared-memory atomic per warp (1,024 on one word would serialise)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        tw += __shfl_xor_sync(kFull, tw, o);
        rw += __shfl_xor_sync(kFull, rw, o);
        dw += __shfl_xor_sync(kFull, dw, o);
    }
    if (lane == 0) {
        atomicAdd(&work[0], tw);
        atomicAdd(&work[1], rw);
        atomicAdd(&work[2], dw);
    }
    // records: tile groups first (the tile kernel reads groups[0, n_tile)), in
    // sequence order; then the row groups, longest first by buckets of 8 shared
    // blocks (the group-rows kernel draws its units in record order, so the
    // longest start first and the short ones even out the end; the order within a
    // bucket does not affect any result)
    constexpr int kBuckets = 32;
    __shared__ int rcount[kBuckets], rbase[kBuckets];
    auto bucket = [](int nb) { return kBuckets - 1 - min(kBuckets - 1, nb >> 3); };  // 0: longest
    if (n_row > 0) {  // (uniform)
        if (threadIdx.x < kBuckets) rcount[threadIdx.x] = 0;
        __syncthreads();
        for (int s = s0; s < s1; ++s)
            if (head_of[s - s0] == s && ((info[s] >> 8) & 1) && (info[s] >> 10) > 0)
                atomicAdd(&rcount[bucket(info[s] >> 10)], 1);
        __syncthreads();
        if (threadIdx.x == 0) {
            int run = n_tile;
#pragma unroll
            for (int b = 0; b < kBuckets; ++b) {
                rbase[b] = run;
                run += rcount[b];
                rcount[b] = 0;
            }
        }
        __syncthreads();
    }
    int gt = ex & 0xffff;
    for (int s = s0; s < s1; ++s) {
        if (head_of[s - s0] != s) continue;
        const int inf = info[s];
        const int n = inf & 255, nb = inf >> 10;
        if (nb == 0) continue;
        if ((inf >> 8) & 1) {  // row groups: the fourth field says whether the unit takes the tails
            const int b = bucket(nb);
            groups[rbase[b] + atomicAdd(&rcount[b], 1)] = make_int4(s, n, nb * kBlockSize, (inf >> 9) & 1);
        } else {
            groups[gt] = make_int4(s, n, nb * kBlockSize, gt * p.num_kv_heads);
            ++gt;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        meta[0] = n_tile;
        meta[1] = n_tile * p.num_kv_heads;
        meta[2] = 0;   // the per-sequence kernel's work counter
        meta[3] = 0;   // the group tiles' work counter
        meta[5] = n_row;
        meta[6] = 0;   // the group-rows kernel's work counter
        // SMs for the group tiles and the group rows, in proportion to their
        // shares of the work (the per-sequence kernel takes the rest), so that the
        // kernels end together; the tiles get at least one SM per 2 units (up to
        // half the SMs), since a short tile unit's time is mostly latency.  A
        // group-rows key costs about 1.7 per-sequence keys (measured on B200), and
        // each of its units about 64 more for the meeting and merge at its end.
        const double t = 1.5 * (double)work[0];
        const double r = 1.7 * (double)work[1] + 64.0 * n_row * p.num_kv_heads;
        const double d = (double)work[2];
        const double all = t + r + d + 1.0;
        const int sms = max(1, p.num_sms);
        int want_t = (int)ceil(sms * t / all);
        want_t = max(want_t, min(sms / 2, (n_tile * p.num_kv_heads + 1) / 2));
        want_t = n_tile == 0 ? 0 : min(sms, max(1, want_t));
        int want_r = n_row == 0 ? 0 : max(1, (int)ceil(sms * r / all));
        want_r = min(want_r, max(n_row == 0 ? 0 : 1, sms - want_t));
        meta[4] = want_t;
        meta[7] = want_r;
    }
}

// Combine split-K partials: one warp per (sequence, query head) with more than
// one partition.  M = max_p m_p; out = sum_p 2^(m_p-M) acc_p / sum_p 2^(m_p-M) l_p.
// The first kPre slots are loaded together with the length that says how many
// slots there are (slots past it are ignored), so most rows take one memory
// round trip after the decode ends.
template <typename T, int D>
__global__ void __launch_bounds__(128) reduce_kernel(const __grid_constant__ Params p) {
    grid_dep_launch();  // the next call's detection may start reading its tables
    grid_dep_wait();    // every partial is written
    constexpr int kDpl = D / 32;
    constexpr int kPre = 4;
    const int lane = threadIdx.x & 31;
    const int64_t wid = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (wid >= (int64_t)p.num_seqs * p.num_q_heads) return;
    const int s = (int)(wid / p.num_q_heads);
    const float2 *ml = p.ws_ml + wid * p.max_parts;
    const float *acc = p.ws_acc + wid * p.max_parts * D + lane * kDpl;
    float2 mlp[kPre];
    float ap[kPre][kDpl];
#pragma unroll
    for (int i = 0; i < kPre; ++i) {
        const bool in = i < p.max_parts;  // inside the workspace row (maybe unwritten)
        mlp[i] = in ? ml[i] : make_float2(-INFINITY, 0.f);
#pragma unroll
        for (int k = 0; k < kDpl; ++k) ap[i][k] = 0.f;
        if (in) {
            if constexpr (kDpl == 4) {
                const float4 a = *reinterpret_cast<const float4 *>(acc + (int64_t)i * D);
                ap[i][0] = a.x; ap[i][1] = a.y; ap[i][2] = a.z; ap[i][3] = a.w;
            } else {
                const float2 a = *reinterpret_cast<const float2 *>(acc + (int64_t)i * D);
                ap[i][0] = a.x; ap[i][1] = a.y;
            }
        }
    }
    int L = checked_len(p, s);
    if (L < 0) L = 0;
    const int ftr = p.first_t ? __ldg(p.first_t + s) : 0;
    if (ftr & kDoneBit) return;                          // written by its group-rows unit
    const int ft = ftr;
    const int n = slot_base(ft) + seq_units(p, L, ft);  // slots written
    if (ft == 0 && n <= 1) return;                       // finished by the decode kernel
    float M = -INFINITY;
#pragma unroll
    for (int i = 0; i < kPre; ++i)
        if (i < n) M = fmaxf(M, mlp[i].x);
    if (n > kPre) {
        float Mr = -INFINITY;
        for (int i = kPre + lane; i < n; i += 32) Mr = fmaxf(Mr, ml[i].x);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) Mr = fmaxf(Mr, __shfl_xor_sync(kFull, Mr, o));
        M = fmaxf(M, Mr);
    }
    float lsum = 0.f, o[kDpl];
#pragma unroll
    for (int k = 0; k < kDpl; ++k) o[k] = 0.f;
#pragma unroll
    for (int i = 0; i < kPre; ++i) {
        if (i >= n) break;
        const float f = fast_exp2(mlp[i].x - M);
        lsum = fmaf(mlp[i].y, f, lsum);
#pragma unroll
        for (int k = 0; k < kDpl; ++k) o[k] = fmaf(ap[i][k], f, o[k]);
    }
#pragma unroll 4
    for (int i = kPre; i < n; ++i) {
        const float2 mi = ml[i];
        const float f = fast_exp2(mi.x - M);
        lsum = fmaf(mi.y, f, lsum);
        if constexpr (kDpl == 4) {
            const float4 a = *reinterpret_cast<const float4 *>(acc + (int64_t)i * D);
            o[0] = fmaf(a.x, f, o[0]); o[1] = fmaf(a.y, f, o[1]);
            o[2] = fmaf(a.z, f, o[2]); o[3] = fmaf(a.w, f, o[3]);
        } else {
            const float2 a = *reinterpret_cast<const float2 *>(acc + (int64_t)i * D);
            o[0] = fmaf(a.x, f, o[0]); o[1] = fmaf(a.y, f, o[1]);
        }
    }
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll
    for (int k = 0; k < kDpl; ++k) store_out<IoT<T>>(p.out, wid * D + lane * kDpl + k, o[k] * inv);
}

template <typename T, int D, int G>
cudaError_t launch_t(const DecodeLaunch &a, Params &prm, cudaStream_t stream) {
    using Lay = Layout<T, D, G>;
    const bool split = prm.part_tokens > 0;
    const size_t smem = Lay::smem_bytes(split ? Lay::kCumArrays * (a.num_seqs + 1) : 0);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static_assert(Lay::smem_bytes(Lay::kCumArrays * (kMaxSplitSeqs + 1)) <= 232448, "decode smem over the sm_100 limit");
    e = cudaFuncSetAttribute(decode_kernel<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Lay::smem_bytes(Lay::kCumArrays * (kMaxSplitSeqs + 1)));
    if (e != cudaSuccess) return e;
    const int sms = num_sms(dev);
    prm.num_sms = sms;
    // Per-sequence units after the group-covered partitions span several
    // partitions, so that the per-unit merge is amortised: 1024 tokens, or 2048
    // when there are few (sequence, kv head) pairs to spread over the SMs
    // (measured on B200: 512-token units cost 4-16% against these).
    if (split) {
        const int want = (int64_t)a.num_seqs * a.cache.num_kv_heads < 4LL * sms ? 2048 : 1024;
        prm.seq_tokens = prm.part_tokens * std::max(1, want / prm.part_tokens);
    }
    // shared-prefix groups: bf16, head_dim 128, split contexts.  Detection, the
    // group tiles, the group rows (g <= 4), this kernel and the combine follow one
    // another with programmatic dependent launch (see the kernels for where each
    // waits).
    bool grouped = false;
    if constexpr (sizeof(T) == 2 && D == 128) {
        if (split && a.ws_group && a.num_seqs <= kMaxGroupSeqs) {
            unsigned char *g = static_cast<unsigned char *>(a.ws_group);
            // group area: first_t[S] (16-byte padded), groups[S], meta
            const size_t sa = ((size_t)a.num_seqs * 4 + 15) / 16 * 16;
            prm.first_t = reinterpret_cast<int32_t *>(g);
            prm.groups = reinterpret_cast<int4 *>(g + sa);
            prm.meta = reinterpret_cast<int32_t *>(const_cast<int4 *>(prm.groups) + a.num_seqs);
            // then lcp_g[S] (16-byte padded) and the comparison blocks' flags (64 x 8 bytes)
            unsigned char *gl_area = reinterpret_cast<unsigned char *>(const_cast<int32_t *>(prm.meta)) + 32;
            prm.lcp_g = reinterpret_cast<int32_t *>(gl_area);
            prm.lflags = reinterpret_cast<unsigned long long *>(gl_area + sa);
            // more than 64 sequences: the comparison is spread over one block per 32
            // sequences (up to kLcpBlocksMax); the epoch makes each call's flags unique
            prm.lcp_blocks = a.num_seqs > 64 ? std::min(kLcpBlocksMax, (a.num_seqs + 31) / 32) : 0;
            prm.epoch = next_epoch();
            // Row groups need 2 <= members <= 16 / g; at g = 8 only pairs qualify,
            // whose gain does not pay for the extra launch, so the group-rows kernel
            // runs for g <= 4 only.
            constexpr bool kRowsLaunch = G <= 4;
            prm.max_members = 128 / G;
            prm.row_groups = kRowsLaunch ? 1 : 0;
            StepWriteArgs wa;
            std::memset(&wa, 0, sizeof(wa));
            unsigned write_blocks = 0;
            if (a.write && a.write->num_tokens > 0) {
                const StepWrite &sw = *a.write;
                wa.key = static_cast<const uint4 *>(sw.key);
                wa.value = static_cast<const uint4 *>(sw.value);
                wa.slot_mapping = sw.slot_mapping;
                wa.num_tokens = sw.num_tokens;
                wa.key_cache = static_cast<uint4 *>(sw.key_cache);
                wa.value_cache = static_cast<uint4 *>(sw.value_cache);
                wa.num_kv_heads = a.cache.num_kv_heads;
                wa.chunks_per_row = a.cache.head_dim * (int)sizeof(T) / 16;
                wa.num_slots = (int64_t)a.cache.num_blocks * kBlockSize;
                wa.chunks = (int64_t)sw.num_tokens * wa.num_kv_heads * wa.chunks_per_row;
                write_blocks = (unsigned)std::min<int64_t>((wa.chunks + kDetectThreads - 1) / kDetectThreads,
                                                           4 * sms);
            }
            // always with programmatic serialization: its table comparison may
            // overlap the end of whatever kernel precedes it (see the kernel)
            e = launch_after(group_detect_kernel, dim3(1 + std::max<unsigned>(write_blocks, (unsigned)prm.lcp_blocks)),
                             dim3(kDetectThreads), 0, stream,
                             static_cast<const Params &>(prm), const_cast<int32_t *>(prm.first_t),
                             const_cast<int4 *>(prm.groups), const_cast<int32_t *>(prm.meta),
                             static_cast<const StepWriteArgs &>(wa));
            if (e != cudaSuccess) return e;
            GroupTileLaunch gl;
            gl.query = a.query;
            gl.num_seqs = a.num_seqs;
            gl.key_cache = a.key_cache;
            gl.value_cache = a.value_cache;
            gl.block_tables = a.block_tables;
            gl.max_blocks_per_seq = a.max_blocks_per_seq;
            gl.groups = prm.groups;
            gl.meta = prm.meta;
            gl.ws_acc = prm.ws_acc;
            gl.ws_ml = prm.ws_ml;
            gl.num_q_heads = a.num_q_heads;
            gl.num_kv_heads = a.cache.num_kv_heads;
            gl.num_blocks = a.cache.num_blocks;
            gl.max_partitions = a.max_partitions;
            gl.scale = a.scale;
            gl.err = a.err;
            // The detection kernel picks how many SMs take the group units (ids drawn
            // from a counter); the tile CTAs beyond that exit at once, and the
            // per-sequence kernel starts on those SMs instead of waiting for them.
            if ((e = launch_group_tiles(gl, sms, stream)) != cudaSuccess) return e;
            // Row groups (members x g <= 16 rows) on the group-rows mode of this
            // kernel, launched behind the tiles the same way: its CTAs beyond the
            // number the detection kernel chose leave at once.
            if constexpr (kRowsLaunch) {
                using LayR = Layout<T, D, kRowTile>;
                static_assert(LayR::smem_bytes(0) <= 232448, "group-rows smem over the sm_100 limit");
                e = cudaFuncSetAttribute(decode_kernel<T, D, kRowTile>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)LayR::smem_bytes(0));
                if (e != cudaSuccess) return e;
                Params rp = prm;
                rp.work_ctr = const_cast<int32_t *>(prm.meta) + 6;
                rp.wait_first = 0;  // the tiles start only after the detection ends
                e = launch_after(decode_kernel<T, D, kRowTile>, dim3((unsigned)sms), dim3(kThreads), LayR::smem_bytes(0),
                                 stream, static_cast<const Params &>(rp));
                if (e != cudaSuccess) return e;
            }
            grouped = true;
            prm.work_ctr = const_cast<int32_t *>(prm.meta) + 2;
        }
    }
    int64_t grid = sms;
    if (!split) grid = std::min<int64_t>(grid, (int64_t)a.num_seqs * a.cache.num_kv_heads);
    if (grid < 1) grid = 1;
    prm.wait_first = (!grouped && a.after_write) ? 1 : 0;
    if (grouped || a.after_write) {
        e = launch_after(decode_kernel<T, D, G>, dim3((unsigned)grid), dim3(kThreads), smem, stream,
                         static_cast<const Params &>(prm));
    } else {
        decode_kernel<T, D, G><<<(unsigned)grid, kThreads, smem, stream>>>(prm);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess || !split) return e;
    const int64_t warps = (int64_t)a.num_seqs * a.num_q_heads;
    return launch_after(reduce_kernel<T, D>, dim3((unsigned)((warps + 3) / 4)), dim3(128), 0, stream,
                        static_cast<const Params &>(prm));
}

template <typename T, int D>
cudaError_t launch_g(const DecodeLaunch &a, Params &prm, cudaStream_t stream) {
    switch (a.num_q_heads / a.cache.num_kv_heads) {
        case 1: return launch_t<T, D, 1>(a, prm, stream);
        case 2: return launch_t<T, D, 2>(a, prm, stream);
        case 4: return launch_t<T, D, 4>(a, prm, stream);
        case 8: return launch_t<T, D, 8>(a, prm, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_append_decode(const StepWrite &w, DecodeLaunch a, cudaStream_t stream) {
    // the shared-prefix path (bf16, head_dim 128, split contexts) starts with the
    // detection kernel, whose grid takes the write along
    const bool grouped = a.cache.dtype == PA_BF16 && a.cache.head_dim == 128 && a.partition_size > 0 &&
                         a.ws_group && a.num_seqs <= kMaxGroupSeqs;
    if (w.num_tokens > 0) {
        if (grouped) {
            a.write = &w;
        } else {
            const cudaError_t e = launch_cache_write(w.key, w.value, w.slot_mapping, w.num_tokens, w.key_cache,
                                                     w.value_cache, a.cache, a.err, stream);
            if (e != cudaSuccess) return e;
            a.after_write = true;  // the decode chain starts behind the write
        }
    }
    return launch_decode(a, stream);
}

cudaError_t launch_decode(const DecodeLaunch &a, cudaStream_t stream) {
    Params prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.q = static_cast<const unsigned char *>(a.query);
    prm.kc = static_cast<const unsigned char *>(a.key_cache);
    prm.vc = static_cast<const unsigned char *>(a.value_cache);
    prm.tables = a.block_tables;
    prm.lens = a.context_lens;
    prm.ws_acc = a.ws_acc;
    prm.ws_ml = a.ws_ml;
    prm.out = a.out;
    prm.err = a.err;
    prm.max_blocks = a.max_blocks_per_seq;
    prm.max_context = a.max_context_len;
    prm.num_seqs = a.num_seqs;
    prm.num_q_heads = a.num_q_heads;
    prm.num_kv_heads = a.cache.num_kv_heads;
    prm.num_blocks = a.cache.num_blocks;
    prm.part_tokens = a.partition_size;
    prm.max_parts = a.max_partitions;
    prm.seq_tokens = a.partition_size;  // launch_t may widen it
    prm.scale_log2 = a.scale * kLog2e;
    prm.v_scale = 1.f;
    prm.wait_ns = wait_limit_ns();
    if (a.cache.dtype == PA_FP8_E4M3) {
        if (a.cache.head_dim != 128) return cudaErrorInvalidValue;
        prm.scale_log2 = a.scale * a.cache.k_scale * kLog2e;
        prm.v_scale = a.cache.v_scale;
        return launch_g<e4m3_t, 128>(a, prm, stream);
    }
    const bool bf16 = a.cache.dtype == PA_BF16;
    if (a.cache.head_dim == 128)
        return bf16 ? launch_g<__nv_bfloat16, 128>(a, prm, stream) : launch_g<float, 128>(a, prm, stream);
    if (a.cache.head_dim == 64)
        return bf16 ? launch_g<__nv_bfloat16, 64>(a, prm, stream) : launch_g<float, 64>(a, prm, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa

