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
//    per unit.  The grid is persistent (one CTA per SM); CTA c takes units
//    c, c + gridDim, ...  Units are ordered "first partition of every sequence,
//    kv head innermost" then "remaining partitions, sequence-major": the first
//    512 tokens of sibling sequences that share prefix blocks are read by CTAs
//    running at the same time, so the shared blocks are served from L2.
//  * Warp 8 is the producer: it reads block-table entries (32 per warp load)
//    and issues 1-D bulk async copies (TMA engine, cp.async.bulk) of each
//    4 KB (block, kv head) slab of K and of V into a ring of shared-memory
//    stages, completion tracked by mbarriers.  No register staging, no
//    address-generation cost on the consumer warps.
//  * Warps 0..7 are consumers.  Consumer w takes logical blocks w, w+8, ... of
//    the unit.  QK: 8 lanes per token (16-byte conflict-free smem reads), packed
//    fp32 FMAs (FFMA2), a transposing shuffle reduction that leaves each lane
//    with one head's score.  Online softmax in fp32 (running max m, running
//    sum l, log2 domain: q is pre-scaled by scale*log2(e)).  PV: each lane owns
//    D/32 output dims of every head, FFMA2 again.  At the end of a unit the 8
//    warps' (m, l, acc) are merged through shared memory.
//  * Split-K (partition_size > 0): a sequence with several partitions writes
//    (m, l, acc) per partition to the workspace and reduce_kernel combines them;
//    single-partition sequences are finished directly.
//  * Every mbarrier wait is bounded (pa_common.cuh); on a timeout the CTA sets
//    an abort flag, stops issuing, drains its in-flight copies and returns.
#include <cfloat>

#include "pa_common.cuh"
#include "pa_launch.h"

namespace pa {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;

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

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }
constexpr int cmin(int a, int b) { return a < b ? a : b; }
constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

template <typename T, int D, int G>
struct Cfg {
    static constexpr int kElem = ElemBytes<T>::value;
    static constexpr int kRowBytes = D * kElem;                 // one token of one head
    static constexpr int kSlabBytes = kBlockSize * kRowBytes;   // one (block, kv head) slab
    static constexpr int kStageBytes = 2 * kSlabBytes;          // K slab + V slab
    static constexpr int kConsumerWarps = 8;
    static constexpr int kThreads = (kConsumerWarps + 1) * 32;
    static constexpr int kStages = cmin(16, (128 * 1024) / kStageBytes);
    // QK: 8 lanes per token; each lane reads kQkChunks 16-byte chunks of a row.
    static constexpr int kQkChunks = kRowBytes / 128;
    static constexpr int kEpc = 16 / kElem;                     // elements per 16-byte chunk
    static constexpr int kQkPairs = kQkChunks * kEpc / 2;       // float2 of q per head per lane
    // PV: each lane owns kDpl consecutive dims of every head.
    static constexpr int kDpl = D / 32;
    static constexpr int kPvPairs = kDpl / 2;
    static constexpr int kPvBytes = kDpl * kElem;
    static constexpr int kLogG = ilog2(G);
    static constexpr int kDupMask = (8 >> kLogG) - 1;           // lanes holding the same score
    static_assert(kRowBytes % 128 == 0, "a row must split into 8 lanes of 16-byte chunks");
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");

    // shared-memory carve-up (byte offsets)
    static constexpr size_t kOffRing = 0;
    static constexpr size_t kOffQ = kOffRing + (size_t)kStages * kStageBytes;
    static constexpr size_t kOffP = align_up(kOffQ + 2ull * G * kRowBytes, 16);
    static constexpr size_t kPWarpFloats = 16 * G + G;          // p[16][G] then alpha[G]
    static constexpr size_t kOffMacc =
        align_up(kOffP + (size_t)kConsumerWarps * kPWarpFloats * 4, 16);
    static constexpr size_t kOffMml = kOffMacc + 2ull * kConsumerWarps * G * D * 4;
    static constexpr size_t kOffBar = align_up(kOffMml + 2ull * kConsumerWarps * G * 8, 8);
    static constexpr size_t kOffSlotOk = kOffBar + (2ull * kStages + 4) * 8;
    static constexpr size_t kOffAbort = kOffSlotOk + (size_t)kStages * 4;
    static constexpr size_t kOffCum = align_up(kOffAbort + 4, 16);
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
    float scale_log2;
};

// Context length of sequence s, or -1 when it is outside [0, max_context] or
// longer than its table.
__device__ __forceinline__ int checked_len(const Params &p, int s) {
    const int L = __ldg(p.lens + s);
    if (L < 0 || L > p.max_context || (int64_t)L > (int64_t)p.max_blocks * kBlockSize) return -1;
    return L;
}

__device__ __forceinline__ int num_parts(const Params &p, int L) {
    if (p.part_tokens <= 0 || L <= 0) return 1;
    return (L + p.part_tokens - 1) / p.part_tokens;
}

struct Unit {
    int s, part, h;
};

// Unit u -> (sequence, partition, kv head).  Units [0, S*Hkv) are partition 0
// of every sequence, kv head innermost; after them come partitions >= 1,
// sequence-major, using cum[s] = sum_{s' < s} (parts(s') - 1).
__device__ __forceinline__ Unit unit_of(int64_t u, int64_t units_first, int hkv, const int *cum,
                                        int S) {
    if (u < units_first) return Unit{(int)(u / hkv), 0, (int)(u % hkv)};
    const int64_t v = u - units_first;
    const int e = (int)(v / hkv), h = (int)(v % hkv);
    int lo = 0, hi = S;  // cum[lo] <= e < cum[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cum[mid] <= e) lo = mid; else hi = mid;
    }
    return Unit{lo, 1 + e - cum[lo], h};
}

// Token range [t0, t0 + nt) of a unit.
__device__ __forceinline__ void unit_range(const Params &p, const Unit &un, int L, int &t0,
                                           int &nt) {
    if (p.part_tokens <= 0) {
        t0 = 0;
        nt = L;
    } else {
        t0 = un.part * p.part_tokens;
        const int t1 = min(L, t0 + p.part_tokens);
        nt = max(0, t1 - t0);
    }
}

template <typename T>
__device__ __forceinline__ void unpack16(const uint4 &r, float2 *f);
template <>
__device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4 &r, float2 *f) {
    f[0] = bf16x2_to_float2(r.x);
    f[1] = bf16x2_to_float2(r.y);
    f[2] = bf16x2_to_float2(r.z);
    f[3] = bf16x2_to_float2(r.w);
}
template <>
__device__ __forceinline__ void unpack16<float>(const uint4 &r, float2 *f) {
    f[0] = make_float2(__uint_as_float(r.x), __uint_as_float(r.y));
    f[1] = make_float2(__uint_as_float(r.z), __uint_as_float(r.w));
}

// Load kBytes (4, 8 or 16) of one row for the PV step and widen to float2 pairs.
template <typename T, int kBytes>
__device__ __forceinline__ void load_pv(const unsigned char *src, float2 *f) {
    if constexpr (kBytes == 16) {
        const uint4 r = *reinterpret_cast<const uint4 *>(src);
        unpack16<T>(r, f);
    } else if constexpr (kBytes == 8) {
        const uint2 r = *reinterpret_cast<const uint2 *>(src);
        if constexpr (sizeof(T) == 2) {
            f[0] = bf16x2_to_float2(r.x);
            f[1] = bf16x2_to_float2(r.y);
        } else {
            f[0] = make_float2(__uint_as_float(r.x), __uint_as_float(r.y));
        }
    } else {
        static_assert(kBytes == 4 && sizeof(T) == 2, "4-byte PV loads are bf16 pairs");
        f[0] = bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(src));
    }
}

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

// One 16-token block for one consumer warp: QK, online-softmax update, PV.
template <typename T, int D, int G>
__device__ __forceinline__ void process_block(const unsigned char *kb, const unsigned char *vb,
                                              int ntok,
                                              const float2 (&qreg)[G][Cfg<T, D, G>::kQkPairs],
                                              float &m, float &l,
                                              float2 (&acc)[G][Cfg<T, D, G>::kPvPairs],
                                              float *pw, int lane) {
    using C = Cfg<T, D, G>;
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
            const uint4 raw =
                *reinterpret_cast<const uint4 *>(kb + t * C::kRowBytes + (part + 8 * i) * 16);
            float2 kv[C::kEpc / 2];
            unpack16<T>(raw, kv);
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int k = 0; k < C::kEpc / 2; ++k)
                    a[h] = ffma2(qreg[h][i * (C::kEpc / 2) + k], kv[k], a[h]);
        }
        float v[G];
#pragma unroll
        for (int h = 0; h < G; ++h) v[h] = a[h].x + a[h].y;
        const float s = reduce8<G, 2>(v, part);
        sc[r] = t < ntok ? s : -INFINITY;
    }
    // online softmax for head hd over the block's 16 tokens
    float bm = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    bm = fmaxf(bm, __shfl_xor_sync(kFull, bm, 8));
    bm = fmaxf(bm, __shfl_xor_sync(kFull, bm, 16));
    const float m_new = fmaxf(m, bm);
    const float alpha = fast_exp2(m - m_new);
    float ps = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        sc[r] = fast_exp2(sc[r] - m_new);
        ps += sc[r];
    }
    ps += __shfl_xor_sync(kFull, ps, 8);
    ps += __shfl_xor_sync(kFull, ps, 16);
    l = l * alpha + ps;
    m = m_new;
    if ((part & C::kDupMask) == 0) {
#pragma unroll
        for (int r = 0; r < 4; ++r) pw[(tq + 4 * r) * G + hd] = sc[r];
        if (tq == 0) pw[16 * G + hd] = alpha;
    }
    __syncwarp();
    // PV
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float al = pw[16 * G + h];
#pragma unroll
        for (int k = 0; k < C::kPvPairs; ++k) {
            acc[h][k].x *= al;
            acc[h][k].y *= al;
        }
    }
    const unsigned char *vrow = vb + lane * C::kPvBytes;
#pragma unroll
    for (int t = 0; t < kBlockSize; ++t) {
        if (t < ntok) {
            float2 vv[C::kPvPairs];
            load_pv<T, C::kPvBytes>(vrow + t * C::kRowBytes, vv);
            float pt[G];
            if constexpr (G >= 4) {
#pragma unroll
                for (int h = 0; h < G; h += 4) {
                    const float4 p4 = *reinterpret_cast<const float4 *>(pw + t * G + h);
                    pt[h] = p4.x; pt[h + 1] = p4.y; pt[h + 2] = p4.z; pt[h + 3] = p4.w;
                }
            } else {
#pragma unroll
                for (int h = 0; h < G; ++h) pt[h] = pw[t * G + h];
            }
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int k = 0; k < C::kPvPairs; ++k)
                    acc[h][k] = ffma2(make_float2(pt[h], pt[h]), vv[k], acc[h][k]);
        }
    }
    __syncwarp();  // pw is rewritten by the next block
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

template <typename T, int D, int G>
__global__ void __launch_bounds__(Cfg<T, D, G>::kThreads, 1) decode_kernel(const Params p) {
    using C = Cfg<T, D, G>;
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *ring = smem + C::kOffRing;
    unsigned char *qbuf = smem + C::kOffQ;
    float *pbuf = reinterpret_cast<float *>(smem + C::kOffP);
    float *macc = reinterpret_cast<float *>(smem + C::kOffMacc);
    float2 *mml = reinterpret_cast<float2 *>(smem + C::kOffMml);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *empty = full + C::kStages;
    uint64_t *qfull = empty + C::kStages;  // [2]
    uint64_t *qempty = qfull + 2;          // [2]
    int *slot_ok = reinterpret_cast<int *>(smem + C::kOffSlotOk);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffAbort);
    int *cum = reinterpret_cast<int *>(smem + C::kOffCum);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.num_seqs, hkv = p.num_kv_heads;
    const bool split = p.part_tokens > 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&qfull[b], 1);
            mbar_init(&qempty[b], C::kConsumerWarps);
        }
        *abort_flag = 0;
        mbar_init_fence();
    }
    // cum[s] = sum_{s' < s} (parts(s') - 1): exclusive scan, one chunk per thread.
    if (split) {
        const int nthr = C::kThreads;
        const int per = (S + nthr - 1) / nthr;
        const int beg = min(S, (int)threadIdx.x * per), end = min(S, beg + per);
        int local = 0;
        for (int s = beg; s < end; ++s) {
            const int L = checked_len(p, s);
            local += num_parts(p, L < 0 ? 0 : L) - 1;
        }
        // scan the per-thread totals: warp inclusive scan, then across warps
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += y;
        }
        int *wsum = reinterpret_cast<int *>(pbuf);  // scratch before pbuf's first use
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        int off = 0;
        for (int w = 0; w < warp; ++w) off += wsum[w];
        int run = off + incl - local;
        for (int s = beg; s < end; ++s) {
            cum[s] = run;
            const int L = checked_len(p, s);
            run += num_parts(p, L < 0 ? 0 : L) - 1;
        }
        if ((int)threadIdx.x == nthr - 1) cum[S] = run;
    }
    __syncthreads();

    const int64_t units_first = (int64_t)S * hkv;
    const int64_t total = units_first + (split ? (int64_t)cum[S] * hkv : 0);
    const int hq_total = p.num_q_heads;

    if (warp == C::kConsumerWarps) {
        // ------------------------------------------------------------ producer
        int64_t gq = 0, issued = 0;
        int uc = 0, q_issued = 0;
        for (int64_t u = blockIdx.x; u < total; u += gridDim.x, ++uc) {
            const Unit un = unit_of(u, units_first, hkv, cum, S);
            int L = checked_len(p, un.s);
            if (L < 0) {
                if (lane == 0 && un.part == 0 && un.h == 0) flag_error(p.err, PA_DEVERR_CONTEXT_LEN);
                L = 0;
            }
            int t0, nt;
            unit_range(p, un, L, t0, nt);
            const int nb = (nt + kBlockSize - 1) / kBlockSize;
            const int b = uc & 1;
            if (lane == 0 && !*abort_flag) {
                bool ok = true;
                if (uc >= 2) ok = mbar_wait_bounded(&qempty[b], ((uc >> 1) - 1) & 1, abort_flag, p.err);
                if (ok) {
                    const uint32_t qbytes = G * C::kRowBytes;
                    mbar_arrive_expect_tx(&qfull[b], qbytes);
                    bulk_g2s(qbuf + b * qbytes,
                             p.q + ((int64_t)un.s * hq_total + (int64_t)un.h * G) * C::kRowBytes,
                             qbytes, &qfull[b]);
                    q_issued = uc + 1;
                }
            }
            const int32_t *trow = p.tables + (int64_t)un.s * p.max_blocks + t0 / kBlockSize;
            for (int jc = 0; jc < nb; jc += 32) {
                const int j = jc + lane;
                const int phys = j < nb ? __ldg(trow + j) : 0;
                const int cnt = min(32, nb - jc);
                for (int jj = 0; jj < cnt; ++jj, ++gq) {
                    const int blk = __shfl_sync(kFull, phys, jj);
                    if (lane == 0 && !*abort_flag) {
                        const int slot = (int)(gq % C::kStages);
                        if (gq >= C::kStages &&
                            !mbar_wait_bounded(&empty[slot], (uint32_t)((gq / C::kStages - 1) & 1),
                                               abort_flag, p.err))
                            continue;
                        const bool ok = blk >= 0 && blk < p.num_blocks;
                        slot_ok[slot] = ok;
                        if (ok) {
                            const int64_t off = ((int64_t)blk * hkv + un.h) * C::kSlabBytes;
                            unsigned char *dst = ring + (size_t)slot * C::kStageBytes;
                            mbar_arrive_expect_tx(&full[slot], 2 * C::kSlabBytes);
                            bulk_g2s(dst, p.kc + off, C::kSlabBytes, &full[slot]);
                            bulk_g2s(dst + C::kSlabBytes, p.vc + off, C::kSlabBytes, &full[slot]);
                        } else {
                            flag_error(p.err, PA_DEVERR_BLOCK_ID);
                            mbar_arrive(&full[slot]);
                        }
                        issued = gq + 1;
                    }
                }
            }
        }
        // After an abort, wait for copies that may still be landing in our smem.
        if (lane == 0 && *abort_flag) {
            for (int64_t g = issued > C::kStages ? issued - C::kStages : 0; g < issued; ++g)
                mbar_wait_drain(&full[g % C::kStages], (uint32_t)((g / C::kStages) & 1));
            for (int k = q_issued > 2 ? q_issued - 2 : 0; k < q_issued; ++k)
                mbar_wait_drain(&qfull[k & 1], (uint32_t)((k >> 1) & 1));
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    float *pw = pbuf + warp * C::kPWarpFloats;
    const int tq = lane >> 3, part = lane & 7;
    const int hd = part >> (3 - C::kLogG);
    int64_t gq = 0;
    int uc = 0;
    for (int64_t u = blockIdx.x; u < total; u += gridDim.x, ++uc) {
        const Unit un = unit_of(u, units_first, hkv, cum, S);
        int L = checked_len(p, un.s);
        if (L < 0) L = 0;
        int t0, nt;
        unit_range(p, un, L, t0, nt);
        const int nb = (nt + kBlockSize - 1) / kBlockSize;
        const int b = uc & 1;

        bool live = !*abort_flag;
        if (live) live = mbar_wait_bounded(&qfull[b], (uint32_t)((uc >> 1) & 1), abort_flag, p.err);
        live = __all_sync(kFull, live);
        float2 qreg[G][C::kQkPairs];
        if (live) {
            const unsigned char *qs = qbuf + b * G * C::kRowBytes;
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int i = 0; i < C::kQkChunks; ++i) {
                    const uint4 raw =
                        *reinterpret_cast<const uint4 *>(qs + h * C::kRowBytes + (part + 8 * i) * 16);
                    float2 f[C::kEpc / 2];
                    unpack16<T>(raw, f);
#pragma unroll
                    for (int k = 0; k < C::kEpc / 2; ++k)
                        qreg[h][i * (C::kEpc / 2) + k] =
                            make_float2(f[k].x * p.scale_log2, f[k].y * p.scale_log2);
                }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&qempty[b]);

        float m = -INFINITY, l = 0.f;
        float2 acc[G][C::kPvPairs];
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int k = 0; k < C::kPvPairs; ++k) acc[h][k] = make_float2(0.f, 0.f);

        for (int j = warp; j < nb; j += C::kConsumerWarps) {
            const int64_t g = gq + j;
            const int slot = (int)(g % C::kStages);
            if (live)
                live = mbar_wait_bounded(&full[slot], (uint32_t)((g / C::kStages) & 1), abort_flag,
                                         p.err);
            live = __all_sync(kFull, live);
            if (live && slot_ok[slot]) {
                const int ntok = min(kBlockSize, nt - j * kBlockSize);
                const unsigned char *kb = ring + (size_t)slot * C::kStageBytes;
                process_block<T, D, G>(kb, kb + C::kSlabBytes, ntok, qreg, m, l, acc, pw, lane);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }
        gq += nb;

        // merge the consumer warps' partial states for this unit
        float *wacc = macc + ((size_t)b * C::kConsumerWarps + warp) * G * D;
        float2 *wml = mml + ((size_t)b * C::kConsumerWarps + warp) * G;
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int k = 0; k < C::kPvPairs; ++k)
                *reinterpret_cast<float2 *>(wacc + h * D + lane * C::kDpl + 2 * k) = acc[h][k];
        if (tq == 0 && (part & C::kDupMask) == 0) wml[hd] = make_float2(m, l);
        named_barrier(1, C::kConsumerWarps * 32);
        if (*abort_flag) continue;

        const float2 *uml = mml + (size_t)b * C::kConsumerWarps * G;
        const float *uacc = macc + (size_t)b * C::kConsumerWarps * G * D;
        const bool single = num_parts(p, L) == 1;
        const int64_t head0 = (int64_t)un.s * hq_total + (int64_t)un.h * G;
        for (int e = threadIdx.x; e < G * D; e += C::kConsumerWarps * 32) {
            const int h = e / D, dd = e - h * D;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < C::kConsumerWarps; ++w) M = fmaxf(M, uml[w * G + h].x);
            float lsum = 0.f, o = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < C::kConsumerWarps; ++w) {
                    const float2 ml = uml[w * G + h];
                    if (ml.x != -INFINITY) {
                        const float f = fast_exp2(ml.x - M);
                        lsum = fmaf(ml.y, f, lsum);
                        o = fmaf(uacc[(w * G + h) * D + dd], f, o);
                    }
                }
            }
            if (single) {
                store_out<T>(p.out, (head0 + h) * D + dd, lsum > 0.f ? o / lsum : 0.f);
            } else {
                const int64_t row = (head0 + h) * p.max_parts + un.part;
                p.ws_acc[row * D + dd] = o;
                if (dd == 0) p.ws_ml[row] = make_float2(M, lsum);
            }
        }
    }
}

// Combine split-K partials: one warp per (sequence, query head) with more than
// one partition.  M = max_p m_p; out = sum_p 2^(m_p-M) acc_p / sum_p 2^(m_p-M) l_p.
template <typename T, int D>
__global__ void __launch_bounds__(128) reduce_kernel(const Params p) {
    constexpr int kDpl = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t wid = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (wid >= (int64_t)p.num_seqs * p.num_q_heads) return;
    const int s = (int)(wid / p.num_q_heads);
    int L = checked_len(p, s);
    if (L < 0) L = 0;
    const int n = num_parts(p, L);
    if (n <= 1) return;
    const float2 *ml = p.ws_ml + wid * p.max_parts;
    const float *acc = p.ws_acc + wid * p.max_parts * D + lane * kDpl;
    float M = -INFINITY;
    for (int i = lane; i < n; i += 32) M = fmaxf(M, ml[i].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
    float lsum = 0.f, o[kDpl];
#pragma unroll
    for (int k = 0; k < kDpl; ++k) o[k] = 0.f;
#pragma unroll 4
    for (int i = 0; i < n; ++i) {
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
    for (int k = 0; k < kDpl; ++k) store_out<T>(p.out, wid * D + lane * kDpl + k, o[k] * inv);
}

template <typename T, int D, int G>
cudaError_t launch_t(const DecodeLaunch &a, const Params &prm, cudaStream_t stream) {
    using C = Cfg<T, D, G>;
    const bool split = prm.part_tokens > 0;
    const size_t smem = C::smem_bytes(split ? a.num_seqs + 1 : 0);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static_assert(C::smem_bytes(kMaxSplitSeqs + 1) <= 232448, "decode smem over the sm_100 limit");
    e = cudaFuncSetAttribute(decode_kernel<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)C::smem_bytes(kMaxSplitSeqs + 1));
    if (e != cudaSuccess) return e;
    int64_t grid = num_sms(dev);
    if (!split) grid = std::min<int64_t>(grid, (int64_t)a.num_seqs * a.cache.num_kv_heads);
    if (grid < 1) grid = 1;
    decode_kernel<T, D, G><<<(unsigned)grid, C::kThreads, smem, stream>>>(prm);
    e = cudaGetLastError();
    if (e != cudaSuccess || !split) return e;
    const int64_t warps = (int64_t)a.num_seqs * a.num_q_heads;
    reduce_kernel<T, D><<<(unsigned)((warps + 3) / 4), 128, 0, stream>>>(prm);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_g(const DecodeLaunch &a, const Params &prm, cudaStream_t stream) {
    switch (a.num_q_heads / a.cache.num_kv_heads) {
        case 1: return launch_t<T, D, 1>(a, prm, stream);
        case 2: return launch_t<T, D, 2>(a, prm, stream);
        case 4: return launch_t<T, D, 4>(a, prm, stream);
        case 8: return launch_t<T, D, 8>(a, prm, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode(const DecodeLaunch &a, cudaStream_t stream) {
    Params prm;
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
    prm.scale_log2 = a.scale * kLog2e;
    const bool bf16 = a.cache.dtype == PA_BF16;
    if (a.cache.head_dim == 128)
        return bf16 ? launch_g<__nv_bfloat16, 128>(a, prm, stream) : launch_g<float, 128>(a, prm, stream);
    if (a.cache.head_dim == 64)
        return bf16 ? launch_g<__nv_bfloat16, 64>(a, prm, stream) : launch_g<float, 64>(a, prm, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
