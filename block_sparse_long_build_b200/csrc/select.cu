// A2 (block scoring) + A3 (selection), sm_100a.
//
// Scores: "Sparse long-context inference with self-indexing attention",
// "Importance scores and block selection" (ranked by raw score: softmax is
// monotone); MoBA gating (Module 14 §14.3) with mean-pooled keys; Quest page
// bounds ("Sparse attention in hybrid LLMs") scored as
// sum_i max(q_i*min_i, q_i*max_i).
// Forced tokens: attention sink (§14.2), sliding window ("Sliding window"),
// MoBA's current block (§14.3); semantic blocks take a token budget
// ("Semantic blocks for sparse attention", K = L/16).
//
// Two kernels, chained by programmatic dependent launch:
//  score_kernel  persistent; work items are (segment, tile of 128 blocks).
//                Each CTA streams its items' summary rows into a ring of
//                shared-memory stages with 2-D TMA loads (128-byte swizzle, so
//                that thread j reading row j is conflict-free) together with
//                the group's queries (1-D bulk copy), scores one block per
//                thread in the fixed fp32 order (fma chain over the dimensions
//                per query head, the G chains interleaved, heads summed in
//                order) and writes orderable uint32 keys to the workspace.
//  pick_kernel   one 512-thread CTA per segment: candidates (not wholly inside
//                the forced set), then a radix select of the k-th key for
//                top-k or a greedy walk for the token budget, an
//                index-ordered compaction (ties go to the lower block index),
//                and the merge of forced ranges and selected blocks into
//                disjoint ranges with parallel scans.
#include <algorithm>
#include <type_traits>

#include "common.cuh"

namespace bsa {

constexpr int kSelThreads = 128;   // scoring threads = rows per tile
constexpr int kPickThreads = 512;
constexpr int kSelMaxG = 16;
constexpr int kSelMaxStages = 3;
constexpr int kScoreStages = 1;    // tile stages per CTA: several CTAs per SM overlap instead
constexpr int kIntMin = -0x7fffffff - 1;
enum { kScoreCentroid = 0, kScoreMinmaxBf16 = 1, kScoreMinmaxF32 = 2 };

struct SelArgs {
    const float *q;
    const int32_t *cur_len;
    const int32_t *offsets;
    const int32_t *kv_pos;
    int32_t *sel_blocks, *sel_count, *ranges, *n_ranges;
    uint32_t *keys;       // ws [nseg][nb_total]
    int32_t *vis;         // ws [nseg][nb_total]
    uint32_t *counters;   // ws [nseg]
    uint32_t *status;
    int B, Hq, Hkv, G, D, L_max, S, nb_total;
    int topk, budget, sink, window, keep_current, local_start, pos_limit;
    int max_sel, max_ranges;
    int row_bytes, nbox;
    int tiles_per_seg, n_items, nst;   // scoring work items and ring stages
    uint32_t tile_bytes;
};

// 16-byte chunk of row j at byte offset `off` of a 128-byte-swizzled tile
// made of boxes of [kSelThreads rows][128 B].
__device__ __forceinline__ const uint4 *tile_chunk(const unsigned char *tile, int j, int off) {
    const int box = off >> 7, c = (off >> 4) & 7;
    return reinterpret_cast<const uint4 *>(tile + box * (kSelThreads * 128) + j * 128 +
                                           ((c ^ (j & 7)) << 4));
}

// Threads per block row and heads per thread of the scoring kernel: one
// thread per block row holds all G head chains, so each summary row is read
// from shared memory once and the query values are warp-wide broadcasts.
__host__ __device__ constexpr int score_tpb(int) { return 1; }
__host__ __device__ constexpr int score_hpt(int GT) { return GT == 0 ? kSelMaxG : GT; }

// Byte-permute selectors that widen the min (bytes 0-1) or the max (bytes
// 2-3) of a packed (min, max) bf16 pair into fp32 bits (zeros from the second
// operand below): x = max where q >= 0, else min.
constexpr uint32_t kPickMin = 0x1044u, kPickMax = 0x3244u;

__device__ __forceinline__ float widen_bf16(uint32_t pair, uint32_t sel) {
    uint32_t x;
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(x) : "r"(pair), "r"(sel));
    return __uint_as_float(x);
}

// Partial scores of tile row j for heads h0 .. h0 + HPT - 1 (those below G):
// per head an fma chain over i = 0..D-1 in the fixed fp32 order; the chains
// of the thread's heads are interleaved.  qs: head rows of D + 4 floats; sl:
// the same layout of min/max selectors (bf16 min/max only).  DT: D when
// known at compile time (the dimension loop unrolls and the row's swizzled
// chunk offsets are computed once), 0 otherwise.
template <int SK, int HPT, int DT>
__device__ __forceinline__ void score_heads(const float *qs, const uint32_t *sl, int h0, int G, int Drt,
                                            const unsigned char *tile, int j, float (&acc)[HPT]) {
    const int D = DT > 0 ? DT : Drt;
    const int qstride = D + 4;
#pragma unroll
    for (int h = 0; h < HPT; ++h) acc[h] = 0.0f;
    const unsigned char *row = tile + j * 128;
    uint32_t sw[8];   // swizzled offset of 16-byte chunk c within the row's 128 bytes
#pragma unroll
    for (int c = 0; c < 8; ++c) sw[c] = (uint32_t)((c ^ (j & 7)) << 4);
    auto chunk = [&](int off) -> uint4 {
        if constexpr (DT > 0)
            return *reinterpret_cast<const uint4 *>(row + (off >> 7) * (kSelThreads * 128) + sw[(off >> 4) & 7]);
        else
            return *tile_chunk(tile, j, off);
    };
    auto step = [&](int i) {
        if constexpr (SK == kScoreMinmaxBf16) {   // dimensions i .. i+3, one (min, max) pair each
            const uint4 w = chunk(i * 4);
#pragma unroll
            for (int h = 0; h < HPT; ++h) {
                if (h0 + h >= G) break;
                const float4 q4 = *reinterpret_cast<const float4 *>(qs + (h0 + h) * qstride + i);
                const uint4 s4 = *reinterpret_cast<const uint4 *>(sl + (h0 + h) * qstride + i);
                acc[h] = __fmaf_rn(q4.x, widen_bf16(w.x, s4.x), acc[h]);
                acc[h] = __fmaf_rn(q4.y, widen_bf16(w.y, s4.y), acc[h]);
                acc[h] = __fmaf_rn(q4.z, widen_bf16(w.z, s4.z), acc[h]);
                acc[h] = __fmaf_rn(q4.w, widen_bf16(w.w, s4.w), acc[h]);
            }
        } else if constexpr (SK == kScoreMinmaxF32) {   // dimensions i, i+1: (min, max) pairs
            const uint4 w = chunk(i * 8);
#pragma unroll
            for (int h = 0; h < HPT; ++h) {
                if (h0 + h >= G) break;
                const float2 q2 = *reinterpret_cast<const float2 *>(qs + (h0 + h) * qstride + i);
                const float x0 = q2.x >= 0.0f ? __uint_as_float(w.y) : __uint_as_float(w.x);
                const float x1 = q2.y >= 0.0f ? __uint_as_float(w.w) : __uint_as_float(w.z);
                acc[h] = __fmaf_rn(q2.x, x0, acc[h]);
                acc[h] = __fmaf_rn(q2.y, x1, acc[h]);
            }
        } else {   // centroid: dimensions i .. i+3
            const uint4 a = chunk(i * 4);
            const float x[4] = {__uint_as_float(a.x), __uint_as_float(a.y), __uint_as_float(a.z),
                                __uint_as_float(a.w)};
#pragma unroll
            for (int h = 0; h < HPT; ++h) {
                if (h0 + h >= G) break;
                const float4 q4 = *reinterpret_cast<const float4 *>(qs + (h0 + h) * qstride + i);
                const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[h] = __fmaf_rn(qv[e], x[e], acc[h]);
            }
        }
    };
    constexpr int W = SK == kScoreMinmaxF32 ? 2 : 4;   // dimensions per 16-byte chunk
    if constexpr (DT > 0) {
#pragma unroll
        for (int i = 0; i < DT; i += W) step(i);
    } else {
        for (int i = 0; i < D; i += W) step(i);
    }
}

// Rows of [r0, r1) whose position is below lim (positions ascend within a
// block): rounds of 16 independent probes narrow the boundary, then at most
// 16 rows are counted directly.
__device__ __forceinline__ int visible_prefix(const int32_t *pos, int r0, int r1, int lim) {
    constexpr int P = 16;
    int lo = r0, hi = r1;   // rows < lo are visible, rows >= hi are not
    while (hi - lo > P) {
        const int w = hi - lo;
        int p[P];
        bool below[P];
#pragma unroll
        for (int k = 0; k < P; ++k) p[k] = lo + (int)((int64_t)(k + 1) * w / (P + 1));
#pragma unroll
        for (int k = 0; k < P; ++k) below[k] = __ldg(pos + p[k]) < lim;
        // positions ascend, so the probes below lim come first
        int nlo = lo, nhi = hi;
#pragma unroll
        for (int k = 0; k < P; ++k)
            if (below[k]) nlo = p[k] + 1;
#pragma unroll
        for (int k = P - 1; k >= 0; --k)
            if (!below[k]) nhi = p[k];
        lo = nlo;
        hi = nhi;
    }
    int c = 0;
#pragma unroll
    for (int k = 0; k < P; ++k) c += (lo + k < hi) && __ldg(pos + lo + k) < lim;
    return lo - r0 + c;
}

// ---------------------------------------------------------------- scoring
template <int SK, int GT, int DT>
__global__ void __launch_bounds__(kSelThreads * score_tpb(GT), 3)
    score_kernel(const __grid_constant__ CUtensorMap tmS, SelArgs a) {
    constexpr int TPB = score_tpb(GT), HPT = score_hpt(GT);
    extern __shared__ unsigned char dsm_raw[];
    unsigned char *ring = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
    const int G = GT > 0 ? GT : a.G, D = a.D, nb = a.nb_total;
    const int qstage = G * (D + 4);                                                 // floats
    float *qbuf = reinterpret_cast<float *>(ring + (size_t)a.nst * a.tile_bytes);   // [nst][G][D+4]
    uint32_t *selb = reinterpret_cast<uint32_t *>(qbuf + (size_t)a.nst * qstage);   // [G][D+4]
    __shared__ uint64_t full[kSelMaxStages];
    const int tid = threadIdx.x, lane = tid & 31;
    const int row = tid / TPB, part = tid % TPB;   // block row of the tile, head slice
    const int my_items =
        a.n_items > (int)blockIdx.x ? (a.n_items - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
    if (tid == 0) {
        prefetch_tmap(&tmS);
        for (int i = 0; i < a.nst; ++i) mbar_init(&full[i], 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();   // queries, lengths and summaries come from earlier kernels
    const int esz = SK == kScoreMinmaxBf16 ? 2 : 4;
    auto issue = [&](int k) {   // thread 0: item k of this CTA into stage k % nst
        const int item = (int)blockIdx.x + k * (int)gridDim.x;
        const int s = item / a.tiles_per_seg, t = item % a.tiles_per_seg;
        const int st = k % a.nst;
        const int b = s / a.Hkv, g = s % a.Hkv;
        unsigned char *dst = ring + (size_t)st * a.tile_bytes;
        mbar_arrive_expect_tx(&full[st], a.tile_bytes + (uint32_t)(G * D * 4));
        for (int bx = 0; bx < a.nbox; ++bx)
            tma_load_2d(dst + bx * (kSelThreads * 128), &tmS, &full[st], bx * (128 / esz),
                        s * nb + t * kSelThreads);
        const float *qg = a.q + ((int64_t)b * a.Hq + (int64_t)g * G) * D;
        for (int h = 0; h < G; ++h)   // head rows padded to D + 4 floats (conflict-free reads)
            bulk_load(qbuf + (size_t)st * qstage + h * (D + 4), qg + h * D, (uint32_t)(D * 4), &full[st]);
    };
    if (tid == 0)
        for (int k = 0; k < a.nst && k < my_items; ++k) issue(k);
    bool timed_out = false;
    for (int k = 0; k < my_items; ++k) {
        const int item = (int)blockIdx.x + k * (int)gridDim.x;
        const int s = item / a.tiles_per_seg, t = item % a.tiles_per_seg;
        const int b = s / a.Hkv;
        const int j = t * kSelThreads + row;
        const bool writer = part == TPB - 1;
        // candidacy needs no summary: worked out while the tile is in flight
        int vis = 0;
        bool valid = false;
        if (writer && j < nb) {
            if (a.offsets) {
                const int32_t *off = a.offsets + (int64_t)s * (nb + 1);
                const int r0 = min(max(off[j], 0), a.L_max), r1 = min(max(off[j + 1], r0), a.L_max);
                vis = visible_prefix(a.kv_pos + (int64_t)s * a.L_max, r0, r1, a.pos_limit);
                valid = vis > 0;
            } else {
                const int n = min(max(a.cur_len[b], 0), a.L_max);
                valid = (int64_t)(j + 1) * a.S <= n;
            }
        }
        const int st = k % a.nst;
        if (!timed_out && !mbar_wait_bounded(&full[st], (uint32_t)((k / a.nst) & 1))) {
            timed_out = true;
            atomicOr(a.status, 2u);
        }
        const float *qs = qbuf + (size_t)st * qstage;
        if constexpr (SK == kScoreMinmaxBf16) {
            // per (head, dimension): which bound the query's sign picks
            for (int e = tid; e < G * D; e += blockDim.x) {
                const int h = e / D, i = e % D;
                selb[h * (D + 4) + i] = qs[h * (D + 4) + i] < 0.0f ? kPickMin : kPickMax;
            }
            __syncthreads();
        }
        float acc[HPT];
        score_heads<SK, HPT, DT>(qs, selb, part * HPT, G, D, ring + (size_t)st * a.tile_bytes, row, acc);
        // heads summed in head order: the slices hand the running sum on
        float run = acc[0];
#pragma unroll
        for (int h = 1; h < HPT; ++h)
            if (part * HPT + h < G) run = __fadd_rn(run, acc[h]);
#pragma unroll
        for (int q = 1; q < TPB; ++q) {
            const float prev = __shfl_up_sync(0xffffffffu, run, 1);
            if (part == q) {
                run = prev;
#pragma unroll
                for (int h = 0; h < HPT; ++h) run = __fadd_rn(run, acc[h]);
            }
        }
        if (writer && j < nb) {
            uint32_t key = 0;
            if (valid) {
                key = f32_order_key(__fadd_rn(run, 0.0f));
                if (key == 0) key = 1;   // 0 marks "not a candidate"
            }
            a.keys[(int64_t)s * nb + j] = key;
            if (a.offsets) a.vis[(int64_t)s * nb + j] = vis;
        }
        __syncthreads();   // stage st has been read by every thread
        if (tid == 0 && k + a.nst < my_items) issue(k + a.nst);
    }
    (void)lane;
    pdl_trigger();
}

// Scoring with two block rows per thread, for G = 4, 8 or 16 and D = 64 or
// 128 (min/max bf16 bounds or fp32 centroids).  A tile is R = kPairRows rows
// and the CTA R threads; lanes 2p and 2p + 1 take rows p and p + R/2 of it, lane 2p the first G/2 heads and
// lane 2p + 1 the others.  Each head's score is still one fp32 fma chain over
// i = 0..D-1, the two rows' chains advanced together by fma.rn.f32x2 (each
// half rounded once, as fmaf); the query values and bound selectors a step
// needs are read once for both rows.  Head sums in head order: lane 2p adds
// its heads, lane 2p + 1 continues from that sum with its own.
#ifndef BSA_SCORE_PAIR_ROWS
#define BSA_SCORE_PAIR_ROWS 64
#endif
#ifndef BSA_SCORE_PAIR_STAGES
#define BSA_SCORE_PAIR_STAGES 1
#endif
constexpr int kPairRows = BSA_SCORE_PAIR_ROWS;   // rows per tile = threads per CTA
static_assert(kPairRows == 64 || kPairRows == 128, "tile of 64 or 128 rows");

// dynamic shared memory of score_pair_kernel: nst tile stages and query
// buffers, the bound selectors and nst barriers (no alignment slack)
inline size_t pair_smem_bytes(int nst, uint32_t tile_bytes, size_t qbytes) {
    return (size_t)nst * (tile_bytes + qbytes) + qbytes + (size_t)nst * 8;
}

template <int SK, int G, int D>
__global__ void __launch_bounds__(kPairRows, 384 / kPairRows)
    score_pair_kernel(const __grid_constant__ CUtensorMap tmS, SelArgs a) {
    constexpr int HPT = G / 2;
    static_assert(G % 2 == 0 && G <= kSelMaxG, "pairs of head slices");
    // No static shared memory and no alignment slack: the dynamic block
    // starts 1024-byte aligned, so the ring sits at its start and the query
    // rows, selectors and barriers after it (sizes in pair_smem_bytes).
    extern __shared__ __align__(1024) unsigned char dsm_raw[];
    unsigned char *ring = dsm_raw;
    const int nb = a.nb_total;
    constexpr int QS = D + 4;                                                       // floats per head row
    float *qbuf = reinterpret_cast<float *>(ring + (size_t)a.nst * a.tile_bytes);   // [nst][G][D+4]
    uint32_t *selb = reinterpret_cast<uint32_t *>(qbuf + (size_t)a.nst * G * QS);   // [G][D+4]
    uint64_t *full = reinterpret_cast<uint64_t *>(selb + G * QS);                  // [nst]
    const int tid = threadIdx.x;
    if (smem_u32(dsm_raw) & 1023u) {   // the swizzled TMA boxes need it: report, touch nothing
        if (tid == 0) atomicOr(a.status, 2u);
        return;
    }
    const int pr = tid >> 1, part = tid & 1;   // row pair (rows pr, pr + 64), head half
    const int my_items =
        a.n_items > (int)blockIdx.x ? (a.n_items - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
    if (tid == 0) {
        prefetch_tmap(&tmS);
        for (int i = 0; i < a.nst; ++i) mbar_init(&full[i], 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();   // queries, lengths and summaries come from earlier kernels
    constexpr int esz = SK == kScoreMinmaxBf16 ? 2 : 4;
    auto issue = [&](int k) {   // thread 0: item k of this CTA into stage k % nst
        const int item = (int)blockIdx.x + k * (int)gridDim.x;
        const int s = item / a.tiles_per_seg, t = item % a.tiles_per_seg;
        const int st = k % a.nst;
        const int b = s / a.Hkv, g = s % a.Hkv;
        unsigned char *dst = ring + (size_t)st * a.tile_bytes;
        mbar_arrive_expect_tx(&full[st], a.tile_bytes + (uint32_t)(G * D * 4));
        for (int bx = 0; bx < a.nbox; ++bx)
            tma_load_2d(dst + bx * (kPairRows * 128), &tmS, &full[st], bx * (128 / esz),
                        s * nb + t * kPairRows);
        const float *qg = a.q + ((int64_t)b * a.Hq + (int64_t)g * G) * D;
        for (int h = 0; h < G; ++h)
            bulk_load(qbuf + (size_t)st * G * QS + h * QS, qg + h * D, (uint32_t)(D * 4), &full[st]);
    };
    if (tid == 0)
        for (int k = 0; k < a.nst && k < my_items; ++k) issue(k);
    bool timed_out = false;
    for (int k = 0; k < my_items; ++k) {
        const int item = (int)blockIdx.x + k * (int)gridDim.x;
        const int s = item / a.tiles_per_seg, t = item % a.tiles_per_seg;
        const int b = s / a.Hkv;
        const int j0 = t * kPairRows + pr, j1 = j0 + kPairRows / 2;
        const bool writer = part == 1;
        // candidacy needs no summary: worked out while the tile is in flight
        int vis0 = 0, vis1 = 0;
        bool valid0 = false, valid1 = false;
        if (writer) {
            if (a.offsets) {
                const int32_t *off = a.offsets + (int64_t)s * (nb + 1);
                const int32_t *pos = a.kv_pos + (int64_t)s * a.L_max;
                if (j0 < nb) {
                    const int r0 = min(max(off[j0], 0), a.L_max), r1 = min(max(off[j0 + 1], r0), a.L_max);
                    vis0 = visible_prefix(pos, r0, r1, a.pos_limit);
                    valid0 = vis0 > 0;
                }
                if (j1 < nb) {
                    const int r0 = min(max(off[j1], 0), a.L_max), r1 = min(max(off[j1 + 1], r0), a.L_max);
                    vis1 = visible_prefix(pos, r0, r1, a.pos_limit);
                    valid1 = vis1 > 0;
                }
            }
        }
        // fixed blocks: the length is loaded now and compared after the scoring
        const int n_fixed = !a.offsets && writer ? __ldg(a.cur_len + b) : 0;
        const int st = k % a.nst;
        if (!timed_out && !mbar_wait_bounded(&full[st], (uint32_t)((k / a.nst) & 1))) {
            timed_out = true;
            atomicOr(a.status, 2u);
        }
        const float *qs = qbuf + (size_t)st * G * QS;
        if constexpr (SK == kScoreMinmaxBf16) {
            // per (head, dimension): which bound the query's sign picks
            for (int e = tid; e < G * D; e += blockDim.x) {
                const int h = e / D, i = e % D;
                selb[h * QS + i] = qs[h * QS + i] < 0.0f ? kPickMin : kPickMax;
            }
            __syncthreads();
        }
        const unsigned char *tile = ring + (size_t)st * a.tile_bytes;
        const unsigned char *rowA = tile + pr * 128;
        const unsigned char *rowB = tile + (pr + kPairRows / 2) * 128;
        uint32_t sw[8];   // swizzled chunk offsets; rows pr and pr + 64 share them
#pragma unroll
        for (int c = 0; c < 8; ++c) sw[c] = (uint32_t)((c ^ (pr & 7)) << 4);
        float acc0[HPT], acc1[HPT];
#pragma unroll
        for (int h = 0; h < HPT; ++h) acc0[h] = acc1[h] = 0.0f;
        const int h0 = part * HPT;
        constexpr int W = 4;   // dimensions per 16-byte chunk (bf16 pairs or fp32)
#pragma unroll
        for (int i = 0; i < D; i += W) {
            const int off = SK == kScoreMinmaxBf16 ? i * 4 : i * 4;   // bytes into the row
            const int box = off >> 7, c = (off >> 4) & 7;
            const uint4 wa = *reinterpret_cast<const uint4 *>(rowA + box * (kPairRows * 128) + sw[c]);
            const uint4 wb = *reinterpret_cast<const uint4 *>(rowB + box * (kPairRows * 128) + sw[c]);
            const uint32_t xa[4] = {wa.x, wa.y, wa.z, wa.w}, xb[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int h = 0; h < HPT; ++h) {
                const float4 q4 = *reinterpret_cast<const float4 *>(qs + (h0 + h) * QS + i);
                const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
                if constexpr (SK == kScoreMinmaxBf16) {
                    const uint4 s4 = *reinterpret_cast<const uint4 *>(selb + (h0 + h) * QS + i);
                    const uint32_t sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        fma2_shared_a(acc0[h], acc1[h], qv[e], widen_bf16(xa[e], sv[e]),
                                      widen_bf16(xb[e], sv[e]));
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        fma2_shared_a(acc0[h], acc1[h], qv[e], __uint_as_float(xa[e]), __uint_as_float(xb[e]));
                }
            }
        }
        // heads summed in head order: lane 2p's heads, then lane 2p + 1's
        float run0 = acc0[0], run1 = acc1[0];
#pragma unroll
        for (int h = 1; h < HPT; ++h) {
            run0 = __fadd_rn(run0, acc0[h]);
            run1 = __fadd_rn(run1, acc1[h]);
        }
        const float prev0 = __shfl_up_sync(0xffffffffu, run0, 1);
        const float prev1 = __shfl_up_sync(0xffffffffu, run1, 1);
        if (writer) {
            if (!a.offsets) {
                const int n = min(max(n_fixed, 0), a.L_max);
                valid0 = j0 < nb && (int64_t)(j0 + 1) * a.S <= n;
                valid1 = j1 < nb && (int64_t)(j1 + 1) * a.S <= n;
            }
            run0 = prev0;
            run1 = prev1;
#pragma unroll
            for (int h = 0; h < HPT; ++h) {
                run0 = __fadd_rn(run0, acc0[h]);
                run1 = __fadd_rn(run1, acc1[h]);
            }
            auto put = [&](int j, bool valid, int vis, float run) {
                if (j >= nb) return;
                uint32_t key = 0;
                if (valid) {
                    key = f32_order_key(__fadd_rn(run, 0.0f));
                    if (key == 0) key = 1;   // 0 marks "not a candidate"
                }
                a.keys[(int64_t)s * nb + j] = key;
                if (a.offsets) a.vis[(int64_t)s * nb + j] = vis;
            };
            put(j0, valid0, vis0, run0);
            put(j1, valid1, vis1, run1);
        }
        __syncthreads();   // stage st has been read by every thread
        if (tid == 0 && k + a.nst < my_items) issue(k + a.nst);
    }
    pdl_trigger();
}

// ---------------------------------------------------------------- picking
constexpr int kPickWarpKeys = 16;   // keys per lane of the one-warp walks (nb <= 512)

// Dynamic shared memory: [keys nb][vis nb][taken nb bytes, padded][sel
// max_sel][hist 256][merge items (max_sel + 4) x int2][prefix maxima
// (max_sel + 4) x int]
struct PickSmem {
    __host__ __device__ static size_t keys(int) { return 0; }
    __host__ __device__ static size_t vis(int nb) { return (size_t)nb * 4; }
    __host__ __device__ static size_t taken(int nb) { return (size_t)nb * 8; }
    __host__ __device__ static size_t sel(int nb) { return (size_t)nb * 8 + (((size_t)nb + 15) & ~size_t(15)); }
    __host__ __device__ static size_t hist(int nb, int max_sel) { return sel(nb) + (size_t)max_sel * 4; }
    __host__ __device__ static size_t mrg(int nb, int max_sel) {
        return (hist(nb, max_sel) + 256 * 4 + 7) & ~size_t(7);
    }
    __host__ __device__ static size_t pmax(int nb, int max_sel) {
        return mrg(nb, max_sel) + (size_t)(max_sel + 4) * 8;
    }
    __host__ __device__ static size_t bytes(int nb, int max_sel) {
        return pmax(nb, max_sel) + (size_t)(max_sel + 4) * 4;
    }
};

// One warp takes, one at a time, the best remaining candidate (highest key,
// then lowest index) -- that fits in what is left of the budget when
// `budget` >= 0 -- up to `limit` blocks, marking them in taken[].  A step is a
// warp max of the live keys and a warp min of the indices holding it (both
// redux.sync); a taken block's key is cleared, and under a budget so is every
// key whose visible rows no longer fit (what is left only shrinks).  Keys
// and visible counts of blocks lane + 32 r live in registers (nb <= 512).
__device__ __forceinline__ void warp_walk_regs(const uint32_t *keys, const int32_t *visb, unsigned char *taken,
                                               int nb, int limit, int budget, int lane) {
    uint32_t wk[kPickWarpKeys];
    int wv[kPickWarpKeys];
    int remaining = budget;
#pragma unroll
    for (int r = 0; r < kPickWarpKeys; ++r) {
        const int j = lane + 32 * r;
        wk[r] = j < nb ? keys[j] : 0u;
        wv[r] = j < nb && budget >= 0 ? visb[j] : 0;
        if (budget >= 0 && wv[r] > remaining) wk[r] = 0u;
    }
    for (int n = 0; n < limit; ++n) {
        uint32_t lm = 0u;
#pragma unroll
        for (int r = 0; r < kPickWarpKeys; ++r) lm = max(lm, wk[r]);
        const uint32_t m = __reduce_max_sync(0xffffffffu, lm);
        if (m == 0u) break;
        int cand = 0x7fffffff;
#pragma unroll
        for (int r = kPickWarpKeys - 1; r >= 0; --r) cand = wk[r] == m ? lane + 32 * r : cand;
        const int j = __reduce_min_sync(0xffffffffu, cand);
        if (budget >= 0) remaining -= visb[j];
#pragma unroll
        for (int r = 0; r < kPickWarpKeys; ++r)
            if (lane + 32 * r == j || (budget >= 0 && wv[r] > remaining)) wk[r] = 0u;
        if (lane == 0) taken[j] = 1;
    }
}

// The same walk over shared memory (any nb).
__device__ void warp_walk_smem(const uint32_t *keys, const int32_t *visb, unsigned char *taken, int nb,
                               int limit, int budget, int lane) {
    int remaining = budget;
    for (int n = 0; n < limit; ++n) {
        uint32_t lm = 0u;
        for (int j = lane; j < nb; j += 32)
            if (keys[j] && !taken[j] && (budget < 0 || visb[j] <= remaining)) lm = max(lm, keys[j]);
        const uint32_t m = __reduce_max_sync(0xffffffffu, lm);
        if (m == 0u) break;
        int cand = 0x7fffffff;
        for (int j = lane; j < nb && cand == 0x7fffffff; j += 32)
            if (keys[j] == m && !taken[j] && (budget < 0 || visb[j] <= remaining)) cand = j;
        const int j = __reduce_min_sync(0xffffffffu, cand);
        if (budget >= 0) remaining -= visb[j];
        if (lane == 0) taken[j] = 1;
        __syncwarp();
    }
}

// One CTA per segment.  The candidate keys live in shared memory; thread t
// owns the contiguous blocks [t kpt, t kpt + kpt) for the index-ordered
// compactions.  Loops stay rolled (short unrolls batch the loads): the
// kernel runs once per selection, so compact code beats straight-line code.
__global__ void __launch_bounds__(kPickThreads, 2) pick_kernel(SelArgs a) {
    extern __shared__ __align__(16) unsigned char psm[];
    const int nb = a.nb_total;
    uint32_t *keys = reinterpret_cast<uint32_t *>(psm + PickSmem::keys(nb));
    int32_t *visb = reinterpret_cast<int32_t *>(psm + PickSmem::vis(nb));
    unsigned char *taken = psm + PickSmem::taken(nb);
    int32_t *sel = reinterpret_cast<int32_t *>(psm + PickSmem::sel(nb));
    int *hist = reinterpret_cast<int *>(psm + PickSmem::hist(nb, a.max_sel));
    int2 *mrg = reinterpret_cast<int2 *>(psm + PickSmem::mrg(nb, a.max_sel));
    int *pmax = reinterpret_cast<int *>(psm + PickSmem::pmax(nb, a.max_sel));
    __shared__ int tmp[40];
    __shared__ int f_lo[3], f_hi[3], n_forced, n_sel_sh, sh_bin, sh_excl;

    const int s = blockIdx.x;
    const int b = s / a.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int32_t *off = a.offsets ? a.offsets + (int64_t)s * (nb + 1) : nullptr;
    const int kpt = (nb + kPickThreads - 1) / kPickThreads;
    const int c0 = tid * kpt;   // this thread's blocks [c0, c0 + kpt)
    pdl_wait();   // keys and visible counts from score_kernel
    if (tid == 0) {
        // forced token ranges, sorted and merged
        const int n = min(max(a.cur_len[b], 0), a.L_max);
        int lo[3], hi[3], m = 0;
        if (off) {
            if (n > a.local_start) { lo[m] = max(a.local_start, 0); hi[m] = n; ++m; }
        } else {
            if (a.sink > 0 && n > 0) { lo[m] = 0; hi[m] = min(a.sink, n); ++m; }
            int t0 = n;
            if (a.window > 0) t0 = min(t0, max(0, n - a.window));
            if (a.keep_current && n > 0) t0 = min(t0, ((n - 1) / a.S) * a.S);
            if (t0 < n) {
                if (m > 0 && t0 <= hi[0]) hi[0] = n;
                else { lo[m] = t0; hi[m] = n; ++m; }
            }
        }
        for (int i = 0; i < m; ++i) { f_lo[i] = lo[i]; f_hi[i] = hi[i]; }
        n_forced = m;
    }
    __syncthreads();
    const int nf = n_forced;

    // candidates: keys > 0 and (fixed blocks) not wholly inside the forced
    // set; coalesced loads, eight in flight per thread
    int my_c = 0;
#pragma unroll 8
    for (int jj = tid; jj < nb; jj += kPickThreads) {
        uint32_t key = a.keys[(int64_t)s * nb + jj];
        if (key && !off) {
            const int64_t r0 = (int64_t)jj * a.S, r1 = r0 + a.S;
            for (int i = 0; i < nf; ++i)
                if (f_lo[i] <= r0 && r1 <= f_hi[i]) key = 0;
        }
        keys[jj] = key;
        taken[jj] = 0;
        if (off) visb[jj] = a.vis[(int64_t)s * nb + jj];
        my_c += key != 0;
    }
    int n_cand;
    cta_excl_sum(my_c, tmp, &n_cand);   // also publishes keys[] to the CTA

    const bool greedy = off && a.topk < 0;
    int k = 0;
    if (!greedy) k = min(min(a.topk >= 0 ? a.topk : a.budget / a.S, n_cand), a.max_sel);
    const bool small_nb = nb <= 32 * kPickWarpKeys;
    if (greedy || (k <= 32 && small_nb)) {
        // ---- one warp walks the ranking: the token budget (take a block
        // when its visible rows fit in what is left; that only shrinks, so a
        // block that does not fit now never will, and each step takes the
        // best remaining candidate that fits), or a small top-k
        if (warp == 0) {
            const int limit = greedy ? a.max_sel : k;
            const int budget = greedy ? a.budget : -1;
            if (small_nb) warp_walk_regs(keys, visb, taken, nb, limit, budget, lane);
            else warp_walk_smem(keys, visb, taken, nb, limit, budget, lane);
        }
        __syncthreads();
        int my_take = 0;
        for (int r = 0; r < kpt; ++r) my_take += c0 + r < nb && taken[c0 + r];
        int tot;
        int p = cta_excl_sum(my_take, tmp, &tot);
        for (int r = 0; r < kpt; ++r)
            if (c0 + r < nb && taken[c0 + r] && p < a.max_sel) sel[p++] = c0 + r;
        if (tid == 0) n_sel_sh = min(tot, a.max_sel);
    } else {
        // ---- top-k: radix select of the k-th largest key, 8 bits per pass
        uint32_t thr = 0xffffffffu;
        int need_eq = 0;
        if (k > 0) {
            uint32_t prefix = 0, pmask = 0;
            int krem = k;
            for (int pass = 0; pass < 4; ++pass) {
                const int shift = 24 - 8 * pass;
                if (tid < 256) hist[tid] = 0;
                __syncthreads();
#pragma unroll 4
                for (int r = 0; r < kpt; ++r) {
                    const uint32_t key = c0 + r < nb ? keys[c0 + r] : 0u;
                    const bool act = key && (key & pmask) == prefix;
                    const uint32_t bin = act ? (key >> shift) & 255u : 256u;
                    // lanes with the same bin add once (most keys share the
                    // high bits)
                    const unsigned peers = __match_any_sync(0xffffffffu, bin);
                    if (act && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
                }
                __syncthreads();
                // thread t < 256 owns bin 255 - t (counted from the top)
                const int v = tid < 256 ? hist[255 - tid] : 0;
                int tot;
                const int ex = cta_excl_sum(v, tmp, &tot);
                if (tid < 256 && ex < krem && ex + v >= krem) { sh_bin = 255 - tid; sh_excl = ex; }
                __syncthreads();
                prefix |= (uint32_t)sh_bin << shift;
                pmask |= 0xffu << shift;
                krem -= sh_excl;
            }
            thr = prefix;
            need_eq = krem;
        }
        // index-ordered compaction: key > thr, or key == thr among the first
        // need_eq
        int my_eq = 0, my_gt = 0;
        if (k > 0)
            for (int r = 0; r < kpt; ++r) {
                const uint32_t key = c0 + r < nb ? keys[c0 + r] : 0u;
                my_eq += key != 0 && key == thr;
                my_gt += key != 0 && key > thr;
            }
        int tot;
        const int eq_base = cta_excl_sum(my_eq, tmp, &tot);
        const int my_take = my_gt + min(my_eq, max(0, need_eq - eq_base));
        int p = cta_excl_sum(my_take, tmp, &tot);
        if (tid == 0) n_sel_sh = tot;
        if (my_take > 0) {
            int eq_seen = eq_base;
            for (int r = 0; r < kpt && c0 + r < nb; ++r) {
                const uint32_t key = keys[c0 + r];
                if (key != 0 && key > thr) sel[p++] = c0 + r;
                else if (key != 0 && key == thr && eq_seen++ < need_eq) sel[p++] = c0 + r;
            }
        }
    }
    __syncthreads();
    const int n_sel = n_sel_sh;

    for (int i = tid; i < n_sel; i += kPickThreads) a.sel_blocks[(int64_t)s * a.max_sel + i] = sel[i];

    // ---- ranges.  Merge the forced ranges and the selected blocks' ranges
    // (both ascending; on equal starts the forced range comes first) ...
    const int m = n_sel + nf;
    for (int i = tid; i < n_sel; i += kPickThreads) {
        const int jj = sel[i];
        int lo, hi;
        if (off) { lo = min(max(off[jj], 0), a.L_max); hi = lo + visb[jj]; }
        else { lo = jj * a.S; hi = lo + a.S; }
        int before = 0;
        for (int f = 0; f < nf; ++f) before += f_lo[f] <= lo;
        mrg[i + before] = make_int2(lo, hi);
    }
    if (tid < nf) {
        const int lo = f_lo[tid];
        int a0 = 0, a1 = n_sel;   // selected blocks starting strictly before lo
        while (a0 < a1) {
            const int mid = (a0 + a1) >> 1;
            const int blo = off ? min(max(off[sel[mid]], 0), a.L_max) : sel[mid] * a.S;
            if (blo < lo) a0 = mid + 1; else a1 = mid;
        }
        mrg[tid + a0] = make_int2(lo, f_hi[tid]);
    }
    __syncthreads();
    // ... then the running maximum of the ends: item i opens a new range when
    // it starts after every earlier item has ended; a range ends at the
    // running maximum of its last item.
    int carry = kIntMin;
    for (int t0 = 0; t0 < m; t0 += kPickThreads) {
        const int i = t0 + tid;
        int tot;
        const int pm = max(cta_incl_max(i < m ? mrg[i].y : kIntMin, tmp, &tot), carry);
        if (i < m) pmax[i] = pm;
        carry = max(carry, tot);
    }
    __syncthreads();
    int32_t *R = a.ranges + (int64_t)s * a.max_ranges * 2;
    int nr = 0;
    for (int t0 = 0; t0 < m; t0 += kPickThreads) {
        const int i = t0 + tid;
        const int start = i < m && (i == 0 || mrg[i].x > pmax[i - 1]);
        int tot;
        const int rid = nr + cta_excl_sum(start, tmp, &tot) + start - 1;   // range of item i
        if (i < m) {
            if (start && rid < a.max_ranges) R[2 * rid] = mrg[i].x;
            const bool last = i == m - 1 || mrg[i + 1].x > pmax[i];
            if (last && rid < a.max_ranges) R[2 * rid + 1] = pmax[i];
        }
        nr += tot;
    }
    if (tid == 0) {
        a.n_ranges[s] = min(nr, a.max_ranges);
        a.sel_count[s] = n_sel;
    }
}


// The same selection for fixed blocks, segments of at most 128 * NK blocks,
// by one 128-thread CTA per segment: thread t holds the keys of blocks
// [t NK, t NK + NK) in registers, so the threads' runs are in index order.
// The k-th largest key T is found bit by bit from the top: T gains bit b when
// at least k candidate keys are >= T | b (a warp count, then the four warps'
// counts through shared memory: one barrier per bit, the counts double-
// buffered by bit parity).  The selected blocks are those with key > T and,
// among the keys equal to T, the k - count(> T) of lowest index; exclusive
// scans over the threads give each taken block its place in index order and
// among the forced ranges, and the merged ranges come from scans of the
// running maximum of the ends.  Shared memory: (lo, hi) of max_sel + 2
// items and their running maxima.
constexpr int kPickFixedThreads = 128;

template <int NK>
__global__ void __launch_bounds__(kPickFixedThreads) pick_fixed_kernel(SelArgs a) {
    extern __shared__ __align__(16) unsigned char psm[];
    int2 *items = reinterpret_cast<int2 *>(psm);
    int *pmax = reinterpret_cast<int *>(psm + (size_t)(a.max_sel + 4) * 8);
    __shared__ int cnt2[2][kPickFixedThreads / 32];
    __shared__ int tmp[40];
    const int s = blockIdx.x, b = s / a.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nb = a.nb_total, j0 = tid * NK;
    pdl_wait();   // keys from score_kernel
    uint32_t wk[NK];
#pragma unroll
    for (int r = 0; r < NK; ++r) wk[r] = j0 + r < nb ? a.keys[(int64_t)s * nb + j0 + r] : 0u;
    // forced token ranges (every thread computes the same), sorted and merged
    const int n = min(max(a.cur_len[b], 0), a.L_max);
    int f_lo[2] = {0, 0}, f_hi[2] = {0, 0}, nf = 0;
    if (a.sink > 0 && n > 0) { f_lo[0] = 0; f_hi[0] = min(a.sink, n); nf = 1; }
    {
        int t0 = n;
        if (a.window > 0) t0 = min(t0, max(0, n - a.window));
        if (a.keep_current && n > 0) t0 = min(t0, ((n - 1) / a.S) * a.S);
        if (t0 < n) {
            if (nf > 0 && t0 <= f_hi[0]) f_hi[0] = n;
            else if (nf == 0) { f_lo[0] = t0; f_hi[0] = n; nf = 1; }
            else { f_lo[1] = t0; f_hi[1] = n; nf = 2; }
        }
    }
    // candidates: keys > 0 and not wholly inside the forced set
    int my_c = 0;
#pragma unroll
    for (int r = 0; r < NK; ++r) {
        if (wk[r]) {
            const int64_t r0 = (int64_t)(j0 + r) * a.S, r1 = r0 + a.S;
#pragma unroll
            for (int i = 0; i < 2; ++i)
                if (i < nf && f_lo[i] <= r0 && r1 <= f_hi[i]) wk[r] = 0u;
        }
        my_c += wk[r] != 0u;
    }
    // CTA sum through the parity-buffered warp counts (one barrier each)
    int par = 0;
    auto cta_sum = [&](int v) -> int {
        v = __reduce_add_sync(0xffffffffu, v);
        if (lane == 0) cnt2[par][warp] = v;
        __syncthreads();
        int t = 0;
#pragma unroll
        for (int w = 0; w < kPickFixedThreads / 32; ++w) t += cnt2[par][w];
        par ^= 1;
        return t;
    };
    const int n_cand = cta_sum(my_c);
    const int k = min(min(a.topk >= 0 ? a.topk : a.budget / a.S, n_cand), a.max_sel);
    uint32_t taken = 0;   // bit r: block j0 + r
    if (k > 0) {
        // T = the k-th largest candidate key (>= 1, since k <= n_cand)
        uint32_t T = 0u;
        for (int bit = 31; bit >= 0; --bit) {
            const uint32_t c = T | (1u << bit);
            int cnt = 0;
#pragma unroll
            for (int r = 0; r < NK; ++r) cnt += wk[r] >= c;
            if (cta_sum(cnt) >= k) T = c;
        }
        int gt = 0, eq = 0;
#pragma unroll
        for (int r = 0; r < NK; ++r) {
            gt += wk[r] > T;
            eq += wk[r] == T;
        }
        const int need_eq = k - cta_sum(gt);
        int tot;
        int eq_rank = cta_excl_sum(eq, tmp, &tot);   // keys equal to T before this thread's
#pragma unroll
        for (int r = 0; r < NK; ++r)
            if (wk[r] > T || (wk[r] == T && eq_rank++ < need_eq)) taken |= 1u << r;
    }
    // index-ordered compaction, each block written at its place among the
    // forced ranges (a forced range comes first on equal starts)
    int tot;
    int p = cta_excl_sum(__popc(taken), tmp, &tot);
    const int n_sel = min(tot, a.max_sel);
    int below[2] = {0, 0};   // taken blocks starting before f_lo[f]
#pragma unroll
    for (int r = 0; r < NK; ++r) {
        if ((taken >> r) & 1u) {
            const int jj = j0 + r;
            const int lo = jj * a.S, hi = lo + a.S;
            int before = 0;
#pragma unroll
            for (int f = 0; f < 2; ++f) {
                before += f < nf && f_lo[f] <= lo;
                below[f] += f < nf && lo < f_lo[f];
            }
            if (p < a.max_sel) {
                a.sel_blocks[(int64_t)s * a.max_sel + p] = jj;
                items[p + before] = make_int2(lo, hi);
            }
            ++p;
        }
    }
#pragma unroll
    for (int f = 0; f < 2; ++f) {
        const int nbelow = cta_sum(below[f]);
        if (f < nf && tid == 0) items[f + nbelow] = make_int2(f_lo[f], f_hi[f]);
    }
    __syncthreads();
    // ranges: item i opens a range when it starts after every earlier item
    // has ended; a range ends at the running maximum of its last item
    const int M = n_sel + nf;
    int carry = kIntMin;
    for (int t0 = 0; t0 < M; t0 += kPickFixedThreads) {
        const int i = t0 + tid;
        const int pm = max(cta_incl_max(i < M ? items[i].y : kIntMin, tmp, &tot), carry);
        if (i < M) pmax[i] = pm;
        carry = max(carry, tot);
    }
    __syncthreads();
    int32_t *R = a.ranges + (int64_t)s * a.max_ranges * 2;
    int nr = 0;
    for (int t0 = 0; t0 < M; t0 += kPickFixedThreads) {
        const int i = t0 + tid;
        const int start = i < M && (i == 0 || items[i].x > pmax[i - 1]);
        const int rid = nr + cta_excl_sum(start, tmp, &tot) + start - 1;   // range of item i
        if (i < M) {
            if (start && rid < a.max_ranges) R[2 * rid] = items[i].x;
            const bool last = i == M - 1 || items[i + 1].x > pmax[i];
            if (last && rid < a.max_ranges) R[2 * rid + 1] = pmax[i];
        }
        nr += tot;
    }
    if (tid == 0) {
        a.n_ranges[s] = min(nr, a.max_ranges);
        a.sel_count[s] = n_sel;
    }
}

bsa_status launch_select(const bsa_kv_desc *d, const float *q, const void *summ, int kind,
                         const bsa_sel_params *p, const int32_t *cur_len, int nb_total,
                         int max_sel, int32_t *sel_blocks, int32_t *sel_count, int max_ranges,
                         int32_t *ranges, int32_t *n_ranges, uint32_t *keys, int32_t *vis,
                         uint32_t *counters, uint32_t *status, cudaStream_t st) {
    (void)counters;
    SelArgs a;
    a.q = q; a.cur_len = cur_len;
    const bool variable = p->block_size == 0;
    a.offsets = variable ? p->block_offsets : nullptr;
    a.kv_pos = variable ? p->kv_pos : nullptr;
    a.sel_blocks = sel_blocks; a.sel_count = sel_count; a.ranges = ranges; a.n_ranges = n_ranges;
    a.keys = keys; a.vis = vis; a.counters = counters; a.status = status;
    a.B = d->B; a.Hq = d->Hq; a.Hkv = d->Hkv; a.G = d->Hq / d->Hkv; a.D = d->D;
    a.L_max = d->L_max; a.S = p->block_size; a.nb_total = nb_total;
    a.topk = p->topk; a.budget = p->budget_tokens; a.sink = p->sink; a.window = p->window;
    a.keep_current = p->keep_current_block; a.local_start = p->local_start;
    a.pos_limit = p->pos_limit; a.max_sel = max_sel; a.max_ranges = max_ranges;
    const bool bf = kind == BSA_SUM_MINMAX && d->kv_dtype != BSA_F32;   // bf16 bounds (FP8: exact)
    const int esz = bf ? 2 : 4;
    const int cols = kind == BSA_SUM_MINMAX ? 2 * d->D : d->D;
    a.row_bytes = cols * esz;
    a.nbox = a.row_bytes / 128;
    // two rows per thread where the group size and head_dim allow
    const bool pair = (kind != BSA_SUM_MINMAX || bf) && (d->D == 64 || d->D == 128) &&
                      (a.G == 4 || a.G == 8 || a.G == 16);
    const int tile_rows = pair ? kPairRows : kSelThreads;
    a.tile_bytes = (uint32_t)(a.nbox * tile_rows * 128);
    const size_t qbytes = (size_t)a.G * (d->D + 4) * 4;
    const size_t cap = 227 * 1024 - 1024;
    a.nst = (int)std::min<size_t>(pair ? BSA_SCORE_PAIR_STAGES : kScoreStages,
                                  (cap - qbytes) / (a.tile_bytes + qbytes));
    if (a.nst < 1) return BSA_ERR_UNSUPPORTED;
    const size_t smem1 = pair ? pair_smem_bytes(a.nst, a.tile_bytes, qbytes)
                              : 1024 + (size_t)a.nst * (a.tile_bytes + qbytes) + qbytes;   // + selectors
    const size_t smem2 = PickSmem::bytes(nb_total, max_sel);
    if (smem2 > cap) return BSA_ERR_UNSUPPORTED;
    a.tiles_per_seg = (int)div_up(nb_total, tile_rows);
    const int nseg = d->B * d->Hkv;
    a.n_items = nseg * a.tiles_per_seg;
    CUtensorMap tm;
    if (!make_rows_tmap(&tm, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                        esz, summ, cols, (int64_t)nseg * nb_total, a.row_bytes, tile_rows))
        return BSA_ERR_CUDA;
    auto launch = [&](auto kern, int threads) -> bsa_status {
        BSA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1));
        int per_sm = 0;
        BSA_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem1));
        const int grid = std::max(1, std::min(a.n_items, num_sms() * std::max(per_sm, 1)));
        BSA_CUDA_TRY(launch_pdl(kern, dim3(grid), dim3(threads), smem1, st, tm, a));
        return BSA_OK;
    };
    auto by_gd = [&](auto sk, auto dt) -> bsa_status {
        constexpr int SK = decltype(sk)::value, DT = decltype(dt)::value;
        if constexpr (SK != kScoreMinmaxF32 && DT > 0) {   // two rows per thread
            if (pair) switch (a.G) {
                case 4: return launch(score_pair_kernel<SK, 4, DT>, kPairRows);
                case 8: return launch(score_pair_kernel<SK, 8, DT>, kPairRows);
                case 16: return launch(score_pair_kernel<SK, 16, DT>, kPairRows);
                default: break;
            }
        }
        switch (a.G) {
            case 1: return launch(score_kernel<SK, 1, DT>, kSelThreads * score_tpb(1));
            case 2: return launch(score_kernel<SK, 2, DT>, kSelThreads * score_tpb(2));
            case 4: return launch(score_kernel<SK, 4, DT>, kSelThreads * score_tpb(4));
            case 8: return launch(score_kernel<SK, 8, DT>, kSelThreads * score_tpb(8));
            case 16: return launch(score_kernel<SK, 16, DT>, kSelThreads * score_tpb(16));
            default: return launch(score_kernel<SK, 0, 0>, kSelThreads * score_tpb(0));
        }
    };
    auto by_g = [&](auto sk) -> bsa_status {
        if (d->D == 128) return by_gd(sk, std::integral_constant<int, 128>());
        if (d->D == 64) return by_gd(sk, std::integral_constant<int, 64>());
        return by_gd(sk, std::integral_constant<int, 0>());
    };
    bsa_status r;
    if (kind == BSA_SUM_MINMAX)
        r = bf ? by_g(std::integral_constant<int, kScoreMinmaxBf16>())
               : by_g(std::integral_constant<int, kScoreMinmaxF32>());
    else
        r = by_g(std::integral_constant<int, kScoreCentroid>());
    if (r != BSA_OK) return r;
    auto pick = [&](auto kern) -> bsa_status {
        BSA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2));
        BSA_CUDA_TRY(launch_pdl(kern, dim3((unsigned)nseg), dim3(kPickThreads), smem2, st, a));
        return BSA_OK;
    };
    // fixed blocks, up to 4,096 per segment: 128 threads per segment with
    // the keys in registers (the token-budget walk over variable blocks
    // measured faster in the 512-thread kernel)
    if (!variable && nb_total <= kPickFixedThreads * 32) {
        const size_t smem3 = (size_t)(max_sel + 4) * 12;
        auto fixed_pick = [&](auto kern) -> bsa_status {
            BSA_CUDA_TRY(launch_pdl(kern, dim3((unsigned)nseg), dim3(kPickFixedThreads), smem3, st, a));
            return BSA_OK;
        };
        if (nb_total <= kPickFixedThreads * 4) return fixed_pick(pick_fixed_kernel<4>);
        if (nb_total <= kPickFixedThreads * 8) return fixed_pick(pick_fixed_kernel<8>);
        if (nb_total <= kPickFixedThreads * 12) return fixed_pick(pick_fixed_kernel<12>);
        if (nb_total <= kPickFixedThreads * 16) return fixed_pick(pick_fixed_kernel<16>);
        return fixed_pick(pick_fixed_kernel<32>);
    }
    return pick(pick_kernel);
}

}  // namespace bsa
