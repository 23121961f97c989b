// A4 (split-K sparse decode over the selected token ranges) + A5 (log-sum-exp
// merge), sm_100a.
//
// out_h = sum_j softmax_j(scale * q_h . k_j) v_j over the selected rows
// ("Module 14: Sparse attention and long context", Exercise 14.1, restricted
// to the selected set), GQA: query head h reads KV head h / G.
//
// Work decomposition.  A segment's ranges are cut into pieces of 16 rows
// (one TMA box row-block each; a range's last piece may be short).  The
// pieces are split evenly over `nsplit` CTAs; inside a CTA, warp w takes the
// pieces w, w+4, w+8, ... and streams them through its own shared-memory ring
// (lane 0 issues the loads, one mbarrier per stage, no CTA-wide barrier in
// the loop).  Each CTA combines its warps and writes an unnormalised partial
// (m, l, o) in base 2; lse_merge_kernel, launched as a programmatic dependent
// of the decode grid, merges the partials in split order, so the result does
// not depend on scheduling.  With one split the decode writes the output.
//
// Tensor-core path (bf16 K/V, D in {64, 128}, G <= 8): pieces arrive by 4-D
// tiled TMA loads with 128-byte swizzle (no multicast).  All G query heads of
// the group share every K/V byte: the 16 MMA rows hold q_hi (rows 0-7) and
// q_lo = q - q_hi (rows 8-15), so one m16n8k16 bf16 MMA gives the logits to
// ~2^-17 relative; the softmax weights are split the same way for P.V.
// Accumulation is fp32.
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include "summary_rows.cuh"

namespace bsa {

constexpr int kPiece = 16;
constexpr int kDecWarps = 4;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kBoxBytes = kPiece * 128;            // 16 rows x 64 bf16
constexpr int kWarpCap = 128;                      // per-warp piece table (refilled when exceeded)
constexpr int kRegRanges = 12;                     // range slots per lane loaded in one batch
constexpr int kMaxClusterSplits = 16;              // splits merged inside one cluster
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kNegInf = -__builtin_huge_valf();

struct DecArgs {
    const float *q;
    float *out, *lse;
    const int32_t *ranges, *n_ranges;
    int max_ranges;
    const int32_t *cur_len;
    const void *K, *V;
    KvRows rows;          // where each logical row lives (contiguous or paged)
    int B, Hq, Hkv, G, D, L_max, nsplit;
    float scale_log2;
    float *part_o;        // [nseg][nsplit][G][D]
    float2 *part_ml;      // [nseg][nsplit][G]
    uint32_t *counters;   // [nseg]; entry b * Hkv counts the CTAs of sequence b (fused append)
    uint32_t *status;     // sticky error bits
    uint32_t stall_ns;    // test hook: a wait of this bound on a barrier nothing completes
    DecAppend app;
};

// Limit of the test stall armed for the next decode launch (0: none).
static std::atomic<uint32_t> g_armed_stall_ns{0};

void arm_decode_wait_limit(uint32_t limit_ns) { g_armed_stall_ns.store(limit_ns); }

// Exclusive scan over the CTA (blockDim.x a multiple of 32, <= 1024).
__device__ __forceinline__ int block_excl_scan(int v, int *tmp, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? tmp[lane] : 0, wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            int t = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += t;
        }
        if (lane < nw) tmp[lane] = wi - w;
        if (lane == 31) tmp[32] = wi;
    }
    __syncthreads();
    int res = incl - v + tmp[warp];
    *total = tmp[32];
    __syncthreads();
    return res;
}

// Loads segment s's ranges (clamped to [0, L_max), the last extended to
// cur_len) and the prefix of their 16-row piece counts.  Returns the number
// of pieces; *nr_out the number of ranges.
__device__ int load_ranges(const DecArgs &a, int s, int b, int *rs, int *re, int *ps, int *tmp,
                           int *nr_out) {
    // One round trip: the count, the length and every slot of the range table
    // are requested together (slots past the count are ignored).
    const int32_t *R = a.ranges + (int64_t)s * a.max_ranges * 2;
    const int nr_raw = a.n_ranges[s];
    const int cl_raw = a.cur_len[b];
    for (int r = threadIdx.x; r < a.max_ranges; r += blockDim.x) {
        const int2 v = *reinterpret_cast<const int2 *>(R + 2 * r);
        rs[r] = v.x;
        re[r] = v.y;
    }
    const int nr = min(max(nr_raw, 0), a.max_ranges);
    const int cl = min(max(cl_raw, 0), a.L_max);
    int carry = 0;
    for (int base = 0; base < nr; base += blockDim.x) {
        const int r = base + threadIdx.x;
        int cnt = 0;
        if (r < nr) {
            int lo = min(max(rs[r], 0), a.L_max);
            int hi = min(max(re[r], lo), a.L_max);
            if (r == nr - 1 && cl > hi) hi = cl;
            rs[r] = lo;
            re[r] = hi;
            cnt = (hi - lo + kPiece - 1) / kPiece;
        }
        int tot;
        int ex = block_excl_scan(cnt, tmp, &tot);
        if (r < nr) ps[r] = carry + ex;
        carry += tot;
    }
    *nr_out = nr;
    __syncthreads();
    return carry;
}

// A range slot of segment s, clamped to [0, L_max); the last range is
// extended to the sequence length cl.
__device__ __forceinline__ int2 clamp_range(const DecArgs &a, int2 v, bool last, int cl) {
    const int lo = min(max(v.x, 0), a.L_max);
    int hi = min(max(v.y, lo), a.L_max);
    if (last && cl > hi) hi = cl;
    return make_int2(lo, hi);
}

// 16-row pieces of range x.  A contiguous cache cuts the range from its
// start; a paged pool cuts it at multiples of 16 rows so that no piece
// straddles a page (the first and last pieces may then use part of their
// 16-row box).
template <bool AL>
__device__ __forceinline__ int piece_count(int2 x) {
    if (x.y <= x.x) return 0;
    return AL ? (x.y + kPiece - 1) / kPiece - x.x / kPiece : (x.y - x.x + kPiece - 1) / kPiece;
}

// Piece q of range x: (first row of its 16-row box, valid rows lo | hi << 8
// of the box).
template <bool AL>
__device__ __forceinline__ int2 piece_of(int2 x, int q) {
    if constexpr (AL) {
        const int row = (x.x / kPiece + q) * kPiece;
        return make_int2(row, max(x.x - row, 0) | (min(x.y - row, kPiece) << 8));
    }
    const int row = x.x + q * kPiece;
    return make_int2(row, min(kPiece, x.y - row) << 8);
}

// Warp-local view of a segment's range table (no CTA-wide barrier): lane l
// owns the slots [r0, r1) = [l k, l k + k), k = ceil(max_ranges / 32), and
// pbase is the number of 16-row pieces in the slots before r0.  The CTA's
// pieces are [first, last); this warp streams first + warp + 4 i.
struct WarpRanges {
    const int32_t *R;
    int nr, cl, r0, r1, pbase, P, first, last;
    int app;   // row the fused append writes (then cl = app + 1), or -1
};

// Writes the table entries of range x (first piece pp) for warp-local
// indices i in [i0, i0 + kWarpCap): (box row, valid rows, TMA row coordinate,
// TMA outer coordinate); a paged pool's coordinates are filled in by
// warp_translate.
template <bool AL>
__device__ __forceinline__ void fill_range(const WarpRanges &w, int2 x, int pp, int warp, int i0,
                                           int b, int4 *tab) {
    const int cnt = piece_count<AL>(x);
    const int lo_p = pp - w.first - warp;                       // i >= ceil(lo_p / 4)
    const int hi_p = min(pp + cnt, w.last) - w.first - warp;    // i <  ceil(hi_p / 4)
    const int ia = max(lo_p > 0 ? (lo_p + kDecWarps - 1) / kDecWarps : 0, i0);
    const int ib = min(hi_p > 0 ? (hi_p + kDecWarps - 1) / kDecWarps : 0, i0 + kWarpCap);
    for (int i = ia; i < ib; ++i) {
        const int2 pr = piece_of<AL>(x, w.first + warp + kDecWarps * i - pp);
        tab[i - i0] = make_int4(pr.x, pr.y, pr.x, b);
    }
}

// Paged pool: the TMA coordinates (row in page, page) of the table entries
// [0, n), looked up in the sequence's page table by all lanes together.  An
// entry outside the pool gives an out-of-bounds box, which reads zeros.
__device__ __forceinline__ void warp_translate(const DecArgs &a, int b, int lane, int n, int4 *tab) {
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
        int4 e = tab[i];
        e.z = e.x % a.rows.P;
        e.w = __ldg(a.rows.table + (int64_t)b * a.rows.pps + e.x / a.rows.P);
        tab[i] = e;
    }
}

template <bool AL>
__device__ __forceinline__ void warp_refill(const DecArgs &a, const WarpRanges &w, int warp, int i0,
                                            int b, int4 *tab);

// Scans the range table and fills the first window of this warp's piece
// table (the caller syncs the warp before reading it).  AL: pieces cut at
// multiples of 16 rows (paged pools).
template <bool AL>
__device__ __forceinline__ WarpRanges warp_ranges(const DecArgs &a, int s, int b, int c, int warp,
                                                  int lane, int4 *tab) {
    WarpRanges w;
    w.R = a.ranges + (int64_t)s * a.max_ranges * 2;
    const int k = (a.max_ranges + 31) >> 5;
    w.r0 = min(lane * k, a.max_ranges);
    w.r1 = min(w.r0 + k, a.max_ranges);
    const int2 *R2 = reinterpret_cast<const int2 *>(w.R);
    // one round trip: the count, the length and this lane's slots together
    int2 rv[kRegRanges];
#pragma unroll
    for (int j = 0; j < kRegRanges; ++j) rv[j] = w.r0 + j < w.r1 ? __ldg(R2 + w.r0 + j) : make_int2(0, 0);
    w.nr = min(max(a.n_ranges[s], 0), a.max_ranges);
    const int len = a.cur_len[b];
    w.app = a.app.k_new && len >= 0 && len < a.L_max ? len : -1;
    w.cl = w.app >= 0 ? len + 1 : min(max(len, 0), a.L_max);
    const int end = min(w.r1, w.nr);
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < kRegRanges; ++j) {
        rv[j] = clamp_range(a, rv[j], w.r0 + j == w.nr - 1, w.cl);
        if (w.r0 + j < end) cnt += piece_count<AL>(rv[j]);
    }
    for (int r = w.r0 + kRegRanges; r < end; ++r) {
        const int2 x = clamp_range(a, __ldg(R2 + r), r == w.nr - 1, w.cl);
        cnt += piece_count<AL>(x);
    }
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
    }
    w.pbase = incl - cnt;
    w.P = __shfl_sync(0xffffffffu, incl, 31);
    int per = (w.P + a.nsplit - 1) / a.nsplit;
    per = (per + kDecWarps - 1) / kDecWarps * kDecWarps;
    w.first = min(c * per, w.P);
    w.last = min(w.P, w.first + per);
    // the first window, from the same slots (now in L1) in a rolled loop: this
    // code runs once per warp, so it stays short
    warp_refill<AL>(a, w, warp, 0, b, tab);
    return w;
}

// Fills the table with the window i in [i0, i0 + kWarpCap).
template <bool AL>
__device__ __forceinline__ void warp_refill(const DecArgs &a, const WarpRanges &w, int warp, int i0,
                                            int b, int4 *tab) {
    int pp = w.pbase;
    const int end = min(w.r1, w.nr);
#pragma unroll 1
    for (int r = w.r0; r < end && pp < w.last; ++r) {
        const int2 x = clamp_range(a, __ldg(reinterpret_cast<const int2 *>(w.R) + r), r == w.nr - 1, w.cl);
        fill_range<AL>(w, x, pp, warp, i0, b, tab);
        pp += piece_count<AL>(x);
    }
}

// Piece p -> (first row, valid rows).
__device__ __forceinline__ int2 piece_rows(int p, const int *rs, const int *re, const int *ps,
                                           int nr) {
    int lo = 0, hi = nr - 1;
    while (lo < hi) {   // largest r with ps[r] <= p
        int mid = (lo + hi + 1) >> 1;
        if (ps[mid] <= p) lo = mid; else hi = mid - 1;
    }
    int row = rs[lo] + (p - ps[lo]) * kPiece;
    return make_int2(row, min(kPiece, re[lo] - row));
}

// Combines the per-warp partials (wm, wl, wo) of this CTA and writes either
// the final output (nsplit == 1) or the split's partial for the merge kernel.
__device__ void finish(const DecArgs &a, int s, int b, int g, int c, const float *wm,
                       const float *wl, const float *wo, float *sml /* [2*kMaxG] */) {
    const int G = a.G, D = a.D;
    if (threadIdx.x < G) {
        const int h = threadIdx.x;
        float M = kNegInf;
        for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, wm[w * kMaxG + h]);
        float L = 0.0f;
        for (int w = 0; w < kDecWarps; ++w) {
            float mw = wm[w * kMaxG + h];
            if (mw != kNegInf) L += wl[w * kMaxG + h] * exp2f(mw - M);
        }
        sml[2 * h] = M;
        sml[2 * h + 1] = L;
    }
    __syncthreads();
    const int64_t qrow = (int64_t)b * a.Hq + (int64_t)g * G;
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
        const int h = e / D, d = e % D;
        const float M = sml[2 * h];
        float O = 0.0f;
        for (int w = 0; w < kDecWarps; ++w) {
            float mw = wm[w * kMaxG + h];
            if (mw != kNegInf) O += wo[(w * kMaxG + h) * D + d] * exp2f(mw - M);
        }
        if (a.nsplit == 1) {
            const float L = sml[2 * h + 1];
            a.out[(qrow + h) * D + d] = L > 0.0f ? O / L : 0.0f;
            if (d == 0 && a.lse) a.lse[qrow + h] = L > 0.0f ? (M + log2f(L)) * kLn2 : kNegInf;
        } else {
            a.part_o[(((int64_t)s * a.nsplit + c) * G + h) * D + d] = O;
            if (d == 0) a.part_ml[((int64_t)s * a.nsplit + c) * G + h] = make_float2(M, sml[2 * h + 1]);
        }
    }
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}

// Reads from the shared memory of CTA `rank` of this cluster at the address
// `local` has in this CTA.
__device__ __forceinline__ float ld_peer(uint32_t local, uint32_t rank) {
    uint32_t remote;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}
__device__ __forceinline__ float2 ld_peer2(uint32_t local, uint32_t rank) {
    uint32_t remote;
    float2 v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
    asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(remote) : "memory");
    return v;
}

// The split-K merge inside a thread-block cluster (the segment's splits):
// every CTA leaves its partial (m, l per head in sml, o in `part`) in its own
// shared memory; after a cluster barrier each CTA merges a slice of the
// output elements reading its peers' partials through distributed shared
// memory, in split order; a second barrier keeps the partials alive until
// every peer has read them.  All threads of all CTAs reach both barriers.
__device__ void cluster_finish(const DecArgs &a, int b, int g, const float *wm, const float *wl,
                               const float *wo, float *sml, float *part) {
    const int G = a.G, D = a.D;
    if (threadIdx.x < G) {
        const int h = threadIdx.x;
        float M = kNegInf;
        for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, wm[w * kMaxG + h]);
        float L = 0.0f;
        for (int w = 0; w < kDecWarps; ++w) {
            const float mw = wm[w * kMaxG + h];
            if (mw != kNegInf) L += wl[w * kMaxG + h] * exp2f(mw - M);
        }
        sml[2 * h] = M;
        sml[2 * h + 1] = L;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
        const int h = e / D, d = e % D;
        const float M = sml[2 * h];
        float O = 0.0f;
        for (int w = 0; w < kDecWarps; ++w) {
            const float mw = wm[w * kMaxG + h];
            if (mw != kNegInf) O += wo[(w * kMaxG + h) * D + d] * exp2f(mw - M);
        }
        part[e] = O;
    }
    cluster_sync_all();
    const uint32_t rank = cluster_ctarank(), n = (uint32_t)a.nsplit;
    const uint32_t sml_a = smem_u32(sml), part_a = smem_u32(part);
    const int64_t qrow = (int64_t)b * a.Hq + (int64_t)g * G;
    for (int e = rank * blockDim.x + threadIdx.x; e < G * D; e += n * blockDim.x) {
        const int h = e / D, d = e % D;
        // all of the peers' values are requested before any is used
        float2 mlk[kMaxClusterSplits];
        float ok[kMaxClusterSplits];
#pragma unroll
        for (uint32_t k = 0; k < (uint32_t)kMaxClusterSplits; ++k)
            if (k < n) {
                mlk[k] = ld_peer2(sml_a + 8 * h, k);
                ok[k] = ld_peer(part_a + 4 * e, k);
            }
        float m = kNegInf, l = 0.0f, o = 0.0f;
#pragma unroll
        for (uint32_t k = 0; k < (uint32_t)kMaxClusterSplits; ++k)
            if (k < n && mlk[k].x != kNegInf) {
                const float mn = fmaxf(m, mlk[k].x);
                const float c_old = exp2f(m - mn), c_new = exp2f(mlk[k].x - mn);
                l = l * c_old + mlk[k].y * c_new;
                o = o * c_old + ok[k] * c_new;
                m = mn;
            }
        a.out[(qrow + h) * D + d] = l > 0.0f ? o / l : 0.0f;
        if (d == 0 && a.lse) a.lse[qrow + h] = l > 0.0f ? (m + log2f(l)) * kLn2 : kNegInf;
    }
    // the partials stay alive until every peer has read them; the values read
    // were consumed above, so this barrier orders no memory
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}

// Log-sum-exp merge of the split partials (A5), one CTA per (segment, query
// head), one thread per output element.  Launched as a programmatic
// dependent of the decode kernel: it waits for the decode grid to complete
// (and its writes to be visible) before reading the partials, so its launch
// overlaps the decode's tail.  Splits are merged in split order.
__global__ void __launch_bounds__(128) lse_merge_kernel(DecArgs a) {
    pdl_wait();
    const int s = blockIdx.x, h = blockIdx.y, G = a.G, D = a.D;
    const int b = s / a.Hkv, g = s % a.Hkv;
    const float2 *pml = a.part_ml + (int64_t)s * a.nsplit * G + h;
    const float *po = a.part_o + ((int64_t)s * a.nsplit * G + h) * D;
    const int64_t qrow = (int64_t)b * a.Hq + (int64_t)g * G + h;
    // Every thread merges its output element over the splits in split order
    // with a running maximum; all loads are independent of one another.
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
        float m = kNegInf, l = 0.0f, o = 0.0f;
#pragma unroll 16
        for (int k = 0; k < a.nsplit; ++k) {
            const float2 ml = __ldcg(&pml[(int64_t)k * G]);
            const float ov = __ldcg(&po[(int64_t)k * G * D + d]);
            if (ml.x != kNegInf) {
                const float mn = fmaxf(m, ml.x);
                const float c_old = exp2f(m - mn), c_new = exp2f(ml.x - mn);
                l = l * c_old + ml.y * c_new;
                o = o * c_old + ov * c_new;
                m = mn;
            }
        }
        a.out[qrow * D + d] = l > 0.0f ? o / l : 0.0f;
        if (d == 0 && a.lse) a.lse[qrow] = l > 0.0f ? (m + log2f(l)) * kLn2 : kNegInf;
    }
}

// End of a fused step for one CTA of segment (b, g): the CTA that wrote row n
// builds the summary of the fixed block that row completes; the last CTA of
// sequence b to get here (every CTA of it has read cur_len by then) sets
// cur_len[b] = n + 1 and resets the counter.
template <typename T>
__device__ __forceinline__ void finish_append(const DecArgs &a, int b, int g, int n, bool owner) {
    if (n < 0) return;
    const DecAppend &p = a.app;
    if (owner && p.summ && p.S > 0 && (n + 1) % p.S == 0) {
        const int j = (n + 1) / p.S - 1;
        const T *K = static_cast<const T *>(a.K);
        char *out = static_cast<char *>(p.summ) + ((int64_t)(b * a.Hkv + g) * p.nb_total + j) * p.row_bytes;
        if (p.kind == BSA_SUM_MINMAX)
            summarize_minmax<T>(K, a.rows, b, g, a.D, (int64_t)j * p.S, (int64_t)(j + 1) * p.S,
                                reinterpret_cast<minmax_t<T> *>(out));
        else
            summarize_centroid<T>(K, a.rows, b, g, a.D, (int64_t)j * p.S, (int64_t)(j + 1) * p.S,
                                  reinterpret_cast<float *>(out));
    }
    if (threadIdx.x == 0) {
        __threadfence();
        uint32_t *ctr = a.counters + b * a.Hkv;
        if (atomicAdd(ctr, 1u) == (uint32_t)(a.Hkv * gridDim.x) - 1u) {
            p.cur_len[b] = n + 1;
            *ctr = 0u;
        }
    }
}

// ======================================================================
// Tensor-core path
// ======================================================================
// Shared memory: one ring per warp, NST stages of one piece each (K then V:
// NH boxes of 16 rows x 64 bf16 columns apiece, or for an FP8 cache one box
// of 16 rows x 128 FP8 columns apiece), then for an FP8 cache one f16 V box
// per warp (the bf16 layout) that each stage's V is widened into.
template <int NH, int NST, bool F8 = false>
struct TcSmem {
    static constexpr int kPieceBytes = F8 ? 2 * kBoxBytes : 2 * NH * kBoxBytes;
    static constexpr int kRing = kDecWarps * NST * kPieceBytes;
    static constexpr int kConv = kRing;                               // FP8: f16 V [warps]
    static constexpr int kConvBytes = F8 ? kDecWarps * NH * kBoxBytes : 0;
    static constexpr int kInfo = kConv + kConvBytes;                  // int [warps][NST], 8-B slots
    static constexpr int kBars = kInfo + kDecWarps * NST * 8;         // u64  [warps][NST]
    static constexpr int kMisc = kBars + kDecWarps * NST * 8;         // float sml[2*kMaxG], int tmp[36]
    static constexpr int kPtab = kMisc + 2 * kMaxG * 4 + 36 * 4;      // int4 [warps][kWarpCap]
    static constexpr int kStall = kPtab + kDecWarps * kWarpCap * 16;  // u64: test-hook barrier
    static constexpr int kBytes = kStall + 8 + 1024;
    static_assert(kRing + kConvBytes >= kDecWarps * kMaxG * (2 + 64 * NH) * 4,
                  "per-warp partials must fit in the ring");
    static_assert(kInfo >= 32768 + kMaxG * 64 * NH * 4, "the cluster merge's partial must fit below the tables");
    static_assert(!F8 || NH == 2, "FP8 pieces are 128 columns");
};

template <int NH, int NST, bool CLUSTER, bool F8, bool PAGED>
__global__ void __launch_bounds__(kDecThreads, 2)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     DecArgs a) {
    using L = TcSmem<NH, NST, F8>;
    using T = std::conditional_t<F8, uint8_t, uint16_t>;   // cache element
    constexpr int D = 64 * NH;
    constexpr int NT = D / 8;   // 8-column MMA tiles across D
    extern __shared__ unsigned char dsm_raw[];
    unsigned char *dsm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
    int2 *info = reinterpret_cast<int2 *>(dsm + L::kInfo);
    uint64_t *full = reinterpret_cast<uint64_t *>(dsm + L::kBars);
    float *sml = reinterpret_cast<float *>(dsm + L::kMisc);
    int4 *ptab = reinterpret_cast<int4 *>(dsm + L::kPtab);

    const int c = blockIdx.x, s = blockIdx.y;
    const int b = s / a.Hkv, g = s % a.Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gid = lane >> 2, tig = lane & 3;

    // Every warp works out its own pieces: no CTA-wide barrier before the
    // first load.
    unsigned char *ring = dsm + warp * NST * L::kPieceBytes;
    unsigned char *conv = dsm + L::kConv + warp * NH * kBoxBytes;   // FP8 only: f16 V
    uint64_t *wfull = full + warp * NST;
    int2 *winfo = info + warp * NST;   // .x: valid rows of the stage's piece
    int4 *wtab = ptab + warp * kWarpCap;
    if (tid == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    if (lane == 0) {
        for (int i = 0; i < NST; ++i) mbar_init(&wfull[i], 1);
        fence_mbar_init();
    }
    if (a.stall_ns && c == 0 && s == 0 && tid == 0) {
        // test hook: a bounded wait on a barrier that nothing completes, before
        // any copy is issued; it gives up after stall_ns and reports a timeout
        uint64_t *bar = reinterpret_cast<uint64_t *>(dsm + L::kStall);
        mbar_init(bar, 1);
        fence_mbar_init();
        if (!mbar_wait_bounded(bar, 0u, a.stall_ns)) atomicOr(a.status, 1u);
    }
    pdl_wait();   // ranges, lengths and the cache come from earlier kernels
    // fused append: lanes 0.. hold 16-byte chunks of the new key, lanes 16..
    // of the new value
    constexpr int kChunks = D * (int)sizeof(T) / 16;
    uint4 nkv = make_uint4(0u, 0u, 0u, 0u);
    if (a.app.k_new) {
        if (lane < kChunks)
            nkv = __ldg(static_cast<const uint4 *>(a.app.k_new) + (int64_t)s * kChunks + lane);
        else if (lane >= 16 && lane - 16 < kChunks)
            nkv = __ldg(static_cast<const uint4 *>(a.app.v_new) + (int64_t)s * kChunks + lane - 16);
    }
    const WarpRanges wr = warp_ranges<PAGED>(a, s, b, c, warp, lane, wtab);
    const int n_my = wr.last - wr.first;
    // this warp's pieces: CTA-local indices warp, warp + 4, warp + 8, ...
    const int my_count = n_my > warp ? (n_my - warp + kDecWarps - 1) / kDecWarps : 0;
    if constexpr (PAGED) warp_translate(a, b, lane, min(my_count, kWarpCap), wtab);
    __syncwarp();
    auto issue = [&](int idx, int st) {   // lane 0 only
        const int4 pr = wtab[idx % kWarpCap];
        winfo[st].x = pr.y;
        mbar_arrive_expect_tx(&wfull[st], (uint32_t)L::kPieceBytes);
        unsigned char *dst = ring + st * L::kPieceBytes;
        if constexpr (F8) {
            tma_load_4d(dst, &tmK, &wfull[st], 0, pr.z, g, pr.w);
            tma_load_4d(dst + kBoxBytes, &tmV, &wfull[st], 0, pr.z, g, pr.w);
        } else {
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                tma_load_4d(dst + h * kBoxBytes, &tmK, &wfull[st], h * 64, pr.z, g, pr.w);
                tma_load_4d(dst + (NH + h) * kBoxBytes, &tmV, &wfull[st], h * 64, pr.z, g, pr.w);
            }
        }
    };
    // Warp-collective, before piece idx is issued: if the piece holds the
    // appended row, write the row (its TMA load then sees it).
    bool wrote = false;
    auto maybe_append = [&](int idx) {
        if (wr.app < 0) return;
        const int4 pr = wtab[idx % kWarpCap];
        if (pr.x + (pr.y & 255) <= wr.app && wr.app < pr.x + (pr.y >> 8)) {
            const int64_t off = PAGED ? a.rows.off(b, g, wr.app)
                                      : b * a.rows.stride_b + g * a.rows.stride_h + (int64_t)wr.app * a.rows.stride_t;
            if (off >= 0) {   // (a row whose page is outside the pool is not written)
                if (lane < kChunks)
                    reinterpret_cast<uint4 *>(static_cast<T *>(const_cast<void *>(a.K)) + off)[lane] = nkv;
                else if (lane >= 16 && lane - 16 < kChunks)
                    reinterpret_cast<uint4 *>(static_cast<T *>(const_cast<void *>(a.V)) + off)[lane - 16] = nkv;
                asm volatile("fence.proxy.async.global;" ::: "memory");
            }
            __syncwarp();
            wrote = true;
        }
    };
    for (int j = 0; j < NST && j < my_count; ++j) {
        maybe_append(j);
        if (lane == 0) issue(j, j);
    }

    // q fragments: rows 0-7 q_hi of head gid, rows 8-15 q_lo; zero past G
    uint32_t qa[D / 16][4];
    {
        const float *qg = a.q + ((int64_t)b * a.Hq + (int64_t)g * a.G + gid) * D;
        const bool live = gid < a.G;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            float x[4];
            // logical columns 2 tig, 2 tig + 1, 2 tig + 8, 2 tig + 9 of the
            // 16-wide step; an FP8 cache pairs them with physical columns
            // 4 tig .. 4 tig + 3 (its K fragments are four consecutive codes),
            // the dot product being the same sum in another order of terms
            const int k0 = kk * 16 + (F8 ? 4 * tig : 2 * tig);
            x[0] = live ? qg[k0] : 0.0f;
            x[1] = live ? qg[k0 + 1] : 0.0f;
            x[2] = live ? qg[k0 + (F8 ? 2 : 8)] : 0.0f;
            x[3] = live ? qg[k0 + (F8 ? 3 : 9)] : 0.0f;
            float hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                hi[e] = F8 ? f16_round(x[e]) : bf16_round(x[e]);
                lo[e] = x[e] - hi[e];
            }
            if constexpr (F8) {
                qa[kk][0] = pack_f16x2(hi[0], hi[1]);
                qa[kk][1] = pack_f16x2(lo[0], lo[1]);
                qa[kk][2] = pack_f16x2(hi[2], hi[3]);
                qa[kk][3] = pack_f16x2(lo[2], lo[3]);
            } else {
                qa[kk][0] = pack_bf16x2(hi[0], hi[1]);
                qa[kk][1] = pack_bf16x2(lo[0], lo[1]);
                qa[kk][2] = pack_bf16x2(hi[2], hi[3]);
                qa[kk][3] = pack_bf16x2(lo[2], lo[3]);
            }
        }
    }

    float o[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m_run = kNegInf, l_run = 0.0f;
    bool timed_out = false;

    for (int idx = 0; idx < my_count; ++idx) {
        const int st = idx % NST;
        if (!timed_out && !mbar_wait_bounded(&wfull[st], (uint32_t)((idx / NST) & 1))) timed_out = true;
        const int vr = winfo[st].x;
        const int vlo = vr & 255, vhi = vr >> 8;   // valid rows [vlo, vhi) of the box
        unsigned char *kp = ring + st * L::kPieceBytes;
        unsigned char *vp = kp + NH * kBoxBytes;
        bool issued_early = false;
        // S = Q K^T for the piece's 16 rows: two 8-row MMA tiles, even and odd
        // k-steps in separate accumulators (shorter dependency chains)
        float sa[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        float sb[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        if constexpr (F8) {
            // V: the stage's FP8 box -> this warp's f16 box in the bf16 layout
            // (FP8 chunk c of a row: columns 16c .. 16c+15, i.e. f16 box c / 4,
            // chunks 2 (c % 4) and 2 (c % 4) + 1); rows outside [vlo, vhi)
            // become zeros so that 0 * junk stays 0
            const unsigned char *vsrc = kp + kBoxBytes;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int u = lane + 32 * k;
                const int r = u >> 3, cc = u & 7;
                const uint4 w = *reinterpret_cast<const uint4 *>(vsrc + r * 128 + ((cc ^ (r & 7)) << 4));
                uint32_t h[8];
                const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    h[2 * e] = fp8x2_to_f16x2((uint16_t)(wv[e] & 0xffffu));
                    h[2 * e + 1] = fp8x2_to_f16x2((uint16_t)(wv[e] >> 16));
                }
                if (r < vlo || r >= vhi)
#pragma unroll
                    for (int e = 0; e < 8; ++e) h[e] = 0u;
                unsigned char *row = conv + (cc >> 2) * kBoxBytes + r * 128;
                const int c0 = 2 * (cc & 3);
                *reinterpret_cast<uint4 *>(row + ((c0 ^ (r & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
                *reinterpret_cast<uint4 *>(row + (((c0 + 1) ^ (r & 7)) << 4)) =
                    make_uint4(h[4], h[5], h[6], h[7]);
            }
            // K fragments straight from the FP8 box: row gid (+8), four codes
            // at columns 16 kk + 4 tig widened to two f16 pairs
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int r = gid + 8 * nt;
                    const uint32_t w = *reinterpret_cast<const uint32_t *>(
                        kp + r * 128 + ((kk ^ (r & 7)) << 4) + 4 * tig);
                    const uint32_t b0 = fp8x2_to_f16x2((uint16_t)(w & 0xffffu));
                    const uint32_t b1 = fp8x2_to_f16x2((uint16_t)(w >> 16));
                    mma_f16_16816(kk & 1 ? sb[nt] : sa[nt], qa[kk], b0, b1);
                }
            __syncwarp();
            // the stage has been read: its next copy can start now
            if (idx + NST < my_count) {
                if ((idx + NST) % kWarpCap == 0) {   // next window of this warp's pieces
                    warp_refill<PAGED>(a, wr, warp, idx + NST, b, wtab);
                    if constexpr (PAGED) warp_translate(a, b, lane, min(my_count - (idx + NST), kWarpCap), wtab);
                    __syncwarp();
                }
                maybe_append(idx + NST);
                if (lane == 0) issue(idx + NST, st);
            }
            issued_early = true;
            vp = conv;
        } else if (vlo > 0 || vhi < kPiece) {   // rows outside the range: zero V so 0 * junk stays 0
            for (int e = lane; e < kPiece * NH * 8; e += 32) {
                const int r = e / (NH * 8), h = (e / 8) % NH, ch = e % 8;
                if (r < vlo || r >= vhi)
                    *reinterpret_cast<uint4 *>(vp + h * kBoxBytes + r * 128 + ch * 16) =
                        make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
        }
        const uint32_t kbase = smem_u32(kp), vbase = smem_u32(vp);
#pragma unroll
        for (int kk = 0; kk < (F8 ? 0 : D / 16); ++kk) {   // bf16: K fragments by ldmatrix
            const int half = kk / 4, ch0 = (kk % 4) * 2;
            const int r = (lane >> 4) * 8 + (lane & 7);
            const int ch = ch0 + ((lane >> 3) & 1);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(kbase + half * kBoxBytes + r * 128 + ((ch ^ (r & 7)) << 4), b0, b1, b2, b3);
            if (kk & 1) {
                mma_bf16_16816(sb[0], qa[kk], b0, b1);
                mma_bf16_16816(sb[1], qa[kk], b2, b3);
            } else {
                mma_bf16_16816(sa[0], qa[kk], b0, b1);
                mma_bf16_16816(sa[1], qa[kk], b2, b3);
            }
        }
        float lg[4];
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int tok = n * 8 + 2 * tig + e;
                const float v = (sa[n][e] + sb[n][e]) + (sa[n][2 + e] + sb[n][2 + e]);
                lg[n * 2 + e] = tok >= vlo && tok < vhi ? v * a.scale_log2 : kNegInf;
            }
        float mx = fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(m_run, mx);
        float p[4];
        if (m_new == kNegInf) {
            p[0] = p[1] = p[2] = p[3] = 0.0f;
        } else {
            const float corr = exp2f(m_run - m_new);
#pragma unroll
            for (int e = 0; e < 4; ++e) p[e] = exp2f(lg[e] - m_new);
            l_run = l_run * corr + ((p[0] + p[1]) + (p[2] + p[3]));
            if (corr != 1.0f) {
#pragma unroll
                for (int i = 0; i < NT; ++i) {
                    o[i][0] *= corr; o[i][1] *= corr; o[i][2] *= corr; o[i][3] *= corr;
                }
            }
            m_run = m_new;
        }
        uint32_t pa[4];
        {
            float ph[4], pl[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                ph[e] = F8 ? f16_round(p[e]) : bf16_round(p[e]);
                pl[e] = p[e] - ph[e];
            }
            if constexpr (F8) {
                pa[0] = pack_f16x2(ph[0], ph[1]);
                pa[1] = pack_f16x2(pl[0], pl[1]);
                pa[2] = pack_f16x2(ph[2], ph[3]);
                pa[3] = pack_f16x2(pl[2], pl[3]);
            } else {
                pa[0] = pack_bf16x2(ph[0], ph[1]);
                pa[1] = pack_bf16x2(pl[0], pl[1]);
                pa[2] = pack_bf16x2(ph[2], ph[3]);
                pa[3] = pack_bf16x2(pl[2], pl[3]);
            }
        }
        // O += P V
#pragma unroll
        for (int cp = 0; cp < D / 16; ++cp) {
            const int half = cp / 4, ch0 = (cp % 4) * 2;
            const int r = ((lane >> 3) & 1) * 8 + (lane & 7);
            const int ch = ch0 + (lane >> 4);
            uint32_t r0, r1, r2, r3;
            ldmatrix_x4_trans(vbase + half * kBoxBytes + r * 128 + ((ch ^ (r & 7)) << 4), r0, r1, r2, r3);
            if constexpr (F8) {
                mma_f16_16816(o[2 * cp], pa, r0, r1);
                mma_f16_16816(o[2 * cp + 1], pa, r2, r3);
            } else {
                mma_bf16_16816(o[2 * cp], pa, r0, r1);
                mma_bf16_16816(o[2 * cp + 1], pa, r2, r3);
            }
        }
        __syncwarp();
        if (!issued_early && idx + NST < my_count) {
            if ((idx + NST) % kWarpCap == 0) {   // next window of this warp's pieces
                warp_refill<PAGED>(a, wr, warp, idx + NST, b, wtab);
                if constexpr (PAGED) warp_translate(a, b, lane, min(my_count - (idx + NST), kWarpCap), wtab);
                __syncwarp();
            }
            maybe_append(idx + NST);
            if (lane == 0) issue(idx + NST, st);
        }
    }
    if (timed_out) atomicOr(a.status, 1u);
    // the merge kernel may be scheduled now; it waits for this grid to finish
    pdl_trigger();

    // per-warp partials -> shared memory (reusing the rings once all are idle)
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    float *wm = reinterpret_cast<float *>(dsm);
    float *wl = wm + kDecWarps * kMaxG;
    float *wo = wl + kDecWarps * kMaxG;
    const bool cta_wrote = __syncthreads_or(wrote);
    if (tig == 0) {
        wm[warp * kMaxG + gid] = m_run;
        wl[warp * kMaxG + gid] = l_run;
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int d = nt * 8 + 2 * tig;
        wo[(warp * kMaxG + gid) * D + d] = o[nt][0] + o[nt][2];
        wo[(warp * kMaxG + gid) * D + d + 1] = o[nt][1] + o[nt][3];
    }
    __syncthreads();
    if constexpr (CLUSTER)
        cluster_finish(a, b, g, wm, wl, wo, sml, reinterpret_cast<float *>(dsm + 32768));
    else
        finish(a, s, b, g, c, wm, wl, wo, sml);
    if (a.app.k_new) finish_append<T>(a, b, g, wr.app, cta_wrote);
}

// ======================================================================
// CUDA-core path (fp32 or bf16 K/V, any G <= 8, D in {64, 128})
// ======================================================================
template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads) decode_generic_kernel(DecArgs a) {
    constexpr int PER = D / 32;
    extern __shared__ __align__(16) unsigned char dsm[];
    float *wm = reinterpret_cast<float *>(dsm);
    float *wl = wm + kDecWarps * kMaxG;
    float *wo = wl + kDecWarps * kMaxG;
    float *sml = wo + kDecWarps * kMaxG * D;
    int *tmp = reinterpret_cast<int *>(sml + 2 * kMaxG);
    int *rs = tmp + 36;
    int *re = rs + a.max_ranges;
    int *ps = re + a.max_ranges;

    const int c = blockIdx.x, s = blockIdx.y;
    const int b = s / a.Hkv, g = s % a.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    int nr;
    const int P = load_ranges(a, s, b, rs, re, ps, tmp, &nr);
    int per = (P + a.nsplit - 1) / a.nsplit;
    per = (per + kDecWarps - 1) / kDecWarps * kDecWarps;
    const int first = c * per, last = min(P, first + per);

    float qr[kMaxG][PER];
    const float *qg = a.q + ((int64_t)b * a.Hq + (int64_t)g * a.G) * D;
#pragma unroll
    for (int h = 0; h < kMaxG; ++h)
#pragma unroll
        for (int k = 0; k < PER; ++k) qr[h][k] = h < a.G ? qg[h * D + lane + 32 * k] : 0.0f;
    float m[kMaxG], l[kMaxG], o[kMaxG][PER];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
        m[h] = kNegInf;
        l[h] = 0.0f;
#pragma unroll
        for (int k = 0; k < PER; ++k) o[h][k] = 0.0f;
    }
    const T *Ks = static_cast<const T *>(a.K);
    const T *Vs = static_cast<const T *>(a.V);
    for (int p = first + warp; p < last; p += kDecWarps) {
        const int2 pr = piece_rows(p, rs, re, ps, nr);
        for (int r = pr.x; r < pr.x + pr.y; ++r) {
            const int64_t ro = a.rows.off(b, g, r);   // < 0: the row's page is outside the pool
            float kv[PER], vv[PER];
#pragma unroll
            for (int k = 0; k < PER; ++k) {
                kv[k] = ro < 0 ? 0.0f : load_elem(Ks, ro + lane + 32 * k);
                vv[k] = ro < 0 ? 0.0f : load_elem(Vs, ro + lane + 32 * k);
            }
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) {
                if (h >= a.G) break;
                float dot = 0.0f;
#pragma unroll
                for (int k = 0; k < PER; ++k) dot = fmaf(qr[h][k], kv[k], dot);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
                const float lg = dot * a.scale_log2;
                const float mn = fmaxf(m[h], lg);
                const float corr = exp2f(m[h] - mn);
                const float pw = exp2f(lg - mn);
                l[h] = l[h] * corr + pw;
#pragma unroll
                for (int k = 0; k < PER; ++k) o[h][k] = o[h][k] * corr + pw * vv[k];
                m[h] = mn;
            }
        }
    }
    pdl_trigger();
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
        if (lane == 0) {
            wm[warp * kMaxG + h] = m[h];
            wl[warp * kMaxG + h] = l[h];
        }
#pragma unroll
        for (int k = 0; k < PER; ++k) wo[(warp * kMaxG + h) * D + lane + 32 * k] = o[h][k];
    }
    __syncthreads();
    finish(a, s, b, g, c, wm, wl, wo, sml);
}

// ======================================================================
// Host side
// ======================================================================
constexpr int kTcStages = 3;   // pieces in flight per warp (bf16)
constexpr int kF8Stages = 4;   // pieces in flight per warp (FP8: half the bytes per piece)

static bool use_tc(const bsa_kv_desc *d) {
    const bool dt = d->kv_dtype == BSA_BF16 ? (d->D == 64 || d->D == 128)
                                            : d->kv_dtype == BSA_FP8_E4M3 && d->D == 128;
    return dt && d->Hq / d->Hkv <= kMaxG && d->stride_t == d->D;
}

bool decode_can_fuse_append(const bsa_kv_desc *d) { return use_tc(d); }

constexpr int kMinWarpPieces = 8;   // pieces per warp below which more splits stop paying

// Few segments: even the largest clusters would leave SMs idle.  Their splits
// are not clustered (so there can be more of them) and the merge kernel
// combines them.
static bool few_segments(const bsa_kv_desc *d) {
    return (int64_t)d->B * d->Hkv * kMaxClusterSplits < num_sms();
}

int decode_nsplit(const bsa_kv_desc *d, int tokens_hint, int max_ranges) {
    const int nseg = d->B * d->Hkv;
    const int64_t pieces = div_up(tokens_hint > 0 ? tokens_hint : 1, kPiece) + max_ranges;
    const int slots = num_sms() * (use_tc(d) ? 2 : 4);
    int nsplit = std::max(1, slots / std::max(nseg, 1));
    if (use_tc(d)) {
        if (few_segments(d))   // every resident slot, while warps keep enough pieces
            nsplit = (int)std::min<int64_t>(
                nsplit, std::max<int64_t>(kMaxClusterSplits, pieces / (kDecWarps * kMinWarpPieces)));
        else
            nsplit = std::min(nsplit, kMaxClusterSplits);   // one cluster per segment
    }
    nsplit = (int)std::min<int64_t>(nsplit, div_up(pieces, kDecWarps));
    return std::max(1, nsplit);
}

// Largest cluster size c <= max_c (c >= 2) for which all nseg clusters of the
// decode kernel can be resident at once, or 0.  Cached per configuration.
static int cluster_splits(const void *kern, int smem, int nseg, int max_c, cudaLaunchConfig_t cfg) {
    struct Key {
        const void *k;
        int smem, nseg, max_c, dev;
    };
    static std::mutex mu;
    static std::vector<std::pair<Key, int>> cache;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    for (auto &e : cache)
        if (e.first.k == kern && e.first.smem == smem && e.first.nseg == nseg &&
            e.first.max_c == max_c && e.first.dev == dev)
            return e.second;
    int best = 0;
    cudaLaunchAttribute attr = cfg.attrs[0];
    for (int c = std::min(max_c, kMaxClusterSplits); c >= 2 && !best; --c) {
        attr.val.clusterDim.x = c;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        cfg.gridDim = dim3(c, (unsigned)nseg);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n >= nseg) best = c;
        cudaGetLastError();
    }
    cache.push_back({{kern, smem, nseg, max_c, dev}, best});
    return best;
}

// Kernels one launch_decode issues: 1 when the splits merge inside clusters
// (or there is one split), 2 when the merge kernel follows.  Mirrors the
// choice launch_decode makes.
int decode_kernel_count(const bsa_kv_desc *d, int tokens_hint, int max_ranges) {
    const int nsplit = decode_nsplit(d, tokens_hint, max_ranges);
    if (nsplit <= 1) return 1;
    if (!use_tc(d) || few_segments(d)) return 2;
    auto clusters_fit = [&](auto kern_cluster, int smem) -> bool {
        if (cudaFuncSetAttribute(kern_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
            cudaFuncSetAttribute(kern_cluster, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.blockDim = dim3(kDecThreads);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cluster_splits(reinterpret_cast<const void *>(kern_cluster), smem, d->B * d->Hkv, nsplit,
                              cfg) > 1;
    };
    auto fits = [&](auto paged) -> bool {
        constexpr bool PG = decltype(paged)::value;
        if (d->kv_dtype == BSA_FP8_E4M3)
            return clusters_fit(decode_tc_kernel<2, kF8Stages, true, true, PG>, TcSmem<2, kF8Stages, true>::kBytes);
        if (d->D == 128)
            return clusters_fit(decode_tc_kernel<2, kTcStages, true, false, PG>, TcSmem<2, kTcStages>::kBytes);
        return clusters_fit(decode_tc_kernel<1, 2 * kTcStages, true, false, PG>, TcSmem<1, 2 * kTcStages>::kBytes);
    };
    const bool fit = d->page_rows > 0 ? fits(std::true_type()) : fits(std::false_type());
    return fit ? 1 : 2;
}

size_t decode_scratch_bytes(const bsa_kv_desc *d, int nsplit) {
    const size_t nseg = (size_t)d->B * d->Hkv, G = d->Hq / d->Hkv;
    return align_up(nseg * nsplit * G * d->D * 4, 256) + align_up(nseg * nsplit * G * 8, 256);
}

bsa_status launch_decode(const bsa_kv_desc *d, const float *q, const void *K, const void *V,
                         const int32_t *ranges, const int32_t *n_ranges, int max_ranges,
                         const int32_t *cur_len, int tokens_hint, float scale, float *out,
                         float *lse, uint32_t *status, uint32_t *counters, void *scratch,
                         cudaStream_t st, const DecAppend *app) {
    if (app && !use_tc(d)) return BSA_ERR_UNSUPPORTED;
    DecArgs a;
    a.app = app ? *app : DecAppend{};
    a.q = q; a.out = out; a.lse = lse; a.ranges = ranges; a.n_ranges = n_ranges;
    a.max_ranges = max_ranges; a.cur_len = cur_len; a.K = K; a.V = V;
    a.rows = kv_rows(d);
    a.B = d->B; a.Hq = d->Hq; a.Hkv = d->Hkv; a.G = d->Hq / d->Hkv; a.D = d->D;
    a.L_max = d->L_max;
    a.nsplit = decode_nsplit(d, tokens_hint, max_ranges);
    a.scale_log2 = scale * 1.4426950408889634f;
    const size_t nseg = (size_t)d->B * d->Hkv;
    a.part_o = static_cast<float *>(scratch);
    a.part_ml = reinterpret_cast<float2 *>(static_cast<char *>(scratch) +
                                           align_up(nseg * a.nsplit * a.G * d->D * 4, 256));
    a.counters = counters;
    a.status = status;
    a.stall_ns = use_tc(d) ? g_armed_stall_ns.exchange(0u) : 0u;
    dim3 grid(a.nsplit, (unsigned)nseg);
    if (use_tc(d)) {
        CUtensorMap tk, tv;
        if (!make_kv_tmap(&tk, d, K, kPiece) || !make_kv_tmap(&tv, d, V, kPiece)) return BSA_ERR_CUDA;
        // The splits of a segment form one thread-block cluster when they fit
        // (merge through distributed shared memory, no second kernel).
        bool clustered = false;
        auto go_tc = [&](auto kern_plain, auto kern_cluster, int smem) -> bsa_status {
            BSA_CUDA_TRY(cudaFuncSetAttribute(kern_plain, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
            if (a.nsplit > 1 && !few_segments(d)) {
                BSA_CUDA_TRY(cudaFuncSetAttribute(kern_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
                BSA_CUDA_TRY(cudaFuncSetAttribute(kern_cluster, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
                cudaLaunchConfig_t cfg = {};
                cfg.blockDim = dim3(kDecThreads);
                cfg.dynamicSmemBytes = smem;
                cfg.stream = st;
                cudaLaunchAttribute attr[2];
                attr[0].id = cudaLaunchAttributeClusterDimension;
                attr[0].val.clusterDim.y = 1;
                attr[0].val.clusterDim.z = 1;
                attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
                attr[1].val.programmaticStreamSerializationAllowed = 1;
                cfg.attrs = attr;
                cfg.numAttrs = 2;
                const int c = cluster_splits(reinterpret_cast<const void *>(kern_cluster), smem,
                                             (int)nseg, a.nsplit, cfg);
                if (c > 1) {
                    a.nsplit = c;
                    cfg.gridDim = dim3(c, (unsigned)nseg);
                    attr[0].val.clusterDim.x = c;
                    BSA_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern_cluster, tk, tv, a));
                    clustered = true;
                    return BSA_OK;
                }
            }
            BSA_CUDA_TRY(launch_pdl(kern_plain, grid, dim3(kDecThreads), smem, st, tk, tv, a));
            return BSA_OK;
        };
        auto by_layout = [&](auto paged) -> bsa_status {
            constexpr bool PG = decltype(paged)::value;
            if (d->kv_dtype == BSA_FP8_E4M3)
                return go_tc(decode_tc_kernel<2, kF8Stages, false, true, PG>,
                             decode_tc_kernel<2, kF8Stages, true, true, PG>, TcSmem<2, kF8Stages, true>::kBytes);
            if (d->D == 128)
                return go_tc(decode_tc_kernel<2, kTcStages, false, false, PG>,
                             decode_tc_kernel<2, kTcStages, true, false, PG>, TcSmem<2, kTcStages>::kBytes);
            return go_tc(decode_tc_kernel<1, 2 * kTcStages, false, false, PG>,   // D = 64
                         decode_tc_kernel<1, 2 * kTcStages, true, false, PG>, TcSmem<1, 2 * kTcStages>::kBytes);
        };
        const bsa_status r = d->page_rows > 0 ? by_layout(std::true_type()) : by_layout(std::false_type());
        if (r != BSA_OK) return r;
        BSA_LAUNCH_CHECK();
        if (clustered) return BSA_OK;
    } else {
        const size_t smem = (size_t)(2 * kDecWarps * kMaxG + kDecWarps * kMaxG * d->D + 2 * kMaxG) * 4 +
                            36 * 4 + (size_t)(3 * max_ranges + 1) * 4;
        auto go = [&](auto kern) -> bsa_status {
            if (smem > 48 * 1024)
                BSA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
            BSA_CUDA_TRY(launch_pdl(kern, grid, dim3(kDecThreads), smem, st, a));
            return BSA_OK;
        };
        bsa_status r;
        if (d->kv_dtype == BSA_BF16)
            r = d->D == 128 ? go(decode_generic_kernel<uint16_t, 128>) : go(decode_generic_kernel<uint16_t, 64>);
        else if (d->kv_dtype == BSA_FP8_E4M3)
            r = d->D == 128 ? go(decode_generic_kernel<uint8_t, 128>) : go(decode_generic_kernel<uint8_t, 64>);
        else
            r = d->D == 128 ? go(decode_generic_kernel<float, 128>) : go(decode_generic_kernel<float, 64>);
        if (r != BSA_OK) return r;
    }
    BSA_LAUNCH_CHECK();
    if (a.nsplit > 1) {
        // the merge, as a programmatic dependent launch of the decode kernel
        BSA_CUDA_TRY(launch_pdl(lse_merge_kernel, dim3((unsigned)nseg, (unsigned)a.G), dim3(128),
                                0, st, a));
    }
    return BSA_OK;
}

}  // namespace bsa
