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
// One kernel, grid (tiles of 128 blocks, segments).  Every CTA brings its
// tile of summary rows into shared memory with 2-D TMA loads (128-byte
// swizzle, so that thread j reading row j is conflict-free), scores it one
// thread per block in the fixed fp32 order (fma chain over the dimensions per
// query head, heads summed in order) and writes orderable uint32 keys to the
// workspace.  The last CTA of a segment to finish (an atomic counter, reset
// afterwards) selects: radix select of the k-th key for top-k, or a bitonic
// sort and a greedy walk for the token budget, then an index-ordered
// compaction, so ties go to the lower block index and the result does not
// depend on which CTA finished last; finally the forced ranges and the
// selected blocks are merged into disjoint ranges with parallel scans.
#include "common.cuh"

namespace bsa {

constexpr int kSelThreads = 128;   // = rows per tile
constexpr int kSelMaxG = 16;
constexpr int kIntMin = -0x7fffffff - 1;

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
};

// 16-byte chunk of row j at byte offset `off` of a 128-byte-swizzled tile
// made of boxes of [kSelThreads rows][128 B].
__device__ __forceinline__ const uint4 *tile_chunk(const unsigned char *tile, int j, int off) {
    const int box = off >> 7, c = (off >> 4) & 7;
    return reinterpret_cast<const uint4 *>(tile + box * (kSelThreads * 128) + j * 128 +
                                           ((c ^ (j & 7)) << 4));
}

__device__ __forceinline__ void bf16x8(uint4 v, float (&f)[8]) {
    f[0] = __uint_as_float(v.x << 16); f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16); f[3] = __uint_as_float(v.y & 0xffff0000u);
    f[4] = __uint_as_float(v.z << 16); f[5] = __uint_as_float(v.z & 0xffff0000u);
    f[6] = __uint_as_float(v.w << 16); f[7] = __uint_as_float(v.w & 0xffff0000u);
}

// Score of tile row j for the group's G heads in the fixed fp32 order.
template <int KIND, typename T>
__device__ __forceinline__ float score_row(const float *qs, int G, int D, const unsigned char *tile,
                                           int j) {
    float acc[kSelMaxG];
#pragma unroll
    for (int h = 0; h < kSelMaxG; ++h) acc[h] = 0.0f;
    if constexpr (KIND == BSA_SUM_MINMAX && sizeof(T) == 2) {
        for (int i = 0; i < D; i += 8) {
            float lo[8], hi[8];
            bf16x8(*tile_chunk(tile, j, i * 2), lo);
            bf16x8(*tile_chunk(tile, j, (D + i) * 2), hi);
#pragma unroll
            for (int h = 0; h < kSelMaxG; ++h) {
                if (h < G) {
                    const float4 qa = *reinterpret_cast<const float4 *>(qs + h * D + i);
                    const float4 qb = *reinterpret_cast<const float4 *>(qs + h * D + i + 4);
                    const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        acc[h] = __fmaf_rn(qv[e], qv[e] >= 0.0f ? hi[e] : lo[e], acc[h]);
                }
            }
        }
    } else if constexpr (KIND == BSA_SUM_MINMAX) {
        for (int i = 0; i < D; i += 4) {
            const float4 a = *reinterpret_cast<const float4 *>(tile_chunk(tile, j, i * 4));
            const float4 c = *reinterpret_cast<const float4 *>(tile_chunk(tile, j, (D + i) * 4));
            const float lo[4] = {a.x, a.y, a.z, a.w}, hi[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
            for (int h = 0; h < kSelMaxG; ++h) {
                if (h < G) {
                    const float4 q4 = *reinterpret_cast<const float4 *>(qs + h * D + i);
                    const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        acc[h] = __fmaf_rn(qv[e], qv[e] >= 0.0f ? hi[e] : lo[e], acc[h]);
                }
            }
        }
    } else {
        for (int i = 0; i < D; i += 4) {
            const float4 cv = *reinterpret_cast<const float4 *>(tile_chunk(tile, j, i * 4));
#pragma unroll
            for (int h = 0; h < kSelMaxG; ++h) {
                if (h < G) {
                    const float4 qv = *reinterpret_cast<const float4 *>(qs + h * D + i);
                    acc[h] = __fmaf_rn(qv.x, cv.x, acc[h]);
                    acc[h] = __fmaf_rn(qv.y, cv.y, acc[h]);
                    acc[h] = __fmaf_rn(qv.z, cv.z, acc[h]);
                    acc[h] = __fmaf_rn(qv.w, cv.w, acc[h]);
                }
            }
        }
    }
    float tot = acc[0];
#pragma unroll
    for (int h = 1; h < kSelMaxG; ++h)
        if (h < G) tot = __fadd_rn(tot, acc[h]);
    return __fadd_rn(tot, 0.0f);
}

// Number of rows of [r0, r1) whose position is below lim (positions ascend).
__device__ __forceinline__ int visible_prefix(const int32_t *pos, int r0, int r1, int lim) {
    int lo = r0, hi = r1;
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if (pos[mid] < lim) lo = mid + 1; else hi = mid;
    }
    return lo - r0;
}

// Dynamic shared memory: [tile: nbox x 16 KiB, 1024-aligned][keys nb][sel
// max_sel][vis nb][sort buffer (budget) or histogram (top-k)][merge items
// (max_sel + 4) x int2][prefix maxima (max_sel + 4) x int]
struct SelSmem {
    __host__ __device__ static size_t tile_bytes(int nbox) { return (size_t)nbox * kSelThreads * 128; }
    __host__ __device__ static int pow2(int nb) {
        int N = 1;
        while (N < nb) N <<= 1;
        return N;
    }
    __host__ __device__ static size_t sort_bytes(int nb, bool variable) {
        return variable ? (size_t)pow2(nb) * 8 : 256 * 4;
    }
    static size_t bytes(int nbox, int nb, int max_sel, bool variable) {
        size_t p2 = (size_t)(2 * nb + max_sel) * 4;   // phase 2 reuses the tile buffer
        p2 = (p2 + 7) & ~size_t(7);
        p2 += sort_bytes(nb, variable);
        p2 += (size_t)(max_sel + 4) * 12;
        return 1024 + std::max(tile_bytes(nbox), p2);
    }
};

template <int KIND, typename T>
__global__ void __launch_bounds__(kSelThreads)
    select_kernel(const __grid_constant__ CUtensorMap tmS, SelArgs a) {
    extern __shared__ unsigned char dsm_raw[];
    unsigned char *tile = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(16) float qs[kSelMaxG * 128];
    __shared__ int tmp[40];
    __shared__ int is_last;
    __shared__ uint64_t bar;

    const int s = blockIdx.y;
    const int b = s / a.Hkv, g = s % a.Hkv;
    const int tid = threadIdx.x;
    const int nb = a.nb_total;
    const int j0 = blockIdx.x * kSelThreads;
    if (tid == 0) {
        prefetch_tmap(&tmS);
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    pdl_trigger();
    pdl_wait();   // queries, lengths and summaries come from earlier kernels
    __syncthreads();
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar, (uint32_t)(a.nbox * kSelThreads * 128));
        const int esz = (KIND == BSA_SUM_MINMAX) ? (int)sizeof(T) : 4;
        for (int bx = 0; bx < a.nbox; ++bx)
            tma_load_2d(tile + bx * (kSelThreads * 128), &tmS, &bar, bx * (128 / esz), s * nb + j0);
    }
    const int n = min(max(a.cur_len[b], 0), a.L_max);
    const int32_t *off = a.offsets ? a.offsets + (int64_t)s * (nb + 1) : nullptr;
    const int32_t *pos = a.kv_pos ? a.kv_pos + (int64_t)s * a.L_max : nullptr;
    for (int e = tid; e < a.G * a.D; e += kSelThreads)
        qs[e] = a.q[((int64_t)b * a.Hq + (int64_t)g * a.G) * a.D + e];

    // ---------------- phase 1: score this CTA's tile, one thread per block
    const int j = j0 + tid;
    bool valid = false;
    int vis = 0;
    if (j < nb) {
        if (off) {
            const int r0 = min(max(off[j], 0), a.L_max), r1 = min(max(off[j + 1], r0), a.L_max);
            vis = visible_prefix(pos, r0, r1, a.pos_limit);
            valid = vis > 0;
        } else {
            valid = (int64_t)(j + 1) * a.S <= n;
        }
    }
    __syncthreads();   // qs
    if (!mbar_wait_bounded(&bar, 0)) atomicOr(a.status, 2u);
    if (j < nb) {
        uint32_t key = 0;
        if (valid) {
            key = f32_order_key(score_row<KIND, T>(qs, a.G, a.D, tile, tid));
            if (key == 0) key = 1;   // 0 marks "not a candidate"
        }
        a.keys[(int64_t)s * nb + j] = key;
        if (off) a.vis[(int64_t)s * nb + j] = vis;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = atomicAdd(&a.counters[s], 1u) == gridDim.x - 1;
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    // ---------------- phase 2: the last CTA of the segment selects (its tile
    // has been scored; the buffer is reused)
    uint32_t *keys = reinterpret_cast<uint32_t *>(tile);
    int32_t *sel = reinterpret_cast<int32_t *>(keys + nb);
    int32_t *visb = sel + a.max_sel;
    unsigned char *after = reinterpret_cast<unsigned char *>(visb + nb);
    after = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(after) + 7) & ~uintptr_t(7));
    unsigned long long *sortbuf = reinterpret_cast<unsigned long long *>(after);
    int2 *mrg = reinterpret_cast<int2 *>(after + SelSmem::sort_bytes(nb, off != nullptr));
    int *pmax = reinterpret_cast<int *>(mrg + a.max_sel + 4);
    __shared__ int f_lo[3], f_hi[3], n_forced, n_sel_sh;

    if (tid == 0) {
        // forced token ranges, sorted and merged
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

    // candidates: keys > 0 and (fixed blocks) not wholly inside the forced set
    int my_c = 0;
    for (int jj = tid; jj < nb; jj += kSelThreads) {
        uint32_t key = __ldcg(&a.keys[(int64_t)s * nb + jj]);
        if (key && !off) {
            const int64_t r0 = (int64_t)jj * a.S, r1 = r0 + a.S;
            for (int i = 0; i < n_forced; ++i)
                if (f_lo[i] <= r0 && r1 <= f_hi[i]) key = 0;
        }
        keys[jj] = key;
        if (off) visb[jj] = __ldcg(&a.vis[(int64_t)s * nb + jj]);
        my_c += key != 0;
    }
    int n_cand;
    cta_excl_sum(my_c, tmp, &n_cand);

    const bool greedy = off && a.topk < 0;
    if (!greedy) {
        // ---- top-k: radix select of the k-th largest key, 8 bits per pass
        int k = a.topk >= 0 ? a.topk : a.budget / a.S;
        k = min(min(k, n_cand), a.max_sel);
        uint32_t thr = 0xffffffffu;
        int need_eq = 0;
        if (k > 0) {
            int *hist = reinterpret_cast<int *>(sortbuf);   // 256 bins
            __shared__ int sh_bin, sh_excl;
            uint32_t prefix = 0, pmask = 0;
            int krem = k;
            for (int pass = 0; pass < 4; ++pass) {
                const int shift = 24 - 8 * pass;
                hist[2 * tid] = 0;
                hist[2 * tid + 1] = 0;
                __syncthreads();
                for (int jj = tid; jj < nb; jj += kSelThreads) {
                    const uint32_t key = keys[jj];
                    if (key && (key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1);
                }
                __syncthreads();
                // thread t owns bins 255-2t and 254-2t (counted from the top)
                const int v0 = hist[255 - 2 * tid], v1 = hist[254 - 2 * tid];
                int tot;
                const int ex = cta_excl_sum(v0 + v1, tmp, &tot);
                if (ex < krem && ex + v0 >= krem) { sh_bin = 255 - 2 * tid; sh_excl = ex; }
                else if (ex + v0 < krem && ex + v0 + v1 >= krem) { sh_bin = 254 - 2 * tid; sh_excl = ex + v0; }
                __syncthreads();
                prefix |= (uint32_t)sh_bin << shift;
                pmask |= 0xffu << shift;
                krem -= sh_excl;
                __syncthreads();
            }
            thr = prefix;
            need_eq = krem;
        }
        // index-ordered compaction: key > thr, or key == thr among the first
        // need_eq; each thread owns a contiguous run of block indices
        const int chunk = (nb + kSelThreads - 1) / kSelThreads;
        const int c0 = min(nb, tid * chunk), c1 = min(nb, c0 + chunk);
        int my_eq = 0, my_gt = 0;
        if (k > 0)
            for (int jj = c0; jj < c1; ++jj) {
                const uint32_t key = keys[jj];
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
            for (int jj = c0; jj < c1; ++jj) {
                const uint32_t key = keys[jj];
                if (key != 0 && key > thr) sel[p++] = jj;
                else if (key != 0 && key == thr && eq_seen++ < need_eq) sel[p++] = jj;
            }
        }
    } else {
        // ---- token budget: bitonic sort by (key desc, index asc), greedy walk
        const int N = SelSmem::pow2(nb);
        for (int jj = tid; jj < N; jj += kSelThreads)
            sortbuf[jj] = jj < nb ? ((unsigned long long)keys[jj] << 32) | (0xffffffffu - (uint32_t)jj)
                                  : 0ull;
        __syncthreads();
        for (int kk = 2; kk <= N; kk <<= 1) {
            for (int jj = kk >> 1; jj > 0; jj >>= 1) {
                for (int i = tid; i < N; i += kSelThreads) {
                    const int ixj = i ^ jj;
                    if (ixj > i) {
                        const unsigned long long x = sortbuf[i], y = sortbuf[ixj];
                        const bool desc = (i & kk) == 0;
                        if (desc ? (x < y) : (x > y)) { sortbuf[i] = y; sortbuf[ixj] = x; }
                    }
                }
                __syncthreads();
            }
        }
        // greedy walk (sequential by definition); selection marks reuse the keys
        for (int jj = tid; jj < nb; jj += kSelThreads) keys[jj] = 0;
        __syncthreads();
        if (tid == 0) {
            int used = 0;
            for (int i = 0; i < n_cand; ++i) {
                const int jj = (int)(0xffffffffu - (uint32_t)(sortbuf[i] & 0xffffffffu));
                const int v = visb[jj];
                if (used + v <= a.budget) { used += v; keys[jj] = 0xffffffffu; }
            }
        }
        __syncthreads();
        const int chunk = (nb + kSelThreads - 1) / kSelThreads;
        const int c0 = min(nb, tid * chunk), c1 = min(nb, c0 + chunk);
        int my_take = 0;
        for (int jj = c0; jj < c1; ++jj) my_take += keys[jj] == 0xffffffffu;
        int tot;
        int p = cta_excl_sum(my_take, tmp, &tot);
        for (int jj = c0; jj < c1; ++jj)
            if (keys[jj] == 0xffffffffu && p < a.max_sel) sel[p++] = jj;
        if (tid == 0) n_sel_sh = min(tot, a.max_sel);
    }
    __syncthreads();
    const int n_sel = n_sel_sh, nf = n_forced;

    for (int i = tid; i < n_sel; i += kSelThreads) a.sel_blocks[(int64_t)s * a.max_sel + i] = sel[i];

    // ---- ranges.  Merge the forced ranges and the selected blocks' ranges
    // (both ascending; on equal starts the forced range comes first) ...
    const int m = n_sel + nf;
    for (int i = tid; i < n_sel; i += kSelThreads) {
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
    for (int t0 = 0; t0 < m; t0 += kSelThreads) {
        const int i = t0 + tid;
        int tot;
        const int pm = max(cta_incl_max(i < m ? mrg[i].y : kIntMin, tmp, &tot), carry);
        if (i < m) pmax[i] = pm;
        carry = max(carry, tot);
    }
    __syncthreads();
    int32_t *R = a.ranges + (int64_t)s * a.max_ranges * 2;
    int nr = 0;
    for (int t0 = 0; t0 < m; t0 += kSelThreads) {
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
        a.counters[s] = 0;   // leave the workspace reusable
    }
}

bsa_status launch_select(const bsa_kv_desc *d, const float *q, const void *summ, int kind,
                         const bsa_sel_params *p, const int32_t *cur_len, int nb_total,
                         int max_sel, int32_t *sel_blocks, int32_t *sel_count, int max_ranges,
                         int32_t *ranges, int32_t *n_ranges, uint32_t *keys, int32_t *vis,
                         uint32_t *counters, uint32_t *status, cudaStream_t st) {
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
    const bool bf = kind == BSA_SUM_MINMAX && d->kv_dtype == BSA_BF16;
    const int esz = bf ? 2 : 4;
    const int cols = kind == BSA_SUM_MINMAX ? 2 * d->D : d->D;
    a.row_bytes = cols * esz;
    a.nbox = a.row_bytes / 128;
    CUtensorMap tm;
    if (!make_rows_tmap(&tm, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                        esz, summ, cols, (int64_t)d->B * d->Hkv * nb_total, a.row_bytes, kSelThreads))
        return BSA_ERR_CUDA;
    const size_t smem = SelSmem::bytes(a.nbox, nb_total, max_sel, variable);
    if (smem > 220 * 1024) return BSA_ERR_UNSUPPORTED;
    dim3 grid((unsigned)div_up(nb_total, kSelThreads), d->B * d->Hkv);
    auto launch = [&](auto kern) -> bsa_status {
        BSA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        BSA_CUDA_TRY(launch_pdl(kern, grid, dim3(kSelThreads), smem, st, tm, a));
        return BSA_OK;
    };
    if (kind == BSA_SUM_MINMAX)
        return bf ? launch(select_kernel<BSA_SUM_MINMAX, uint16_t>)
                  : launch(select_kernel<BSA_SUM_MINMAX, float>);
    if (kind == BSA_SUM_CENTROID) return launch(select_kernel<BSA_SUM_CENTROID, float>);
    return launch(select_kernel<BSA_SUM_CENTROID_NORM, float>);
}

}  // namespace bsa
