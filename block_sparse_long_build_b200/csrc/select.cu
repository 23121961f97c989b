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
// One kernel, grid (chunks of 256 blocks, segments).  Every CTA scores its
// chunk, one thread per block, in the fixed fp32 order (fma chain over the
// dimensions per query head, heads summed in order) and writes orderable
// uint32 keys to the workspace.  The last CTA of a segment to finish (an
// atomic counter, reset afterwards) selects: radix select of the k-th key for
// top-k, or a bitonic sort and a greedy walk for the token budget, then an
// index-ordered compaction, so ties always go to the lower block index and
// the result does not depend on which CTA finished last.
#include "common.cuh"

namespace bsa {

constexpr int kSelThreads = 256;
constexpr int kSelMaxG = 16;

struct SelArgs {
    const float *q;
    const void *summ;
    const int32_t *cur_len;
    const int32_t *offsets;
    const int32_t *kv_pos;
    int32_t *sel_blocks, *sel_count, *ranges, *n_ranges;
    uint32_t *keys;       // ws [nseg][nb_total]
    int32_t *vis;         // ws [nseg][nb_total]
    uint32_t *counters;   // ws [nseg]
    int B, Hq, Hkv, G, D, L_max, S, nb_total, kind;
    int topk, budget, sink, window, keep_current, local_start, pos_limit;
    int max_sel, max_ranges;
};

// Exclusive scan of one int per thread over a 256-thread CTA.  `tmp` holds
// at least 9 ints; *total receives the CTA-wide sum.
__device__ __forceinline__ int cta_excl_scan(int v, int *tmp, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < 8 ? tmp[lane] : 0;
        int wi = w;
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) {
            int t = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += t;
        }
        if (lane < 8) tmp[lane] = wi - w;
        if (lane == 7) tmp[8] = wi;
    }
    __syncthreads();
    int res = incl - v + tmp[warp];
    *total = tmp[8];
    __syncthreads();
    return res;
}

// Score of one block for the group's G heads in the fixed fp32 order.
template <int KIND, typename T>
__device__ __forceinline__ float score_block(const float *qs, int G, int D, const void *row) {
    float acc[kSelMaxG];
#pragma unroll
    for (int h = 0; h < kSelMaxG; ++h) acc[h] = 0.0f;
    if constexpr (KIND == BSA_SUM_MINMAX) {
        const T *mn = static_cast<const T *>(row);
        const T *mx = mn + D;
        for (int i = 0; i < D; i += 4) {
            float lo[4], hi[4];
            if constexpr (sizeof(T) == 2) {
                uint2 a = *reinterpret_cast<const uint2 *>(mn + i);
                uint2 c = *reinterpret_cast<const uint2 *>(mx + i);
                lo[0] = __uint_as_float(a.x << 16); lo[1] = __uint_as_float(a.x & 0xffff0000u);
                lo[2] = __uint_as_float(a.y << 16); lo[3] = __uint_as_float(a.y & 0xffff0000u);
                hi[0] = __uint_as_float(c.x << 16); hi[1] = __uint_as_float(c.x & 0xffff0000u);
                hi[2] = __uint_as_float(c.y << 16); hi[3] = __uint_as_float(c.y & 0xffff0000u);
            } else {
                float4 a = *reinterpret_cast<const float4 *>(mn + i);
                float4 c = *reinterpret_cast<const float4 *>(mx + i);
                lo[0] = a.x; lo[1] = a.y; lo[2] = a.z; lo[3] = a.w;
                hi[0] = c.x; hi[1] = c.y; hi[2] = c.z; hi[3] = c.w;
            }
#pragma unroll
            for (int h = 0; h < kSelMaxG; ++h) {
                if (h < G) {
                    float4 qv = *reinterpret_cast<const float4 *>(qs + h * D + i);
                    acc[h] = __fmaf_rn(qv.x, qv.x >= 0.0f ? hi[0] : lo[0], acc[h]);
                    acc[h] = __fmaf_rn(qv.y, qv.y >= 0.0f ? hi[1] : lo[1], acc[h]);
                    acc[h] = __fmaf_rn(qv.z, qv.z >= 0.0f ? hi[2] : lo[2], acc[h]);
                    acc[h] = __fmaf_rn(qv.w, qv.w >= 0.0f ? hi[3] : lo[3], acc[h]);
                }
            }
        }
    } else {
        const float *c = static_cast<const float *>(row);
        for (int i = 0; i < D; i += 4) {
            float4 cv = *reinterpret_cast<const float4 *>(c + i);
#pragma unroll
            for (int h = 0; h < kSelMaxG; ++h) {
                if (h < G) {
                    float4 qv = *reinterpret_cast<const float4 *>(qs + h * D + i);
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

template <int KIND, typename T>
__global__ void __launch_bounds__(kSelThreads) select_kernel(SelArgs a) {
    extern __shared__ __align__(16) unsigned char dsm[];
    __shared__ __align__(16) float qs[kSelMaxG * 128];
    __shared__ int tmp[16];
    __shared__ int is_last;

    const int s = blockIdx.y;
    const int b = s / a.Hkv, g = s % a.Hkv;
    const int tid = threadIdx.x;
    const int n = min(max(a.cur_len[b], 0), a.L_max);
    const int32_t *off = a.offsets ? a.offsets + (int64_t)s * (a.nb_total + 1) : nullptr;
    const int32_t *pos = a.kv_pos ? a.kv_pos + (int64_t)s * a.L_max : nullptr;

    // ---------------- phase 1: score this CTA's chunk of blocks
    for (int e = tid; e < a.G * a.D; e += kSelThreads)
        qs[e] = a.q[((int64_t)b * a.Hq + (int64_t)g * a.G) * a.D + e];
    __syncthreads();
    const int j = blockIdx.x * kSelThreads + tid;
    if (j < a.nb_total) {
        bool valid;
        int vis = 0;
        if (off) {
            int r0 = min(max(off[j], 0), a.L_max), r1 = min(max(off[j + 1], r0), a.L_max);
            vis = visible_prefix(pos, r0, r1, a.pos_limit);
            valid = vis > 0;
        } else {
            valid = (int64_t)(j + 1) * a.S <= n;
        }
        uint32_t key = 0;
        if (valid) {
            size_t row_elems = KIND == BSA_SUM_MINMAX ? 2 * a.D : a.D;
            size_t esz = KIND == BSA_SUM_MINMAX ? sizeof(T) : sizeof(float);
            const char *row = static_cast<const char *>(a.summ) +
                              ((int64_t)s * a.nb_total + j) * row_elems * esz;
            key = f32_order_key(score_block<KIND, T>(qs, a.G, a.D, row));
            if (key == 0) key = 1;   // 0 marks "not a candidate"
        }
        a.keys[(int64_t)s * a.nb_total + j] = key;
        if (off) a.vis[(int64_t)s * a.nb_total + j] = vis;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        unsigned prev = atomicAdd(&a.counters[s], 1u);
        is_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    // ---------------- phase 2: the last CTA of the segment selects
    const int nb = a.nb_total;
    uint32_t *keys = reinterpret_cast<uint32_t *>(dsm);
    int32_t *sel = reinterpret_cast<int32_t *>(keys + nb);
    int32_t *vis = sel + a.max_sel;
    unsigned long long *sortbuf =
        reinterpret_cast<unsigned long long *>(dsm + ((((size_t)(2 * nb + a.max_sel)) * 4 + 7) & ~(size_t)7));
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
            int64_t r0 = (int64_t)jj * a.S, r1 = r0 + a.S;
            for (int i = 0; i < n_forced; ++i)
                if (f_lo[i] <= r0 && r1 <= f_hi[i]) key = 0;
        }
        keys[jj] = key;
        if (off) vis[jj] = __ldcg(&a.vis[(int64_t)s * nb + jj]);
        my_c += key != 0;
    }
    int n_cand;
    cta_excl_scan(my_c, tmp, &n_cand);

    const bool greedy = off && a.topk < 0;
    if (!greedy) {
        // ---- top-k: radix select of the k-th largest key
        int k = a.topk >= 0 ? a.topk : a.budget / a.S;
        k = min(min(k, n_cand), a.max_sel);
        uint32_t thr = 0xffffffffu;
        int need_eq = 0;
        if (k > 0) {
            int *hist = reinterpret_cast<int *>(sortbuf);   // 256 ints of scratch
            __shared__ int sh_bin, sh_excl;
            uint32_t prefix = 0, pmask = 0;
            int krem = k;
            for (int pass = 0; pass < 4; ++pass) {
                const int shift = 24 - 8 * pass;
                hist[tid] = 0;
                __syncthreads();
                for (int jj = tid; jj < nb; jj += kSelThreads) {
                    uint32_t key = keys[jj];
                    if (key && (key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1);
                }
                __syncthreads();
                const int v = hist[255 - tid];
                int tot;
                const int incl = cta_excl_scan(v, tmp, &tot) + v;
                if (incl >= krem && incl - v < krem) { sh_bin = 255 - tid; sh_excl = incl - v; }
                __syncthreads();
                prefix |= (uint32_t)sh_bin << shift;
                pmask |= 0xffu << shift;
                krem -= sh_excl;
                __syncthreads();
            }
            thr = prefix;
            need_eq = krem;
        }
        // index-ordered compaction: key > thr, or key == thr among the first need_eq
        int base_eq = 0, base_sel = 0;
        for (int t0 = 0; t0 < nb; t0 += kSelThreads) {
            const int jj = t0 + tid;
            const uint32_t key = (jj < nb && k > 0) ? keys[jj] : 0;
            const int eq = key != 0 && key == thr;
            int tot_eq, tot_take;
            const int eq_rank = base_eq + cta_excl_scan(eq, tmp, &tot_eq);
            const int take = (key != 0 && key > thr) || (eq && eq_rank < need_eq);
            const int p = base_sel + cta_excl_scan(take, tmp, &tot_take);
            if (take) sel[p] = jj;
            base_eq += tot_eq;
            base_sel += tot_take;
        }
        if (tid == 0) n_sel_sh = base_sel;
    } else {
        // ---- token budget: bitonic sort by (key desc, index asc), greedy walk
        int N = 1;
        while (N < nb) N <<= 1;
        for (int jj = tid; jj < N; jj += kSelThreads)
            sortbuf[jj] = jj < nb ? ((unsigned long long)keys[jj] << 32) | (0xffffffffu - (uint32_t)jj)
                                  : 0ull;
        __syncthreads();
        for (int kk = 2; kk <= N; kk <<= 1) {
            for (int jj = kk >> 1; jj > 0; jj >>= 1) {
                for (int i = tid; i < N; i += kSelThreads) {
                    int ixj = i ^ jj;
                    if (ixj > i) {
                        unsigned long long x = sortbuf[i], y = sortbuf[ixj];
                        bool desc = (i & kk) == 0;
                        if (desc ? (x < y) : (x > y)) { sortbuf[i] = y; sortbuf[ixj] = x; }
                    }
                }
                __syncthreads();
            }
        }
        // greedy walk (sequential by definition); selection marks reuse the
        // key array
        for (int jj = tid; jj < nb; jj += kSelThreads) keys[jj] = 0;
        __syncthreads();
        if (tid == 0) {
            int used = 0;
            for (int i = 0; i < n_cand; ++i) {
                int jj = (int)(0xffffffffu - (uint32_t)(sortbuf[i] & 0xffffffffu));
                int v = vis[jj];
                if (used + v <= a.budget) { used += v; keys[jj] = 0xffffffffu; }
            }
        }
        __syncthreads();
        int base_sel = 0;
        for (int t0 = 0; t0 < nb; t0 += kSelThreads) {
            const int jj = t0 + tid;
            const int take = jj < nb && keys[jj] == 0xffffffffu;
            int tot;
            const int p = base_sel + cta_excl_scan(take, tmp, &tot);
            if (take && p < a.max_sel) sel[p] = jj;
            base_sel += tot;
        }
        if (tid == 0) n_sel_sh = min(base_sel, a.max_sel);
    }
    __syncthreads();
    const int n_sel = n_sel_sh;

    for (int i = tid; i < n_sel; i += kSelThreads)
        a.sel_blocks[(int64_t)s * a.max_sel + i] = sel[i];
    if (tid == 0) {
        a.sel_count[s] = n_sel;
        // merge forced ranges and selected block ranges (both ascending)
        int32_t *R = a.ranges + (int64_t)s * a.max_ranges * 2;
        int nr = 0, fi = 0, si = 0;
        int cur_lo = 0, cur_hi = -1;
        while (fi < n_forced || si < n_sel) {
            int lo, hi;
            int blo = 0, bhi = 0;
            if (si < n_sel) {
                int jj = sel[si];
                if (off) { blo = min(max(off[jj], 0), a.L_max); bhi = blo + vis[jj]; }
                else { blo = jj * a.S; bhi = blo + a.S; }
            }
            if (si < n_sel && (fi >= n_forced || blo < f_lo[fi])) { lo = blo; hi = bhi; ++si; }
            else { lo = f_lo[fi]; hi = f_hi[fi]; ++fi; }
            if (hi <= lo) continue;
            if (cur_hi >= 0 && lo <= cur_hi) {
                cur_hi = max(cur_hi, hi);
            } else {
                if (cur_hi >= 0 && nr < a.max_ranges) { R[2 * nr] = cur_lo; R[2 * nr + 1] = cur_hi; ++nr; }
                cur_lo = lo; cur_hi = hi;
            }
        }
        if (cur_hi >= 0 && nr < a.max_ranges) { R[2 * nr] = cur_lo; R[2 * nr + 1] = cur_hi; ++nr; }
        a.n_ranges[s] = nr;
        a.counters[s] = 0;   // leave the workspace reusable
    }
}

size_t select_smem_bytes(int nb, int max_sel, bool variable) {
    size_t base = align_up((size_t)(2 * nb + max_sel) * 4, 8);
    int N = 1;
    while (N < nb) N <<= 1;
    size_t sortb = variable ? (size_t)N * 8 : 256 * 4;
    return base + sortb;
}

bsa_status launch_select(const bsa_kv_desc *d, const float *q, const void *summ, int kind,
                         const bsa_sel_params *p, const int32_t *cur_len, int nb_total,
                         int max_sel, int32_t *sel_blocks, int32_t *sel_count, int max_ranges,
                         int32_t *ranges, int32_t *n_ranges, uint32_t *keys, int32_t *vis,
                         uint32_t *counters, cudaStream_t st) {
    SelArgs a;
    a.q = q; a.summ = summ; a.cur_len = cur_len;
    const bool variable = p->block_size == 0;
    a.offsets = variable ? p->block_offsets : nullptr;
    a.kv_pos = variable ? p->kv_pos : nullptr;
    a.sel_blocks = sel_blocks; a.sel_count = sel_count; a.ranges = ranges; a.n_ranges = n_ranges;
    a.keys = keys; a.vis = vis; a.counters = counters;
    a.B = d->B; a.Hq = d->Hq; a.Hkv = d->Hkv; a.G = d->Hq / d->Hkv; a.D = d->D;
    a.L_max = d->L_max; a.S = p->block_size; a.nb_total = nb_total; a.kind = kind;
    a.topk = p->topk; a.budget = p->budget_tokens; a.sink = p->sink; a.window = p->window;
    a.keep_current = p->keep_current_block; a.local_start = p->local_start;
    a.pos_limit = p->pos_limit; a.max_sel = max_sel; a.max_ranges = max_ranges;
    size_t smem = select_smem_bytes(nb_total, max_sel, variable);
    if (smem > 200 * 1024) return BSA_ERR_UNSUPPORTED;
    dim3 grid((unsigned)div_up(nb_total, kSelThreads), d->B * d->Hkv);
    auto launch = [&](auto kern) -> bsa_status {
        if (smem > 48 * 1024)
            BSA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              (int)smem));
        kern<<<grid, kSelThreads, smem, st>>>(a);
        BSA_LAUNCH_CHECK();
        return BSA_OK;
    };
    if (kind == BSA_SUM_MINMAX)
        return d->kv_dtype == BSA_BF16 ? launch(select_kernel<BSA_SUM_MINMAX, uint16_t>)
                                       : launch(select_kernel<BSA_SUM_MINMAX, float>);
    if (kind == BSA_SUM_CENTROID) return launch(select_kernel<BSA_SUM_CENTROID, float>);
    return launch(select_kernel<BSA_SUM_CENTROID_NORM, float>);
}

}  // namespace bsa
