// A6 (per-query block selection and grouping) + A7 (block-grouped contraction
// on tcgen05 tensor cores) for the semantic-block prefill, sm_100a.
//
// "Semantic blocks for sparse attention": during prefill, neighbouring
// queries pick different blocks; instead of taking the union, the queries
// that need the same block are gathered and the block's keys and values are
// loaded once for the whole group.  The current fragment is attended densely
// and causally, and while the prefix is short the whole prefix is dense.
//
// Per call (one chunk of Tq queries at positions q_pos0 .. q_pos0+Tq-1):
//   P1 prefill_select_kernel  one warp per (query, KV head): scores the
//      KV head's block centres in the fixed fp32 order (as bsa_select) and
//      walks them greedily under the token budget; writes a selection bitmap
//      and appends the query to each selected block's list.
//   P2 prefill_tiles_kernel   prefix of 128-row tiles over (KV head, block).
//   P3 prefill_attend_kernel  persistent; work items are 128-row tiles:
//      local (32 queries x 4 heads against the position-ordered keys
//      [pos_limit, q], causal) and grouped (the gathered rows of one block
//      against its visible prefix).  Q rows are gathered into 128-byte-
//      swizzled shared memory, K/V tiles arrive by TMA (no multicast),
//      S = Q K^T accumulates in TMEM (tcgen05.mma, bf16 in, fp32 out), one
//      thread per row runs the online softmax and writes P (bf16) back to
//      TMEM, O += P V reads P from TMEM.  Each item leaves an unnormalised
//      partial (o, m, l) in its (query, KV head, slot) record.
//   P4 prefill_merge_kernel   log-sum-exp merge of a query's slots (local
//      first, then blocks in index order).
#include "common.cuh"

namespace bsa {

constexpr int kPfMaxBlocks = 256;          // blocks per KV head (bitmap of 8 words)
constexpr int kPfWords = kPfMaxBlocks / 32;
constexpr int kPfMaxSel = 64;              // selected blocks kept per (query, KV head)
constexpr int kPfSlots = kPfMaxSel + 1;    // slot 0 = local part
constexpr int kPfSelWarps = 16;            // P1 warps per CTA (8 when shared memory is short)
constexpr int kPfRowsPerWarp = 8;          // P1 query rows per warp
constexpr int kPfCentStride = 132;         // padded centre row (floats): 16-byte rows, conflict-free
constexpr int kTile = 128;                 // rows per MMA tile, keys per key tile
constexpr size_t kMaxSmemPerCta = 227 * 1024;   // opt-in dynamic shared memory per CTA
constexpr int kPfThreads = 128;
constexpr float kPfNegInf = -__builtin_huge_valf();
constexpr float kPfLn2 = 0.69314718055994530942f;

struct PfArgs {
    int Hq, Hkv, G, D, nb, L_max, Lpos;
    int Tq, q_pos0, pos_limit, budget;
    float scale_log2;
    const uint16_t *Q;         // [Tq][Hq][D] bf16
    const float *cent;         // [Hkv][nb][D]
    const int32_t *offsets;    // [Hkv][nb + 1]
    const int32_t *kv_pos;     // [Hkv][L_max]
    uint32_t *bitmap;          // [Tq][Hkv][kPfWords]
    int32_t *vis;              // [Hkv][nb]
    int32_t *qcount;           // [Hkv][nb]          (zeroed per call)
    int32_t *qlist;            // [Hkv][nb][Tq]
    int32_t *tile_prefix;      // [Hkv * nb + 1]
    int32_t *work;             // [1]                (zeroed per call)
    float *part_o;             // [Tq][Hkv][kPfSlots][G][D]
    float2 *part_ml;           // [Tq][Hkv][kPfSlots][G]
    uint32_t *status;
    float *out, *lse;          // [Tq][Hq][D], [Tq][Hq]
    int n_local;               // local work items
};

__device__ __forceinline__ int pf_visible(const int32_t *pos, int r0, int r1, int lim) {
    int lo = r0, hi = r1;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (pos[mid] < lim) lo = mid + 1; else hi = mid;
    }
    return lo - r0;
}

// ---------------------------------------------------------------- P1
__global__ void __launch_bounds__(32 * kPfSelWarps) prefill_select_kernel(PfArgs a) {
    extern __shared__ float psm[];
    const int D = a.D, G = a.G, nb = a.nb;
    const int nw = blockDim.x >> 5;
    float *cs = psm;                                   // [nb][kPfCentStride]
    float *qv = cs + nb * kPfCentStride;               // [nw][G][D]
    int *visS = reinterpret_cast<int *>(qv + nw * G * D);   // [nb]
    const int g = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_wait();
    const float *cg = a.cent + (int64_t)g * nb * D;
    for (int e = tid; e < nb * D; e += blockDim.x) cs[(e / D) * kPfCentStride + e % D] = cg[e];
    const int32_t *off = a.offsets + (int64_t)g * (nb + 1);
    const int32_t *pos = a.kv_pos + (int64_t)g * a.L_max;
    for (int j = tid; j < nb; j += blockDim.x) {
        const int r0 = min(max(off[j], 0), a.L_max), r1 = min(max(off[j + 1], r0), a.L_max);
        const int v = pf_visible(pos, r0, r1, a.pos_limit);
        visS[j] = v;
        if (blockIdx.x == 0) a.vis[g * nb + j] = v;
    }
    __syncthreads();
    float *qw = qv + warp * G * D;
    for (int r = 0; r < kPfRowsPerWarp; ++r) {
        const int i = (blockIdx.x * nw + warp) * kPfRowsPerWarp + r;
        if (i >= a.Tq) break;
        const uint16_t *qi = a.Q + ((int64_t)i * a.Hq + (int64_t)g * G) * D;
        for (int e = lane; e < G * D; e += 32) qw[e] = bf16_to_f32(qi[e]);
        __syncwarp();
        // lane owns blocks lane + 32 t; composite keys (orderable score, ~index).
        // The (block, head) fma chains are interleaved over d for ILP; each
        // chain still runs d = 0..D-1 in order.
        unsigned long long key[kPfWords];
        {
            constexpr int kMaxGh = 4;   // heads accumulated together per pass
            float tot[kPfWords];
            for (int h0 = 0; h0 < G; h0 += kMaxGh) {
                float acc[kPfWords][kMaxGh];
#pragma unroll
                for (int t = 0; t < kPfWords; ++t)
#pragma unroll
                    for (int h = 0; h < kMaxGh; ++h) acc[t][h] = 0.0f;
                for (int d = 0; d < D; d += 4) {
                    float4 qd[kMaxGh];
#pragma unroll
                    for (int h = 0; h < kMaxGh; ++h)
                        qd[h] = h0 + h < G ? *reinterpret_cast<const float4 *>(qw + (h0 + h) * D + d)
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int t = 0; t < kPfWords; ++t) {
                        const int j = min(lane + 32 * t, nb - 1);
                        const float4 c = *reinterpret_cast<const float4 *>(cs + j * kPfCentStride + d);
#pragma unroll
                        for (int h = 0; h < kMaxGh; ++h) {
                            acc[t][h] = __fmaf_rn(qd[h].x, c.x, acc[t][h]);
                            acc[t][h] = __fmaf_rn(qd[h].y, c.y, acc[t][h]);
                            acc[t][h] = __fmaf_rn(qd[h].z, c.z, acc[t][h]);
                            acc[t][h] = __fmaf_rn(qd[h].w, c.w, acc[t][h]);
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < kPfWords; ++t)
#pragma unroll
                    for (int h = 0; h < kMaxGh; ++h)
                        if (h0 + h < G) tot[t] = (h0 + h == 0) ? acc[t][h] : __fadd_rn(tot[t], acc[t][h]);
            }
#pragma unroll
            for (int t = 0; t < kPfWords; ++t) {
                key[t] = 0ull;
                const int j = lane + 32 * t;
                // only candidates that can ever fit the budget
                if (j < nb && visS[j] > 0 && visS[j] <= a.budget) {
                    uint32_t k32 = f32_order_key(__fadd_rn(tot[t], 0.0f));
                    if (k32 == 0) k32 = 1;
                    key[t] = ((unsigned long long)k32 << 32) | (0xffffffffu - (uint32_t)j);
                }
            }
        }
        // greedy walk in rank order: take a block when its visible rows fit.
        // What is left of the budget only shrinks, so a block that does not
        // fit now never will: after each take such blocks are dropped, and the
        // best remaining candidate always fits.
        uint32_t selbits = 0;   // bit t: block lane + 32 t selected
        int remaining = a.budget, nsel = 0;
        while (nsel < kPfMaxSel) {
            unsigned long long best = 0ull;
#pragma unroll
            for (int t = 0; t < kPfWords; ++t) best = key[t] > best ? key[t] : best;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
                best = other > best ? other : best;
            }
            if (best == 0ull) break;
            const int j = (int)(0xffffffffu - (uint32_t)(best & 0xffffffffu));
            remaining -= visS[j];
            ++nsel;
            if (lane == (j & 31)) selbits |= 1u << (j >> 5);
            if (lane == 0) {
                const int p = atomicAdd(&a.qcount[g * nb + j], 1);
                a.qlist[((int64_t)g * nb + j) * a.Tq + p] = i;
            }
#pragma unroll
            for (int t = 0; t < kPfWords; ++t) {
                const int jj = lane + 32 * t;
                if (key[t] && (jj == j || visS[jj] > remaining)) key[t] = 0ull;
            }
        }
        if (nsel >= kPfMaxSel && lane == 0) atomicOr(a.status, 4u);
        uint32_t *bm = a.bitmap + ((int64_t)i * a.Hkv + g) * kPfWords;
#pragma unroll
        for (int t = 0; t < kPfWords; ++t) {
            const uint32_t word = __ballot_sync(0xffffffffu, (selbits >> t) & 1u);
            if (lane == 0) bm[t] = word;
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------- P2
__global__ void __launch_bounds__(1024) prefill_tiles_kernel(PfArgs a) {
    __shared__ int tmp[40];
    const int n = a.Hkv * a.nb;
    int carry = 0;
    for (int base = 0; base < n; base += blockDim.x) {
        const int e = base + threadIdx.x;
        const int t = e < n ? (a.qcount[e] * a.G + kTile - 1) / kTile : 0;
        int tot;
        const int ex = cta_excl_sum(t, tmp, &tot);
        if (e < n) a.tile_prefix[e] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0) a.tile_prefix[n] = carry;
}

// ---------------------------------------------------------------- P3
// Warp-specialised: warps 0..7 run the softmax, two threads per row (warp w
// owns TMEM lanes 32*(w%4).. and the column half w/4); lane 0 of warp 8
// issues every TMA load and every tcgen05.mma.  S is double-buffered in TMEM
// so that S(t+1) = Q K(t+1)^T runs on the tensor cores while the softmax of
// tile t runs; P.V of tile t follows the softmax.  O is rescaled only when a
// row's running maximum grows by more than 2^8 (the exponentials then stay
// below 256), so P.V rarely sits on the softmax's critical path.
constexpr int kPfSoftWarps = 8;
constexpr int kPfAttThreads = 32 * (kPfSoftWarps + 1);
constexpr float kPfRescale = 8.0f;   // log2 of the largest exponential kept without rescaling

struct PfSmem {
    static constexpr int kQ = 0;                          // 2 boxes x 16 KiB
    static constexpr int kK = 32768;                      // 2 stages x 32 KiB
    static constexpr int kV = kK + 2 * 32768;             // 2 stages x 32 KiB
    static constexpr int kRowQ = kV + 2 * 32768;          // int [128] query index
    static constexpr int kRowPos = kRowQ + kTile * 4;     // int [128] query position
    static constexpr int kPair = kRowPos + kTile * 4;     // float [2][128] half-row maxima / sums
    static constexpr int kBars = kPair + 2 * kTile * 4;   // u64: kfull[2] vfull[2] sfull[2] pfull[2] odone[2]
    static constexpr int kMisc = kBars + 10 * 8;          // int item, tmem base
    static constexpr int kBytes = kMisc + 16 + 1024;
};

struct PfItem {
    int g, kbeg, kend, jblk, mtile, ntiles;
    bool local;
};

__device__ __forceinline__ void pair_sync(int q) {   // the two warps holding rows 32q..32q+31
    asm volatile("bar.sync %0, 64;" ::"r"(1 + q) : "memory");
}

__global__ void __launch_bounds__(kPfAttThreads, 1)
    prefill_attend_kernel(const __grid_constant__ CUtensorMap tmKp, const __grid_constant__ CUtensorMap tmVp,
                          const __grid_constant__ CUtensorMap tmKl, const __grid_constant__ CUtensorMap tmVl,
                          PfArgs a) {
    extern __shared__ unsigned char praw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(praw) + 1023) & ~uintptr_t(1023));
    unsigned char *Qs = sm + PfSmem::kQ;
    int *rowq = reinterpret_cast<int *>(sm + PfSmem::kRowQ);
    int *rowpos = reinterpret_cast<int *>(sm + PfSmem::kRowPos);
    float *pairv = reinterpret_cast<float *>(sm + PfSmem::kPair);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + PfSmem::kBars);
    uint64_t *kfull = bars, *vfull = bars + 2, *sfull = bars + 4, *pfull = bars + 6, *odone = bars + 8;   // odone[2]
    int *item_sh = reinterpret_cast<int *>(sm + PfSmem::kMisc);
    uint32_t *tmem_sh = reinterpret_cast<uint32_t *>(sm + PfSmem::kMisc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.G, D = a.D;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
            smem_u32(tmem_sh)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        prefetch_tmap(&tmKp); prefetch_tmap(&tmVp); prefetch_tmap(&tmKl); prefetch_tmap(&tmVl);
        for (int i = 0; i < 6; ++i) mbar_init(&bars[i], 1);
        mbar_init(&pfull[0], kPfSoftWarps);
        mbar_init(&pfull[1], kPfSoftWarps);
        mbar_init(&odone[0], 1);
        mbar_init(&odone[1], 1);
        fence_mbar_init();
    }
    pdl_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_sh;
    const uint32_t tO = tmem + 256;                 // S0 = cols 0..127, S1 = 128..255, O = 256..383
    const int n_group = a.tile_prefix[a.Hkv * a.nb];
    const int n_items = a.n_local + n_group;
    const int qpt = kTile / G;
    const int tiles_per_head = (a.Tq + qpt - 1) / qpt;
    constexpr uint32_t kIdescQK = umma_idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t kIdescPV = umma_idesc_bf16(128, 128, 0, 1);
    // phase counters (every role tracks the barriers it waits on)
    uint32_t kuse[2] = {0, 0}, vuse[2] = {0, 0}, puse[2] = {0, 0};   // issuing lane only
    uint32_t sbase[2] = {0, 0}, obase[2] = {0, 0};                       // every thread
    bool timed_out = false;

    for (;;) {
        if (tid == 0) *item_sh = atomicAdd(a.work, 1);
        __syncthreads();
        const int item = *item_sh;
        if (item >= n_items) break;
        // ---- decode the work item (every thread, same result)
        PfItem it;
        it.local = item < a.n_local;
        it.jblk = -1;
        if (it.local) {
            it.g = item / tiles_per_head;
            const int i0 = (item % tiles_per_head) * qpt;
            it.mtile = i0;
            it.kbeg = a.pos_limit;
            it.kend = a.q_pos0 + min(a.Tq, i0 + qpt);
        } else {
            const int u = item - a.n_local;
            int lo = 0, hi = a.Hkv * a.nb - 1;   // largest e with prefix[e] <= u
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (a.tile_prefix[mid] <= u) lo = mid; else hi = mid - 1;
            }
            it.g = lo / a.nb;
            it.jblk = lo % a.nb;
            it.mtile = u - a.tile_prefix[lo];
            it.kbeg = min(max(a.offsets[(int64_t)it.g * (a.nb + 1) + it.jblk], 0), a.L_max);
            it.kend = it.kbeg + a.vis[it.g * a.nb + it.jblk];
        }
        it.ntiles = max(0, (it.kend - it.kbeg + kTile - 1) / kTile);
        const int g = it.g;
        if (tid < kTile) {
            const int r = tid;
            if (it.local) {
                const int i = it.mtile + r / G;
                rowq[r] = i < a.Tq ? i : -1;
                rowpos[r] = a.q_pos0 + i;
            } else {
                const int cnt = a.qcount[g * a.nb + it.jblk];
                const int idx = it.mtile * kTile + r, qi = idx / G;
                rowq[r] = qi < cnt ? a.qlist[((int64_t)g * a.nb + it.jblk) * a.Tq + qi] : -1;
                rowpos[r] = 0x7fffffff;   // every key of a visible prefix is earlier
            }
        }
        __syncthreads();
        // ---- gather Q rows (bf16) into the swizzled K-major layout
        for (int c = tid; c < kTile * 16; c += kPfAttThreads) {
            const int r = c >> 4, ch = c & 15, half = ch >> 3, cc = ch & 7;
            const int qi = rowq[r];
            uint4 v = make_uint4(0, 0, 0, 0);
            if (qi >= 0) {
                const int hh = r % G;
                v = *reinterpret_cast<const uint4 *>(
                    a.Q + ((int64_t)qi * a.Hq + (int64_t)g * G + hh) * D + ch * 8);
            }
            *reinterpret_cast<uint4 *>(Qs + half * 16384 + r * 128 + ((cc ^ (r & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        const int T = it.ntiles;

        // Barrier protocol.  kfull/vfull/pfull are waited by the issuing lane
        // for every phase (plain counters).  S(t) completes on sfull[t&1] and
        // P.V(t) on odone[t&1]; a wait for one of them is for a specific MMA
        // whose predecessor on the same barrier is already known complete, so
        // the parity follows from the MMA's index: base[b] (MMAs on barrier b
        // in earlier items) + t/2.
        auto par = [](uint32_t base, int t) { return (base + (uint32_t)(t >> 1)) & 1u; };
        if (warp == kPfSoftWarps) {
            // ================= TMA + MMA issue (one lane)
            if (lane == 0) {
                const CUtensorMap *mk = it.local ? &tmKl : &tmKp;
                const CUtensorMap *mv = it.local ? &tmVl : &tmVp;
                auto load_k = [&](int t) {
                    unsigned char *dst = sm + PfSmem::kK + (t & 1) * 32768;
                    mbar_arrive_expect_tx(&kfull[t & 1], 32768);
                    tma_load_4d(dst, mk, &kfull[t & 1], 0, it.kbeg + t * kTile, g, 0);
                    tma_load_4d(dst + 16384, mk, &kfull[t & 1], 64, it.kbeg + t * kTile, g, 0);
                };
                auto load_v = [&](int t) {
                    unsigned char *dst = sm + PfSmem::kV + (t & 1) * 32768;
                    mbar_arrive_expect_tx(&vfull[t & 1], 32768);
                    tma_load_4d(dst, mv, &vfull[t & 1], 0, it.kbeg + t * kTile, g, 0);
                    tma_load_4d(dst + 16384, mv, &vfull[t & 1], 64, it.kbeg + t * kTile, g, 0);
                };
                auto pv = [&](int t) {   // O (+)= P(t) V(t), P read from S(t & 1)
                    if (!timed_out && !mbar_wait_bounded(&pfull[t & 1], puse[t & 1] & 1)) timed_out = true;
                    ++puse[t & 1];
                    if (!timed_out && !mbar_wait_bounded(&vfull[t & 1], vuse[t & 1] & 1)) timed_out = true;
                    ++vuse[t & 1];
                    tc_fence_after();
                    const uint32_t v0 = smem_u32(sm + PfSmem::kV + (t & 1) * 32768);
                    const uint32_t tP = tmem + (t & 1) * 128;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint64_t vd = umma_sdesc_sw128(v0 + k * 2048, 16384, 1024);
                        umma_ts(tO, tP + k * 8, vd, kIdescPV, (t > 0 || k > 0) ? 1u : 0u);
                        umma_ts(tO, tP + 64 + k * 8, vd, kIdescPV, 1u);
                    }
                    umma_commit(&odone[t & 1]);
                };
                for (int t = 0; t < 2 && t < T; ++t) { load_k(t); load_v(t); }
                for (int t = 0; t < T; ++t) {
                    if (!timed_out && !mbar_wait_bounded(&kfull[t & 1], kuse[t & 1] & 1)) timed_out = true;
                    ++kuse[t & 1];
                    if (t >= 2) {   // S(t&1) and V stage t&1 are free once P.V(t-2) is done
                        if (!timed_out && !mbar_wait_bounded(&odone[t & 1], par(obase[t & 1], t - 2))) timed_out = true;
                        load_v(t);
                    }
                    tc_fence_after();
                    const uint32_t q0 = smem_u32(Qs);
                    const uint32_t k0 = smem_u32(sm + PfSmem::kK + (t & 1) * 32768);
                    const uint32_t tS = tmem + (t & 1) * 128;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
                        umma_ss(tS, umma_sdesc_sw128(q0 + off, 16, 1024),
                                umma_sdesc_sw128(k0 + off, 16, 1024), kIdescQK, k > 0);
                    }
                    umma_commit(&sfull[t & 1]);
                    if (t + 2 < T) {   // K stage t&1 is free once S(t) is done
                        if (!timed_out && !mbar_wait_bounded(&sfull[t & 1], par(sbase[t & 1], t))) timed_out = true;
                        load_k(t + 2);
                    }
                    if (t >= 1) pv(t - 1);
                }
                if (T >= 1) pv(T - 1);
            }
            __syncwarp();
        } else {
            // ================= softmax warps
            const int q = warp & 3, half = warp >> 2;
            const int r = q * 32 + lane;                 // this thread's row
            const uint32_t lane_base = (uint32_t)(q * 32) << 16;
            const int my_pos = rowpos[r];
            float m_used = kPfNegInf, l_part = 0.0f;
            for (int t = 0; t < T; ++t) {
                if (!timed_out && !mbar_wait_bounded(&sfull[t & 1], par(sbase[t & 1], t))) timed_out = true;
                tc_fence_after();
                const uint32_t tS = tmem + (t & 1) * 128;
                uint32_t sv[2][32];
                tmem_ld32(tS + lane_base + half * 64, sv[0]);
                tmem_ld32(tS + lane_base + half * 64 + 32, sv[1]);
                tmem_ld_wait();
                const int key0 = it.kbeg + t * kTile + half * 64;
                float mx = kPfNegInf;
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int kr = key0 + c2 * 32 + e;
                        const bool ok = kr < it.kend && kr <= my_pos;
                        const float v = ok ? __uint_as_float(sv[c2][e]) * a.scale_log2 : kPfNegInf;
                        sv[c2][e] = __float_as_uint(v);
                        mx = fmaxf(mx, v);
                    }
                // both halves of the row have read S(t) before either writes P
                pairv[half * kTile + r] = mx;
                pair_sync(q);
                const float m_tile = fmaxf(pairv[r], pairv[kTile + r]);
                pair_sync(q);
                // lazy rescale: keep the reference maximum unless this tile
                // exceeds it by more than 2^8
                bool rescale = false;
                float factor = 1.0f, m_ref = m_used;
                if (m_tile != kPfNegInf) {
                    if (m_used == kPfNegInf) {
                        m_ref = m_tile;   // nothing accumulated yet for this row
                    } else if (m_tile > m_used + kPfRescale) {
                        rescale = true;
                        factor = exp2f(m_used - m_tile);
                        m_ref = m_tile;
                    }
                }
                if (t > 0 && __any_sync(0xffffffffu, rescale)) {
                    // O must hold P.V(t-1) before it is scaled
                    if (!timed_out && !mbar_wait_bounded(&odone[(t - 1) & 1], par(obase[(t - 1) & 1], t - 1)))
                        timed_out = true;
                    tc_fence_after();
#pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2) {
                        uint32_t ov[32];
                        tmem_ld32(tO + lane_base + half * 64 + c2 * 32, ov);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            ov[e] = __float_as_uint(__uint_as_float(ov[e]) * factor);
                        tmem_st32(tO + lane_base + half * 64 + c2 * 32, ov);
                    }
                }
                l_part *= factor;
                m_used = m_ref;
                // P = P_hi + P_lo (bf16) over this half's 64 keys: P_hi in the
                // tile's S columns 32*half.., P_lo in 64 + 32*half..
                float lsum = 0.0f;
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    uint32_t ph[16], pl[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const float p0 = m_used == kPfNegInf ? 0.0f : exp2f(__uint_as_float(sv[c2][e]) - m_used);
                        const float p1 = m_used == kPfNegInf ? 0.0f : exp2f(__uint_as_float(sv[c2][e + 1]) - m_used);
                        lsum += p0 + p1;
                        const float h0 = bf16_round(p0), h1 = bf16_round(p1);
                        ph[e / 2] = pack_bf16x2(h0, h1);
                        pl[e / 2] = pack_bf16x2(p0 - h0, p1 - h1);
                    }
                    tmem_st16(tS + lane_base + half * 32 + c2 * 16, ph);
                    tmem_st16(tS + lane_base + 64 + half * 32 + c2 * 16, pl);
                }
                l_part += lsum;
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&pfull[t & 1]);
            }
            // ---- epilogue: wait for the last two P.V, then this item's partial
            if (T >= 1 && !timed_out && !mbar_wait_bounded(&odone[(T - 1) & 1], par(obase[(T - 1) & 1], T - 1)))
                timed_out = true;
            if (T >= 2 && !timed_out && !mbar_wait_bounded(&odone[(T - 2) & 1], par(obase[(T - 2) & 1], T - 2)))
                timed_out = true;
            tc_fence_after();
            pairv[half * kTile + r] = l_part;
            pair_sync(q);
            const float l_row = pairv[r] + pairv[kTile + r];
            pair_sync(q);
            const int qi = rowq[r];
            int64_t rec = -1;
            if (qi >= 0) {
                int slot = 0;
                if (!it.local) {
                    const uint32_t *bm = a.bitmap + ((int64_t)qi * a.Hkv + g) * kPfWords;
                    for (int w = 0; w < (it.jblk >> 5); ++w) slot += __popc(bm[w]);
                    slot += __popc(bm[it.jblk >> 5] & ((1u << (it.jblk & 31)) - 1u)) + 1;
                }
                if (slot < kPfSlots)
                    rec = (((int64_t)qi * a.Hkv + g) * kPfSlots + slot) * G + (r % G);
            }
            float *po = rec >= 0 ? a.part_o + rec * D + half * 64 : nullptr;
            if (T > 0) {
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    uint32_t ov[32];
                    tmem_ld32(tO + lane_base + half * 64 + c2 * 32, ov);
                    tmem_ld_wait();
                    if (po) {
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4 *>(po + c2 * 32 + e) =
                                make_float4(__uint_as_float(ov[e]), __uint_as_float(ov[e + 1]),
                                            __uint_as_float(ov[e + 2]), __uint_as_float(ov[e + 3]));
                    }
                }
            } else if (po) {
                for (int d = 0; d < 64; ++d) po[d] = 0.0f;
            }
            if (rec >= 0 && half == 0) a.part_ml[rec] = make_float2(m_used, l_row);
        }
        // every role advances the per-barrier MMA counts by this item's tiles
        sbase[0] += (uint32_t)((T + 1) >> 1);
        sbase[1] += (uint32_t)(T >> 1);
        obase[0] += (uint32_t)((T + 1) >> 1);
        obase[1] += (uint32_t)(T >> 1);
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (timed_out) atomicOr(a.status, 8u);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
}

// ---------------------------------------------------------------- P4
__global__ void __launch_bounds__(128) prefill_merge_kernel(PfArgs a) {
    pdl_wait();
    const int i = blockIdx.x, g = blockIdx.y, G = a.G, D = a.D;
    const uint32_t *bm = a.bitmap + ((int64_t)i * a.Hkv + g) * kPfWords;
    int nsel = 0;
    for (int w = 0; w < kPfWords; ++w) nsel += __popc(bm[w]);
    const int nslot = min(1 + nsel, kPfSlots);
    const int D4 = D / 4;
    // one thread per (head, 4 dimensions); slots merged in slot order, with
    // all of a pass's loads independent of one another
    for (int e = threadIdx.x; e < G * D4; e += blockDim.x) {
        const int hh = e / D4, d4 = e % D4;
        const int64_t rec0 = ((int64_t)i * a.Hkv + g) * kPfSlots * G + hh;
        float M = kPfNegInf;
#pragma unroll 8
        for (int s = 0; s < nslot; ++s) M = fmaxf(M, __ldcg(&a.part_ml[rec0 + (int64_t)s * G]).x);
        float L = 0.0f;
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int s = 0; s < nslot; ++s) {
            const int64_t rec = rec0 + (int64_t)s * G;
            const float2 ml = __ldcg(&a.part_ml[rec]);
            const float4 ov = __ldcg(reinterpret_cast<const float4 *>(a.part_o + rec * D) + d4);
            const float w = ml.x != kPfNegInf ? exp2f(ml.x - M) : 0.0f;
            L += ml.y * w;
            O.x += ov.x * w; O.y += ov.y * w; O.z += ov.z * w; O.w += ov.w * w;
        }
        const int64_t orow = (int64_t)i * a.Hq + (int64_t)g * G + hh;
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        reinterpret_cast<float4 *>(a.out + orow * D)[d4] =
            make_float4(O.x * inv, O.y * inv, O.z * inv, O.w * inv);
        if (d4 == 0 && a.lse) a.lse[orow] = L > 0.0f ? (M + log2f(L)) * kPfLn2 : kPfNegInf;
    }
}

// ---------------------------------------------------------------- host
struct PfLayout {
    size_t bitmap, vis, qcount, qlist, prefix, work, part_o, part_ml, total;
};

static PfLayout pf_layout(const bsa_kv_desc *d, const bsa_sel_params *p, int Tq) {
    PfLayout L;
    const size_t G = d->Hq / d->Hkv, nb = p->n_blocks, H = d->Hkv;
    size_t o = 0;
    L.bitmap = o;  o += align_up((size_t)Tq * H * kPfWords * 4, 256);
    L.vis = o;     o += align_up(H * nb * 4, 256);
    L.qcount = o;  o += align_up(H * nb * 4, 256);
    L.work = o;    o += 256;
    L.qlist = o;   o += align_up(H * nb * (size_t)Tq * 4, 256);
    L.prefix = o;  o += align_up((H * nb + 1) * 4, 256);
    L.part_o = o;  o += align_up((size_t)Tq * H * kPfSlots * G * d->D * 4, 256);
    L.part_ml = o; o += align_up((size_t)Tq * H * kPfSlots * G * 8, 256);
    L.total = o;
    return L;
}

size_t prefill_ws_bytes(const bsa_kv_desc *d, const bsa_sel_params *p, int Tq) {
    return pf_layout(d, p, Tq).total;
}

bsa_status launch_prefill(const bsa_kv_desc *d, const void *K, const void *V,
                          const bsa_sel_params *p, const void *summaries, const bsa_kv_desc *pd,
                          const void *K_pos, const void *V_pos, const void *Q, int q_pos0, int Tq,
                          float scale, float *out, float *lse, uint32_t *status, void *ws,
                          size_t ws_bytes, cudaStream_t st) {
    const int G = d->Hq / d->Hkv;
    if (p->n_blocks > kPfMaxBlocks || kTile % G != 0 || G > 16) return BSA_ERR_UNSUPPORTED;
    const PfLayout L = pf_layout(d, p, Tq);
    if (ws_bytes < L.total) return BSA_ERR_WORKSPACE;
    char *w = static_cast<char *>(ws);
    PfArgs a;
    a.Hq = d->Hq; a.Hkv = d->Hkv; a.G = G; a.D = d->D; a.nb = p->n_blocks;
    a.L_max = d->L_max; a.Lpos = pd->L_max;
    a.Tq = Tq; a.q_pos0 = q_pos0; a.pos_limit = p->pos_limit; a.budget = p->budget_tokens;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.Q = static_cast<const uint16_t *>(Q);
    a.cent = static_cast<const float *>(summaries);
    a.offsets = p->block_offsets;
    a.kv_pos = p->kv_pos;
    a.bitmap = reinterpret_cast<uint32_t *>(w + L.bitmap);
    a.vis = reinterpret_cast<int32_t *>(w + L.vis);
    a.qcount = reinterpret_cast<int32_t *>(w + L.qcount);
    a.qlist = reinterpret_cast<int32_t *>(w + L.qlist);
    a.tile_prefix = reinterpret_cast<int32_t *>(w + L.prefix);
    a.work = reinterpret_cast<int32_t *>(w + L.work);
    a.part_o = reinterpret_cast<float *>(w + L.part_o);
    a.part_ml = reinterpret_cast<float2 *>(w + L.part_ml);
    a.status = status;
    a.out = out; a.lse = lse;
    const int qpt = kTile / G;
    a.n_local = d->Hkv * ((Tq + qpt - 1) / qpt);

    CUtensorMap kp, vp, kl, vl;
    if (!make_kv_tmap(&kp, d, K, kTile) || !make_kv_tmap(&vp, d, V, kTile) ||
        !make_kv_tmap(&kl, pd, K_pos, kTile) || !make_kv_tmap(&vl, pd, V_pos, kTile))
        return BSA_ERR_CUDA;
    // zero the per-block counts and the work counter
    BSA_CUDA_TRY(cudaMemsetAsync(w + L.qcount, 0, (size_t)d->Hkv * p->n_blocks * 4, st));
    BSA_CUDA_TRY(cudaMemsetAsync(w + L.work, 0, 4, st));
    // P1: selection
    auto smem1_for = [&](int nw) {
        return ((size_t)a.nb * kPfCentStride + (size_t)nw * G * a.D + a.nb) * 4;
    };
    const int nw1 = smem1_for(kPfSelWarps) <= kMaxSmemPerCta ? kPfSelWarps : kPfSelWarps / 2;
    const size_t smem1 = smem1_for(nw1);
    BSA_CUDA_TRY(cudaFuncSetAttribute(prefill_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem1));
    BSA_CUDA_TRY(launch_pdl(prefill_select_kernel,
                            dim3((unsigned)div_up(Tq, nw1 * kPfRowsPerWarp), (unsigned)d->Hkv),
                            dim3(32 * nw1), smem1, st, a));
    // P2: tile prefix over (KV head, block)
    prefill_tiles_kernel<<<1, 1024, 0, st>>>(a);
    BSA_LAUNCH_CHECK();
    // P3: persistent tensor-core attention over local and grouped tiles
    BSA_CUDA_TRY(cudaFuncSetAttribute(prefill_attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      PfSmem::kBytes));
    prefill_attend_kernel<<<num_sms(), kPfAttThreads, PfSmem::kBytes, st>>>(kp, vp, kl, vl, a);
    BSA_LAUNCH_CHECK();
    // P4: merge of every query's slots
    BSA_CUDA_TRY(launch_pdl(prefill_merge_kernel, dim3((unsigned)Tq, (unsigned)d->Hkv), dim3(128), 0,
                            st, a));
    return BSA_OK;
}

}  // namespace bsa
