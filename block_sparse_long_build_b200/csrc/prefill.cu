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
//      S = Q K^T accumulates in TMEM (tcgen05.mma, bf16 in, fp32 out), four
//      threads per row run the online softmax and write P (fp16) back to
//      TMEM, and O += P V reads P from TMEM with the V tile converted to
//      fp16 in shared memory (the two operands of one product share a type).  Each item leaves an unnormalised
//      partial (o, m, l) in its (query, KV head, slot) record.
//   P4 prefill_merge_kernel   log-sum-exp merge of a query's slots (local
//      first, then blocks in index order).
#include "common.cuh"

namespace bsa {

constexpr int kPfMaxBlocks = 256;          // blocks per KV head (bitmap of 8 words)
constexpr int kPfWords = kPfMaxBlocks / 32;
constexpr int kPfMaxSel = 64;              // selected blocks kept per (query, KV head)
constexpr int kPfSlots = kPfMaxSel + 1;    // slot 0 = local part
constexpr int kPfSlotShift = 24;           // qlist entry: query | slot << 24
constexpr int kPfSelWarps = 16;            // P1 warps per CTA (fewer when shared memory is short)
constexpr int kPfMergeThreads = 128;       // P4 threads per CTA
constexpr int kPfD = 128;                  // head dimension of the prefill path
constexpr int kPfCentStride = 132;         // padded centre row (floats): 16-byte rows, conflict-free
constexpr int kTile = 128;                 // rows per MMA tile, keys per key tile
constexpr size_t kMaxSmemPerCta = 227 * 1024;   // opt-in dynamic shared memory per CTA
constexpr float kPfNegInf = -__builtin_huge_valf();
constexpr float kPfLn2 = 0.69314718055994530942f;

struct PfArgs {
    int Hq, Hkv, G, D, nb, L_max, Lpos;
    int Tq, q_pos0, pos_limit, budget;
    int pos_base;              // position of row 0 of the position-ordered K/V
    float scale_log2;
    const uint16_t *Q;         // [Tq][Hq][D] bf16
    const float *cent;         // [Hkv][nb][D]
    const int32_t *offsets;    // [Hkv][nb + 1]
    const int32_t *kv_pos;     // [Hkv][L_max]
    uint32_t *bitmap;          // [Tq][Hkv][kPfWords]
    int32_t *vis;              // [Hkv][nb]
    int32_t *qcount;           // [Hkv][nb]          (zeroed per call)
    int32_t *qlist;            // [Hkv][nb][Tq]       query | slot << kPfSlotShift
    int32_t *tile_prefix;      // [Hkv * nb + 1]
    float *part_o;             // [Tq][Hkv][kPfSlots][G][D]
    float2 *part_ml;           // [Tq][Hkv][kPfSlots][G]
    uint32_t *status;
    float *out, *lse;          // [Tq][Hq][D], [Tq][Hq]
    int n_local;               // local work items
    int sel_rows_per_warp;     // P1: query rows per warp (one wave of CTAs)
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
    uint16_t *qst = reinterpret_cast<uint16_t *>(qv + nw * G * D);   // [nw][G][D] bf16 staging
    int *visS = reinterpret_cast<int *>(qst + nw * G * D);           // [nb]
    const int g = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rpw = a.sel_rows_per_warp, row0 = (blockIdx.x * nw + warp) * rpw;
    float *qw = qv + warp * G * D;
    uint16_t *qs = qst + warp * G * D;
    // query row i's G heads (bf16) into this warp's staging buffer, 16 bytes a copy
    auto stage_q = [&](int i) {
        const uint16_t *qi = a.Q + ((int64_t)i * a.Hq + (int64_t)g * G) * D;
        for (int e = 8 * lane; e < G * D; e += 256)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(qs + e)), "l"(qi + e)
                         : "memory");
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    pdl_wait();
    // centres into padded rows, asynchronously, while the visible counts are searched
    const float *cg = a.cent + (int64_t)g * nb * D;
    for (int e = 4 * tid; e < nb * D; e += 4 * blockDim.x)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                         smem_u32(cs + (e / D) * kPfCentStride + e % D)),
                     "l"(cg + e)
                     : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
    if (row0 < a.Tq) stage_q(row0);
    const int32_t *off = a.offsets + (int64_t)g * (nb + 1);
    const int32_t *pos = a.kv_pos + (int64_t)g * a.L_max;
    for (int j = tid; j < nb; j += blockDim.x) {
        const int r0 = min(max(off[j], 0), a.L_max), r1 = min(max(off[j + 1], r0), a.L_max);
        const int v = pf_visible(pos, r0, r1, a.pos_limit);
        visS[j] = v;
        if (blockIdx.x == 0) a.vis[g * nb + j] = v;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    // this lane's centre rows (blocks lane + 32 t)
    int crow[kPfWords], vr[kPfWords];   // vr: visible rows (INT_MAX past the last block)
#pragma unroll
    for (int t = 0; t < kPfWords; ++t) {
        crow[t] = min(lane + 32 * t, nb - 1) * kPfCentStride;
        vr[t] = lane + 32 * t < nb ? visS[lane + 32 * t] : 0x7fffffff;
    }
    for (int r = 0; r < rpw; ++r) {
        const int i = row0 + r;
        if (i >= a.Tq) break;
        // row i is staged (the wait covers this lane's copies, the warp
        // barrier everyone's); widen it, then stage row i + 1 behind the work
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncwarp();
        for (int e = 4 * lane; e < G * D; e += 128) {
            const uint2 u = *reinterpret_cast<const uint2 *>(qs + e);
            *reinterpret_cast<float4 *>(qw + e) =
                make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                            __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
        }
        __syncwarp();
        if (r + 1 < rpw && i + 1 < a.Tq) stage_q(i + 1);
        // lane owns blocks lane + 32 t; sk[t] = orderable score key of block
        // lane + 32 t (0: not a candidate). The (block, head) fma chains are
        // interleaved over d for ILP; each chain still runs d = 0..D-1 in order.
        uint32_t sk[kPfWords];
        {
            constexpr int kMaxGh = 4;   // heads accumulated together per pass
            float tot[kPfWords];
            for (int h0 = 0; h0 < G; h0 += kMaxGh) {
                float acc[kPfWords][kMaxGh];
#pragma unroll
                for (int t = 0; t < kPfWords; ++t)
#pragma unroll
                    for (int h = 0; h < kMaxGh; ++h) acc[t][h] = 0.0f;
#pragma unroll 1
                for (int d = 0; d < kPfD; d += 4) {
                    float4 qd[kMaxGh];
#pragma unroll
                    for (int h = 0; h < kMaxGh; ++h)
                        qd[h] = h0 + h < G ? *reinterpret_cast<const float4 *>(qw + (h0 + h) * kPfD + d)
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int t = 0; t < kPfWords; ++t) {
                        const float4 c = *reinterpret_cast<const float4 *>(cs + crow[t] + d);
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
                sk[t] = 0u;
                // only candidates that can ever fit the budget
                if (vr[t] > 0 && vr[t] <= a.budget) {
                    const uint32_t k32 = f32_order_key(__fadd_rn(tot[t], 0.0f));
                    sk[t] = k32 ? k32 : 1u;
                }
            }
        }
        // greedy walk in rank order: take a block when its visible rows fit.
        // What is left of the budget only shrinks, so a block that does not
        // fit now never will: after each take such blocks are dropped, and the
        // best remaining candidate always fits.
        // The best candidate is the highest key, ties to the lowest block
        // index: a warp max of the keys, then a warp min of the indices that
        // hold it.
        uint32_t selbits = 0;   // bit t: block lane + 32 t selected
        int remaining = a.budget, nsel = 0;
        while (nsel < kPfMaxSel) {
            uint32_t lm = 0u;
#pragma unroll
            for (int t = 0; t < kPfWords; ++t) lm = max(lm, sk[t]);
            const uint32_t m = __reduce_max_sync(0xffffffffu, lm);
            if (m == 0u) break;
            int cand = 0x7fffffff;
#pragma unroll
            for (int t = kPfWords - 1; t >= 0; --t) cand = sk[t] == m ? lane + 32 * t : cand;
            const int j = __reduce_min_sync(0xffffffffu, cand);
            remaining -= visS[j];
            ++nsel;
            if (lane == (j & 31)) selbits |= 1u << (j >> 5);
#pragma unroll
            for (int t = 0; t < kPfWords; ++t)
                if (lane + 32 * t == j || vr[t] > remaining) sk[t] = 0u;
        }
        if (nsel >= kPfMaxSel) {   // capacity reached: report it only if a block still fits
            uint32_t lm = 0u;
#pragma unroll
            for (int t = 0; t < kPfWords; ++t) lm = max(lm, sk[t]);
            if (__reduce_max_sync(0xffffffffu, lm) != 0u && lane == 0) atomicOr(a.status, 4u);
        }
        uint32_t *bm = a.bitmap + ((int64_t)i * a.Hkv + g) * kPfWords;
        uint32_t words[kPfWords];
#pragma unroll
        for (int t = 0; t < kPfWords; ++t) {
            words[t] = __ballot_sync(0xffffffffu, (selbits >> t) & 1u);
            if (lane == 0) bm[t] = words[t];
        }
        // the query joins each selected block's list with its partial slot:
        // 1 + the block's rank among the selected blocks in index order
        int below = 0;
#pragma unroll
        for (int t = 0; t < kPfWords; ++t) {
            if ((selbits >> t) & 1u) {
                const int j = lane + 32 * t;
                const int slot = 1 + below + __popc(words[t] & ((1u << lane) - 1u));
                const int p = atomicAdd(&a.qcount[g * nb + j], 1);
                a.qlist[((int64_t)g * nb + j) * a.Tq + p] = i | (slot << kPfSlotShift);
            }
            below += __popc(words[t]);
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
// Warp-specialised and pipelined across work items:
//   warps 0-15  softmax + epilogue, four threads per row (warp w owns TMEM
//               lanes 32 (w % 4).. and the column quarter w / 4); each warp
//               also converts its 2 KiB slice of every V tile to fp16 while
//               the tile's S is computed
//   warp 16     lane 0 streams the K tiles, lane 1 the V tiles by TMA (no
//               multicast); the two lanes wait on different barriers
//   warp 17     lane 0 issues every tcgen05.mma
//   warps 18-19 describe work items (alternately, each one ahead), gather
//               their Q rows into the Q buffer and publish them (rows,
//               positions, records)
// TMEM: S double-buffered by a running tile counter u that crosses items
// (columns 0..127, 128..255), O (256..383), and Q double-buffered by item
// parity (384..447, 448..511).  The MMA lane copies an item's Q rows from
// shared memory into TMEM once (tcgen05.cp), so S = Q K^T reads only K from
// shared memory, whose bandwidth the products otherwise saturate.  The one
// shared-memory Q buffer is refilled as soon as it is copied, V has three
// stages so that its loads start a tile earlier, and the item descriptions
// run up to four deep.  An item's epilogue reads O out right after the
// softmax of the next item's first tile, before that tile's P.V overwrites
// it.  O is rescaled only when a row's running maximum grows by more than 2^8
// (the exponentials then stay below 256).
//
// Barriers and their phases (every waiter derives the parity from an index):
//   qready[m] item n (m = n & 3) described, Q gathered (32 lanes of its producer)
//                                                         parity (n >> 2) & 1
//   qfree[b]  item n's Q copied to TMEM (b = n & 1)         parity (n >> 1) & 1
//   qtfree[b] item n's last S complete: TMEM Q[b] free      parity (n >> 1) & 1
//   efree[b]  item n's O read out (16 warps)                parity (n >> 1) & 1
//   slotfree[m] item n's rows read (16 warps)               parity (n >> 2) & 1
//   kfull[s]  K(u) landed (s = u & 1)                       parity (u >> 1) & 1
//   vfull[s]  V(u) landed (s = u % 3; also awaited by the softmax warps,
//             which convert it)                           parity (u / 3) & 1
//   kfree[s]  S(u) complete (tcgen05.commit)                parity (u >> 1) & 1
//   vfree[s]  P.V(u) complete (s = u % 3)                   parity (u / 3) & 1
//   sfull[s]  S(u) complete; pfull[s] P(u) in TMEM and V(u) in fp16 (16
//             warps); odone[s] P.V(u) complete
constexpr int kPfSoftWarps = 16;
constexpr int kPfLoadWarp = 16, kPfMmaWarp = 17, kPfProdWarp = 18;
constexpr int kPfVStages = 3;
constexpr int kPfAttThreads = 32 * 20;
// warps 0-15 softmax, 16 loads, 17 MMA, 18-19 producers
static_assert(kPfSoftWarps == 16 && kPfProdWarp + 2 == kPfAttThreads / 32, "warp roles");
constexpr float kPfRescale = 8.0f;   // log2 of the largest exponential kept without rescaling
constexpr int kPfPrefixCap = 4097;   // tile prefix entries staged in shared memory

struct PfSmem {
    static constexpr int kQ = 0;                          // 2 boxes x 16 KiB
    static constexpr int kK = 32768;                      // 2 stages x 32 KiB
    static constexpr int kV = kK + 65536;                 // 3 stages x 32 KiB
    static constexpr int kRowPos = kV + kPfVStages * 32768;   // int [4][128] query position
    static constexpr int kRowQ = kRowPos + 4 * kTile * 4; // int [4][128] row of Q (-1: none)
    static constexpr int kRowRec = kRowQ + 4 * kTile * 4; // int [4][128] partial record (-1: none)
    static constexpr int kDesc = kRowRec + 4 * kTile * 4; // int [4][8]: g, kbeg, kend, T, local, end
    static constexpr int kPair = kDesc + 4 * 8 * 4;       // float [3][4][128]: quarter-row maxima (by
                                                          // tile parity), quarter-row sums
    static constexpr int kBars = kPair + 3 * 4 * kTile * 4;   // u64 [31]
    static_assert(kBars % 8 == 0, "barrier alignment");
    static constexpr int kMisc = kBars + 31 * 8;          // tmem base
    static constexpr int kPrefix = kMisc + 32;            // int [kPfPrefixCap]
    static constexpr int kBytes = kPrefix + kPfPrefixCap * 4 + 1024;
};

// 2^x by the MUFU instruction, subnormal results flushed to zero (weights below
// 2^-126 of the row maximum contribute nothing at fp32 accumulation).
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void quad_sync(int q) {   // the four warps holding rows 32q..32q+31
    asm volatile("bar.sync %0, 128;" ::"r"(1 + q) : "memory");
}
// the same barrier, returning whether any of the 128 threads passed true
__device__ __forceinline__ bool quad_any(int q, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\tbar.red.or.pred po, %2, 128, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(1 + q)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ float fmax3(float x, float y, float z) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(x), "f"(y), "f"(z));
    return d;
}
// largest of 32 values, as a tree of depth four
__device__ __forceinline__ float max32(const uint32_t (&v)[32]) {
    float m[11];
#pragma unroll
    for (int i = 0; i < 10; ++i)
        m[i] = fmax3(__uint_as_float(v[3 * i]), __uint_as_float(v[3 * i + 1]), __uint_as_float(v[3 * i + 2]));
    m[10] = fmaxf(__uint_as_float(v[30]), __uint_as_float(v[31]));
    return fmaxf(fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]), fmax3(m[6], m[7], m[8])),
                 fmaxf(m[9], m[10]));
}

// This warp's 2 KiB slice of a 32 KiB V stage, bf16 to fp16 in place (the
// 128-byte swizzle moves whole 16-byte chunks, so the layout is unchanged).
// Magnitudes beyond the fp16 range saturate to +-65504.
__device__ __forceinline__ void v_to_f16(unsigned char *stage, int warp, int lane) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint4 *p = reinterpret_cast<uint4 *>(stage + warp * 2048 + (lane + 32 * i) * 16);
        uint4 x = *p;
        uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float lo = __uint_as_float(w[j] << 16), hi = __uint_as_float(w[j] & 0xffff0000u);
            asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(w[j]) : "f"(hi), "f"(lo));
        }
        *p = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Pairs of fp32 operations in one instruction each: ffma2 gives
// (x0 y0 + z0, x1 y1 + z1); fadd2 adds (x0, x1) into (d0, d1).
__device__ __forceinline__ void ffma2(float &d0, float &d1, float x0, float x1, float y0, float y1, float z0,
                                      float z1) {
    asm("{\n\t.reg .b64 px, py, pz;\n\tmov.b64 px, {%2, %3};\n\tmov.b64 py, {%4, %5};\n\t"
        "mov.b64 pz, {%6, %7};\n\tfma.rn.f32x2 pz, px, py, pz;\n\tmov.b64 {%0, %1}, pz;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(x0), "f"(x1), "f"(y0), "f"(y1), "f"(z0), "f"(z1));
}
__device__ __forceinline__ void fadd2(float &d0, float &d1, float x0, float x1) {
    asm("{\n\t.reg .b64 px, pd;\n\tmov.b64 px, {%2, %3};\n\tmov.b64 pd, {%0, %1};\n\t"
        "add.rn.f32x2 pd, pd, px;\n\tmov.b64 {%0, %1}, pd;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(x0), "f"(x1));
}

__global__ void __launch_bounds__(kPfAttThreads, 1)
    prefill_attend_kernel(const __grid_constant__ CUtensorMap tmKp, const __grid_constant__ CUtensorMap tmVp,
                          const __grid_constant__ CUtensorMap tmKl, const __grid_constant__ CUtensorMap tmVl,
                          PfArgs a) {
    extern __shared__ unsigned char praw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(praw) + 1023) & ~uintptr_t(1023));
    int *rowpos_s = reinterpret_cast<int *>(sm + PfSmem::kRowPos);
    int *rowq_s = reinterpret_cast<int *>(sm + PfSmem::kRowQ);
    int *rowrec_s = reinterpret_cast<int *>(sm + PfSmem::kRowRec);
    int *desc_s = reinterpret_cast<int *>(sm + PfSmem::kDesc);
    float *pairv = reinterpret_cast<float *>(sm + PfSmem::kPair);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + PfSmem::kBars);
    uint64_t *qready = bars, *qfree = bars + 4, *efree = bars + 6, *kfull = bars + 8, *vfull = bars + 10,
             *kfree = bars + 13, *vfree = bars + 15, *sfull = bars + 18, *pfull = bars + 20, *odone = bars + 22,
             *drain = bars + 24, *qtfree = bars + 25, *slotfree = bars + 27;
    uint32_t *tmem_sh = reinterpret_cast<uint32_t *>(sm + PfSmem::kMisc);
    int *prefix_s = reinterpret_cast<int *>(sm + PfSmem::kPrefix);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.G, D = a.D;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
            smem_u32(tmem_sh)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        prefetch_tmap(&tmKp); prefetch_tmap(&tmVp); prefetch_tmap(&tmKl); prefetch_tmap(&tmVl);
        for (int i = 0; i < 4; ++i) {
            mbar_init(&qready[i], 32);   // the producer warp
            mbar_init(&slotfree[i], kPfSoftWarps);
        }
        for (int i = 0; i < kPfVStages; ++i) {
            mbar_init(&vfull[i], 1);
            mbar_init(&vfree[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qfree[i], 1);
            mbar_init(&efree[i], kPfSoftWarps);
            mbar_init(&kfull[i], 1);
            mbar_init(&kfree[i], 1);
            mbar_init(&sfull[i], 1);
            mbar_init(&pfull[i], kPfSoftWarps);
            mbar_init(&odone[i], 1);
            mbar_init(&qtfree[i], 1);
        }
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    pdl_wait();
    const int n_pref = a.Hkv * a.nb + 1;
    const bool prefix_in_smem = n_pref <= kPfPrefixCap;
    if (prefix_in_smem)
        for (int e = tid; e < n_pref; e += kPfAttThreads) prefix_s[e] = a.tile_prefix[e];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_sh;   // S0 = cols 0..127, S1 = 128..255, O0 = 256.., O1 = 384..
    const int *prefix = prefix_in_smem ? prefix_s : a.tile_prefix;
    const int n_group = prefix[a.Hkv * a.nb];
    const int n_items = a.n_local + n_group;
    const int qpt = kTile / G;
    const int tiles_per_head = (a.Tq + qpt - 1) / qpt;
    bool timed_out = false;
    auto wait = [&](uint64_t *bar, uint32_t parity) {
        if (!timed_out && !mbar_wait_bounded(bar, parity)) timed_out = true;
    };

    if (warp == kPfProdWarp || warp == kPfProdWarp + 1) {
        // ================= producers.  The CTA's n-th item is blockIdx.x +
        // n gridDim.x; warp kPfProdWarp + p takes the items with n = p (mod 2).
        // A warp describes its next item (rows, positions, records: two
        // rounds of dependent loads) as soon as it has published the current
        // one, so only the Q copies sit between the free Q buffer and the next
        // item.
        const int pt = lane;
        // item n's description into slot n & 3; false for the end marker
        auto describe = [&](int n) -> bool {
            const int m = n & 3;
            const int item = (int)blockIdx.x + n * (int)gridDim.x;
            int *desc = desc_s + m * 8;
            if (item >= n_items) {
                if (pt == 0) desc[5] = 1;
                __syncwarp();
                return false;
            }
            int g, kbeg, kend, mtile, jblk = -1;
            const bool local = item < a.n_local;
            if (local) {
                g = item / tiles_per_head;
                mtile = (item % tiles_per_head) * qpt;   // first query
                kbeg = a.pos_limit;
                kend = a.q_pos0 + min(a.Tq, mtile + qpt);
            } else {
                const int u = item - a.n_local;
                int lo = 0, hi = a.Hkv * a.nb - 1;   // largest e with prefix[e] <= u
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (prefix[mid] <= u) lo = mid; else hi = mid - 1;
                }
                g = lo / a.nb;
                jblk = lo % a.nb;
                mtile = u - prefix[lo];
                kbeg = min(max(a.offsets[(int64_t)g * (a.nb + 1) + jblk], 0), a.L_max);
                kend = kbeg + a.vis[g * a.nb + jblk];
            }
            if (pt == 0) {
                // every item has at least one key tile (a wholly masked one
                // gives o = 0, l = 0), so each role sees the same tiles and
                // the barrier phases stay in step
                kend = max(kend, kbeg);
                desc[0] = g; desc[1] = kbeg; desc[2] = kend;
                desc[3] = max(1, (kend - kbeg + kTile - 1) / kTile);
                desc[4] = local; desc[5] = 0;
            }
            const int cnt = local ? 0 : a.qcount[g * a.nb + jblk];
            for (int r = pt; r < kTile; r += 32) {
                int qi = -1, rec = -1, pos;
                if (local) {
                    const int i = mtile + r / G;
                    pos = a.q_pos0 + i;
                    if (i < a.Tq) { qi = i; rec = ((i * a.Hkv + g) * kPfSlots) * G + (r % G); }
                } else {
                    pos = 0x7fffffff;   // every key of a visible prefix is earlier
                    const int idx = (mtile * kTile + r) / G;
                    if (idx < cnt) {
                        const int e = a.qlist[((int64_t)g * a.nb + jblk) * a.Tq + idx];
                        qi = e & ((1 << kPfSlotShift) - 1);
                        const int slot = e >> kPfSlotShift;
                        rec = ((qi * a.Hkv + g) * kPfSlots + slot) * G + (r % G);
                    }
                }
                rowpos_s[m * kTile + r] = pos;
                rowq_s[m * kTile + r] = qi >= 0 ? qi * a.Hq + g * G + (r % G) : -1;   // row of Q
                rowrec_s[m * kTile + r] = rec;
            }
            __syncwarp();
            return true;
        };
        // item n's Q rows (bf16) into buffer n & 1, swizzled K-major, with
        // asynchronous 16-byte copies (a row with no query is zero-filled)
        auto gather = [&](int n) {
            const int m = n & 3;
            unsigned char *Qs = sm + PfSmem::kQ;
#pragma unroll 4
            for (int c = pt; c < kTile * 16; c += 32) {
                const int r = c >> 4, ch = c & 15, half = ch >> 3, cc = ch & 7;
                const int row = rowq_s[m * kTile + r];
                const uint16_t *src = row >= 0 ? a.Q + (int64_t)row * D + ch * 8 : a.Q;
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                                 smem_u32(Qs + half * 16384 + r * 128 + ((cc ^ (r & 7)) << 4))),
                             "l"(src), "r"(row >= 0 ? 16 : 0)
                             : "memory");
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        };
        int n = warp - kPfProdWarp;
        bool valid = describe(n);
        for (;;) {
            const int m = n & 3;
            if (!valid) {   // end marker: nothing to gather
                mbar_arrive(&qready[m]);
                break;
            }
            // item n-1 (the other warp's) has been copied out of the buffer;
            // one barrier per item parity, so that this wait is never two
            // phases behind
            if (n >= 1) wait(&qfree[(n - 1) & 1], ((n - 1) >> 1) & 1);
            if (timed_out) break;
            gather(n);
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            fence_proxy_async_smem();
            __syncwarp();
            mbar_arrive(&qready[m]);
            // this warp's next item goes to slot (n + 2) & 3 once item n-2's
            // epilogue has read it; its dependent loads then overlap the
            // consumption of items n-1 and n
            if (n >= 2) wait(&slotfree[(n + 2) & 3], ((n - 2) >> 2) & 1);
            if (timed_out) break;
            valid = describe(n + 2);
            n += 2;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");   // nothing in flight at exit
    } else if (warp == kPfLoadWarp) {
        // ================= K loader (lane 0) and V loader (lane 1)
        if (lane < 2) {
            const bool isk = lane == 0;
            const int nst = isk ? 2 : kPfVStages;   // stages: tile u in stage u % nst
            uint64_t *full = isk ? kfull : vfull, *freeb = isk ? kfree : vfree;
            unsigned char *base = sm + (isk ? PfSmem::kK : PfSmem::kV);
            int u = 0;
            for (int n = 0;; ++n) {
                const int m = n & 3;
                wait(&qready[m], (n >> 2) & 1);
                const int *desc = desc_s + m * 8;
                if (timed_out || desc[5]) break;
                const int g = desc[0], T = desc[3];
                // local items address the position-ordered window from its base
                const int kbeg = desc[1] - (desc[4] ? a.pos_base : 0);
                const CUtensorMap *map = desc[4] ? (isk ? &tmKl : &tmVl) : (isk ? &tmKp : &tmVp);
                for (int t = 0; t < T; ++t, ++u) {
                    const int st = u % nst;
                    if (u >= nst) wait(&freeb[st], ((u - nst) / nst) & 1);
                    unsigned char *dst = base + st * 32768;
                    mbar_arrive_expect_tx(&full[st], 32768);
                    tma_load_4d(dst, map, &full[st], 0, kbeg + t * kTile, g, 0);
                    tma_load_4d(dst + 16384, map, &full[st], 64, kbeg + t * kTile, g, 0);
                }
            }
            // the last loads of each stage have landed before the CTA can exit
            const bool to = timed_out;
            timed_out = false;
            for (int v = max(0, u - nst); v < u; ++v) wait(&full[v % nst], (v / nst) & 1);
            timed_out = timed_out || to;
        }
        __syncwarp();
    } else if (warp == kPfMmaWarp) {
        // ================= tcgen05.mma issue (one lane)
        if (lane == 0) {
            constexpr uint32_t kIdescQK = umma_idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t kIdescPV = umma_idesc_f16(128, 128, 0, 1);   // P and V in fp16
            int pend_u = -1, pend_n = 0;
            bool pend_first = false;
            auto pv = [&](int v, int pn, bool first) {   // O (+)= P(v) V(v)
                const int st = v & 1;
                // O has been read out by the previous item's epilogue
                if (first && pn >= 1) wait(&efree[(pn - 1) & 1], ((pn - 1) >> 1) & 1);
                wait(&pfull[st], (v >> 1) & 1);   // also: every warp's slice of V(v) in fp16
                const int vs = v % kPfVStages;
                tc_fence_after();
                const uint32_t v0 = smem_u32(sm + PfSmem::kV + vs * 32768);
                const uint32_t tP = tmem + st * 128, tO = tmem + 256;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint64_t vd = umma_sdesc_sw128(v0 + k * 2048, 16384, 1024);
                    umma_ts(tO, tP + k * 8, vd, kIdescPV, (!first || k > 0) ? 1u : 0u);
                }
                umma_commit(&odone[st]);
                umma_commit(&vfree[vs]);
            };
            int u = 0;
            for (int n = 0;; ++n) {
                const int b = n & 1, m = n & 3;
                wait(&qready[m], (n >> 2) & 1);
                const int *desc = desc_s + m * 8;
                if (timed_out || desc[5]) break;
                const int T = desc[3];
                // the item's Q rows from shared memory into TMEM buffer b, once
                // the S products of its previous user (item n - 2) are done;
                // tcgen05.cp and the products that read it run in issue order
                if (n >= 2) wait(&qtfree[b], ((n - 2) >> 1) & 1);
                tc_fence_after();
                const uint32_t q0 = smem_u32(sm + PfSmem::kQ);
                const uint32_t tQ = tmem + 384 + b * 64;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    tmem_cp_128x256b(tQ + k * 8, umma_sdesc_sw128(q0 + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024));
                umma_commit(&qfree[b]);   // the shared-memory Q buffer is copied
                for (int t = 0; t < T; ++t, ++u) {
                    const int st = u & 1;
                    wait(&kfull[st], (u >> 1) & 1);
                    if (u >= 2) wait(&odone[st], ((u - 2) >> 1) & 1);   // P(u-2) consumed: S[st] free
                    tc_fence_after();
                    const uint32_t k0 = smem_u32(sm + PfSmem::kK + st * 32768);
                    const uint32_t tS = tmem + st * 128;
                    const uint64_t kd = umma_sdesc_sw128(k0, 16, 1024);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        umma_ts(tS, tQ + k * 8, kd + (uint64_t)(((k >> 2) * 16384 + (k & 3) * 32) >> 4), kIdescQK,
                                k > 0);
                    umma_commit(&sfull[st]);
                    umma_commit(&kfree[st]);
                    if (t == T - 1) umma_commit(&qtfree[b]);   // TMEM Q buffer b is read
                    if (pend_u >= 0) pv(pend_u, pend_n, pend_first);
                    pend_u = u;
                    pend_n = n;
                    pend_first = t == 0;
                }
            }
            if (pend_u >= 0) pv(pend_u, pend_n, pend_first);
            // every issued MMA has completed before the CTA frees its TMEM
            const bool to = timed_out;
            umma_commit(drain);
            timed_out = false;
            wait(drain, 0);
            timed_out = timed_out || to;
        }
        __syncwarp();
    } else if (warp < kPfSoftWarps) {
        // ================= softmax warps
        const int q = warp & 3, cq = warp >> 2;      // row quarter (TMEM lanes), key quarter
        const int r = q * 32 + lane;                 // this thread's row
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        // An item's epilogue (its last P.V, then its partial) runs after the
        // softmax of the next item's first tile, so that the tensor cores
        // work on that tile meanwhile.
        bool pend = false;
        int pend_n = 0, pend_u = 0;
        float pend_m = 0.0f, pend_l = 0.0f;
        auto epilogue = [&]() {
            const int pend_b = pend_n & 1, pend_m4 = pend_n & 3;
            wait(&odone[pend_u & 1], (pend_u >> 1) & 1);
            tc_fence_after();
            float *pl4 = pairv + 8 * kTile;
            pl4[cq * kTile + r] = pend_l;
            quad_sync(q);
            const float l_row = (pl4[r] + pl4[kTile + r]) + (pl4[2 * kTile + r] + pl4[3 * kTile + r]);
            quad_sync(q);
            const int rec = rowrec_s[pend_m4 * kTile + r];
            float *po = rec >= 0 ? a.part_o + (int64_t)rec * D + cq * 32 : nullptr;
            uint32_t ov[32];
            tmem_ld32(tmem + 256 + lane_base + cq * 32, ov);
            tmem_ld_wait();
            // O and the item's shared-memory rows may be reused
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&efree[pend_b]);
                mbar_arrive(&slotfree[pend_m4]);
            }
            if (po) {
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4 *>(po + e) =
                        make_float4(__uint_as_float(ov[e]), __uint_as_float(ov[e + 1]),
                                    __uint_as_float(ov[e + 2]), __uint_as_float(ov[e + 3]));
            }
            if (rec >= 0 && cq == 0) a.part_ml[rec] = make_float2(pend_m, l_row);
            pend = false;
        };
        int u = 0;
        for (int n = 0;; ++n) {
            const int m = n & 3;
            wait(&qready[m], (n >> 2) & 1);
            const int *desc = desc_s + m * 8;
            if (timed_out || desc[5]) break;
            const int kbeg = desc[1], kend = desc[2], T = desc[3];
            const int my_pos = rowpos_s[m * kTile + r];
            const uint32_t tO = tmem + 256;
            float m_used = kPfNegInf, l_part = 0.0f;
            for (int t = 0; t < T; ++t, ++u) {
                const int st = u & 1;
                // V(u) to fp16 (this warp's slice), while S(u) is computed;
                // P(u)'s arrival below also tells the MMA lane that the slice
                // is converted
                wait(&vfull[u % kPfVStages], (u / kPfVStages) & 1);
                v_to_f16(sm + PfSmem::kV + (u % kPfVStages) * 32768, warp, lane);
                fence_proxy_async_smem();
                wait(&sfull[st], (u >> 1) & 1);
                tc_fence_after();
                const uint32_t tS = tmem + st * 128;
                uint32_t sv[32];
                tmem_ld32(tS + lane_base + cq * 32, sv);
                tmem_ld_wait();
                // maxima on the raw logits (the scale is positive); masked
                // keys become -inf
                const int key0 = kbeg + t * kTile + cq * 32;
                if (!(key0 + 31 < kend && key0 + 31 <= my_pos)) {   // some key of the quarter hidden
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int kr = key0 + e;
                        if (!(kr < kend && kr <= my_pos)) sv[e] = __float_as_uint(kPfNegInf);
                    }
                }
                const float qmax = max32(sv);
                // Lazy rescale: a row keeps its reference maximum unless this
                // tile exceeds it by more than 2^8 (or it has none yet and the
                // tile has a visible key).  The tile's row maximum is over all
                // four quarters, and it exceeds a bound exactly when one
                // quarter's does, so the quarters first agree, in one barrier,
                // on whether any row must move; only then are maxima exchanged.
                // The barrier also orders every quarter's read of S(u) before
                // any quarter writes P into it.
                const float qm = qmax * a.scale_log2;
                const bool need = qm != kPfNegInf && (m_used == kPfNegInf || qm > m_used + kPfRescale);
                float factor = 1.0f;
                if (quad_any(q, need)) {
                    float *pm = pairv + (st * 4) * kTile;
                    pm[cq * kTile + r] = qmax;
                    quad_sync(q);
                    const float m_tile =
                        fmaxf(fmaxf(pm[r], pm[kTile + r]), fmaxf(pm[2 * kTile + r], pm[3 * kTile + r])) * a.scale_log2;
                    bool rescale = false;
                    float m_ref = m_used;
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
                        // O must hold P.V(u-1) before it is scaled
                        wait(&odone[(u - 1) & 1], ((u - 1) >> 1) & 1);
                        tc_fence_after();
                        uint32_t ov[32];
                        tmem_ld32(tO + lane_base + cq * 32, ov);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * factor);
                        tmem_st32(tO + lane_base + cq * 32, ov);
                    }
                    m_used = m_ref;
                }
                l_part *= factor;
                // P in fp16 over this quarter's 32 keys, written to the tile's S
                // columns 16 cq..  (two keys a column).  The row sum l adds the
                // rounded weights, so O / l is a weighted mean of V with weights
                // that sum to one: each fp16 half is read back exactly as its
                // bits shifted into an fp32 2^-112 times its value, and the sum
                // is scaled by 2^112 at the end.  A row with no visible key so
                // far has only -inf logits, which give 0 with any finite offset.
                float ls0 = 0.0f, ls1 = 0.0f;
                uint32_t ph[16];
                const float neg_m = m_used == kPfNegInf ? 0.0f : -m_used;
                const float sc = a.scale_log2;
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float x0, x1;
                    ffma2(x0, x1, __uint_as_float(sv[e]), __uint_as_float(sv[e + 1]), sc, sc, neg_m, neg_m);
                    const float p0 = ex2_ftz(x0), p1 = ex2_ftz(x1);
                    uint32_t w;
                    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(p1), "f"(p0));
                    ph[e / 2] = w;
                    fadd2(ls0, ls1, __uint_as_float((w & 0xffffu) << 13), __uint_as_float((w >> 16) << 13));
                }
                tmem_st16(tS + lane_base + cq * 16, ph);
                l_part += (ls0 + ls1) * 0x1p112f;
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&pfull[st]);
                if (t == 0 && pend) epilogue();   // the previous item's
            }
            pend = true;   // T >= 1: the item's last tile is u - 1
            pend_n = n;
            pend_u = u - 1;
            pend_m = m_used;
            pend_l = l_part;
        }
        if (pend) epilogue();
    }
    if (timed_out) atomicOr(a.status, 8u);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
}

// ---------------------------------------------------------------- P4
__global__ void __launch_bounds__(kPfMergeThreads, 8) prefill_merge_kernel(PfArgs a) {
    pdl_wait();
    const int i = blockIdx.x, g = blockIdx.y, G = a.G, D = a.D, D4 = D / 4;
    // one thread per (head, 4 dimensions) and pass; the slots are merged in
    // slot order with a running maximum
    for (int e = threadIdx.x; e < G * D4; e += blockDim.x) {
        const int hh = e / D4, d4 = e % D4;
        const int64_t rec0 = ((int64_t)i * a.Hkv + g) * kPfSlots * G + hh;
        // the first slots' records are read before the slot count is known
        // (every query has kPfSlots records reserved), so the two reads overlap
        constexpr int kEarly = 4;
        float2 ml0[kEarly];
        float4 ov0[kEarly];
#pragma unroll
        for (int s = 0; s < kEarly; ++s) {
            ml0[s] = __ldcg(&a.part_ml[rec0 + (int64_t)s * G]);
            ov0[s] = __ldcg(reinterpret_cast<const float4 *>(a.part_o + (rec0 + (int64_t)s * G) * D) + d4);
        }
        const uint32_t *bm = a.bitmap + ((int64_t)i * a.Hkv + g) * kPfWords;
        int nsel = 0;
#pragma unroll
        for (int w = 0; w < kPfWords; ++w) nsel += __popc(__ldcg(bm + w));
        const int nslot = min(1 + nsel, kPfSlots);
        float M = kPfNegInf, L = 0.0f;
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
        auto fold = [&](float2 ml, float4 o) {
            const float mn = fmaxf(M, ml.x);
            if (mn != kPfNegInf) {
                const float c = exp2f(M - mn), w = exp2f(ml.x - mn);
                L = L * c + ml.y * w;
                O.x = O.x * c + o.x * w; O.y = O.y * c + o.y * w;
                O.z = O.z * c + o.z * w; O.w = O.w * c + o.w * w;
                M = mn;
            }
        };
#pragma unroll
        for (int s = 0; s < kEarly; ++s)
            if (s < nslot) fold(ml0[s], ov0[s]);
#pragma unroll 4
        for (int s = kEarly; s < nslot; ++s) {
            const int64_t rec = rec0 + (int64_t)s * G;
            fold(__ldcg(&a.part_ml[rec]), __ldcg(reinterpret_cast<const float4 *>(a.part_o + rec * D) + d4));
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
    size_t bitmap, vis, qcount, qlist, prefix, part_o, part_ml, total;
};

static PfLayout pf_layout(const bsa_kv_desc *d, const bsa_sel_params *p, int Tq) {
    PfLayout L;
    const size_t G = d->Hq / d->Hkv, nb = p->n_blocks, H = d->Hkv;
    size_t o = 0;
    L.bitmap = o;  o += align_up((size_t)Tq * H * kPfWords * 4, 256);
    L.vis = o;     o += align_up(H * nb * 4, 256);
    L.qcount = o;  o += align_up(H * nb * 4, 256);
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
                          const void *K_pos, const void *V_pos, int pos_base, const void *Q, int q_pos0, int Tq,
                          float scale, float *out, float *lse, uint32_t *status, void *ws,
                          size_t ws_bytes, cudaStream_t st) {
    const int G = d->Hq / d->Hkv;
    if (p->n_blocks > kPfMaxBlocks || kTile % G != 0 || G > 16) return BSA_ERR_UNSUPPORTED;
    // query index and slot share a qlist entry; partial records index with int32
    if (Tq >= (1 << kPfSlotShift) || (int64_t)Tq * d->Hkv * kPfSlots * G >= (int64_t)1 << 31)
        return BSA_ERR_UNSUPPORTED;
    const PfLayout L = pf_layout(d, p, Tq);
    if (ws_bytes < L.total) return BSA_ERR_WORKSPACE;
    char *w = static_cast<char *>(ws);
    PfArgs a;
    a.Hq = d->Hq; a.Hkv = d->Hkv; a.G = G; a.D = d->D; a.nb = p->n_blocks;
    a.L_max = d->L_max; a.Lpos = pd->L_max;
    a.Tq = Tq; a.q_pos0 = q_pos0; a.pos_limit = p->pos_limit; a.budget = p->budget_tokens;
    a.pos_base = pos_base;
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
    // zero the per-block counts
    BSA_CUDA_TRY(cudaMemsetAsync(w + L.qcount, 0, (size_t)d->Hkv * p->n_blocks * 4, st));
    // P1: selection
    auto smem1_for = [&](int nw) {
        return ((size_t)a.nb * kPfCentStride + (size_t)nw * G * a.D + a.nb) * 4 + (size_t)nw * G * a.D * 2;
    };
    int nw1 = kPfSelWarps;
    while (nw1 > 1 && smem1_for(nw1) > kMaxSmemPerCta) nw1 /= 2;
    const size_t smem1 = smem1_for(nw1);
    BSA_CUDA_TRY(cudaFuncSetAttribute(prefill_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem1));
    // one wave: about num_sms / Hkv CTAs per KV head, the rows split evenly
    const int ctas_per_head = std::max(1, num_sms() / d->Hkv);
    a.sel_rows_per_warp = std::max(1, (int)div_up(Tq, (int64_t)ctas_per_head * nw1));
    BSA_CUDA_TRY(launch_pdl(prefill_select_kernel,
                            dim3((unsigned)div_up(Tq, nw1 * a.sel_rows_per_warp), (unsigned)d->Hkv),
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
    BSA_CUDA_TRY(launch_pdl(prefill_merge_kernel, dim3((unsigned)Tq, (unsigned)d->Hkv),
                            dim3(kPfMergeThreads), 0, st, a));
    return BSA_OK;
}

}  // namespace bsa
