// The semantic index: spherical k-means over each segment's keys and the
// block-ordered store ("Semantic blocks for sparse attention", first section:
// similar keys from anywhere in the request are grouped by spherical k-means
// and each group is stored together and summarised by its centre).
//
// Arithmetic (fixed, so that the labels can be compared bit for bit):
//   u_r   = k_r / ||k_r||   (||.|| = sqrt of an fma chain over i; zero stays zero)
//   c_j   = u_{init[j]} to start
//   round: label_r = argmax_j fma-chain_i(u_r[i] * c_j[i]), lowest j on ties;
//          between rounds c_j = m / ||m||, m = (sum of u_r over cluster j in
//          position order) / n_j; an empty cluster keeps its centre.
//   `iters` rounds of assignment, iters - 1 updates between them.
//
// The unit keys u_r are computed once per build (km_unit_kernel) into the
// workspace; the rounds read them instead of dividing again.
//
// Kernels, per round (every segment at once):
//   km_assign_tiled_kernel  (k <= 256) a CTA per 1,024 keys of a segment, 64
//                       keys at a time: unit keys and centres transposed in
//                       shared memory, 8 keys x 8 centres of fma chains per
//                       thread, a warp argmax; the chunk's label histogram
//   km_assign_kernel    (k > 256) the same with one key's unit vector per
//                       thread in registers, four centres' chains at a time
//   km_scan_kernel      a CTA per segment: cluster sizes, CSR offsets and each
//                       chunk's first slot per cluster
//   km_scatter_kernel   a CTA per chunk: stable slots (rank among equal labels
//                       by __match_any_sync within a warp, warps in order), so
//                       order[] lists each cluster's keys by position
//   km_update_kernel    a CTA per (segment, cluster): thread i sums dimension i
//                       of the cluster's unit keys in position order
#include "common.cuh"

namespace bsa {

constexpr int kKmChunk = 1024;      // keys per assignment / scatter CTA
constexpr int kKmAssignThreads = 256;
constexpr int kKmMaxK = 1024;       // clusters (one scan thread each)

struct KmArgs {
    const void *K;
    int64_t stride_b, stride_h, stride_t;
    int Hkv, D, k, nchunk;
    int64_t L;
    const int32_t *init;   // [nseg][k]
    float *C;              // [nseg][k][D]
    int32_t *labels;       // [nseg][L]
    int32_t *offsets;      // [nseg][k + 1]
    int32_t *order;        // [nseg][L]
    float *norms;          // [nseg][L]
    float *U;              // [nseg][L][D]: unit keys
    int32_t *chist;        // [nseg][nchunk][k]: counts, then first slots
};

template <typename T>
__device__ __forceinline__ const T *km_row(const KmArgs &a, int s, int64_t r) {
    const int b = s / a.Hkv, g = s % a.Hkv;
    return static_cast<const T *>(a.K) + b * a.stride_b + g * a.stride_h + r * a.stride_t;
}

// ||k_r|| for every key: fma chain over i, then sqrt.
template <typename T>
__global__ void __launch_bounds__(256) km_norms_kernel(KmArgs a) {
    const int s = blockIdx.y;
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= a.L) return;
    const T *row = km_row<T>(a, s, r);
    float acc = 0.0f;
#pragma unroll 8
    for (int i = 0; i < a.D; ++i) {
        const float v = load_elem(row, i);
        acc = __fmaf_rn(v, v, acc);
    }
    a.norms[(int64_t)s * a.L + r] = __fsqrt_rn(acc);
}

// u_r = k_r / ||k_r|| (zero stays zero), one element per thread.
template <typename T>
__global__ void __launch_bounds__(256) km_unit_kernel(KmArgs a) {
    const int s = blockIdx.y;
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= a.L * a.D) return;
    const int64_t r = e / a.D;
    const int i = (int)(e % a.D);
    const float nr = a.norms[(int64_t)s * a.L + r];
    const float v = load_elem(km_row<T>(a, s, r), i);
    a.U[(int64_t)s * a.L * a.D + e] = nr > 0.0f ? __fdiv_rn(v, nr) : 0.0f;
}

// c_j = u_{init[j]}: CTA (j, segment), thread i.
template <typename T>
__global__ void km_init_kernel(KmArgs a) {
    const int j = blockIdx.x, s = blockIdx.y, i = threadIdx.x;
    const int64_t r = min(max((int64_t)a.init[(int64_t)s * a.k + j], (int64_t)0), a.L - 1);   // clamped
    const float nr = a.norms[(int64_t)s * a.L + r];
    const float v = load_elem(km_row<T>(a, s, r), i);
    a.C[((int64_t)s * a.k + j) * a.D + i] = nr > 0.0f ? __fdiv_rn(v, nr) : 0.0f;
}

// Labels for one chunk of kKmChunk keys (four per thread, one at a time) and
// the chunk's histogram.  Shared memory: centres [k4][D] (k4 = k rounded up
// to 4, zero rows past k), histogram [k].
template <typename T, int D>
__global__ void __launch_bounds__(kKmAssignThreads) km_assign_kernel(KmArgs a) {
    extern __shared__ __align__(16) float kms[];
    const int s = blockIdx.y, c = blockIdx.x, k = a.k, k4 = (k + 3) & ~3;
    float *Cs = kms;
    int *hist = reinterpret_cast<int *>(Cs + (size_t)k4 * D);
    const float *Cg = a.C + (int64_t)s * k * D;
    for (int e = threadIdx.x; e < k4 * D; e += blockDim.x) Cs[e] = e < k * D ? Cg[e] : 0.0f;
    for (int j = threadIdx.x; j < k; j += blockDim.x) hist[j] = 0;
    __syncthreads();
    for (int t = 0; t < kKmChunk / kKmAssignThreads; ++t) {
        const int64_t r = (int64_t)c * kKmChunk + t * kKmAssignThreads + threadIdx.x;
        if (r < a.L) {
            const float *ur = a.U + ((int64_t)s * a.L + r) * D;
            float u[D];
#pragma unroll
            for (int i = 0; i < D; i += 4) {
                const float4 v = *reinterpret_cast<const float4 *>(ur + i);
                u[i] = v.x; u[i + 1] = v.y; u[i + 2] = v.z; u[i + 3] = v.w;
            }
            float best = -__builtin_huge_valf();
            int lab = 0;
            for (int j = 0; j < k4; j += 4) {
                const float *c0 = Cs + (size_t)j * D;
                float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int i = 0; i < D; i += 4) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 cv = *reinterpret_cast<const float4 *>(c0 + q * D + i);
                        acc[q] = __fmaf_rn(u[i], cv.x, acc[q]);
                        acc[q] = __fmaf_rn(u[i + 1], cv.y, acc[q]);
                        acc[q] = __fmaf_rn(u[i + 2], cv.z, acc[q]);
                        acc[q] = __fmaf_rn(u[i + 3], cv.w, acc[q]);
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (j + q < k && acc[q] > best) { best = acc[q]; lab = j + q; }
            }
            a.labels[(int64_t)s * a.L + r] = lab;
            atomicAdd(&hist[lab], 1);
        }
    }
    __syncthreads();
    int32_t *h = a.chist + ((int64_t)s * a.nchunk + c) * k;
    for (int j = threadIdx.x; j < k; j += blockDim.x) h[j] = hist[j];
}

// The same labels, register-blocked for k <= 256 (the common case): a tile of
// 64 keys at a time, their unit vectors transposed in shared memory
// uT[d][key] next to the centres cT[d][j]; warp w owns keys 8w .. 8w+7 of the
// tile and lane l the centres 4l .. 4l+3 and 128 + 4l .. 128 + 4l+3, so each
// d step is two broadcast loads of u, two conflict-free loads of c and 64
// fmas into acc[key][centre] -- every (key, centre) chain still runs over
// d = 0 .. D-1 in order (two chains per fma.rn.f32x2: each half is its own
// fused multiply-add, rounded once).  Each lane keeps its best centre per key (lowest
// index on equal dots); the warp then takes the largest dot (redux.sync max
// of its orderable key, -0 folded into +0) and the lowest centre holding it.
constexpr int kKmTile = 64;
constexpr int kKmTiledMaxK = 256;

template <typename T, int D>
__global__ void __launch_bounds__(256) km_assign_tiled_kernel(KmArgs a) {
    extern __shared__ __align__(16) float kms[];
    float *cT = kms;                       // [D][256]
    float *uT = cT + D * kKmTiledMaxK;     // [D][kKmTile]
    int *hist = reinterpret_cast<int *>(uT + D * kKmTile);   // [k]
    const int s = blockIdx.y, c = blockIdx.x, k = a.k;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float *Cg = a.C + (int64_t)s * k * D;
    for (int e = tid; e < D * kKmTiledMaxK; e += blockDim.x) {
        const int d = e / kKmTiledMaxK, j = e % kKmTiledMaxK;
        cT[e] = j < k ? Cg[(int64_t)j * D + d] : 0.0f;
    }
    for (int j = tid; j < k; j += blockDim.x) hist[j] = 0;
    const int64_t key0 = (int64_t)c * kKmChunk;
    // the tile's unit rows: thread = (key kk, quarter part of D); the next
    // tile's rows are fetched (16-byte loads) while the current tile computes
    constexpr int Q = D / 4, NV = Q / 4;
    const int kk = tid >> 2, part = tid & 3;
    uint4 raw[NV];
    auto fetch = [&](int t0) {
        const int64_t r = key0 + t0 + kk;
        if (r < a.L) {
            const uint4 *src = reinterpret_cast<const uint4 *>(a.U + ((int64_t)s * a.L + r) * D + part * Q);
#pragma unroll
            for (int v = 0; v < NV; ++v) raw[v] = __ldg(src + v);
        } else {
#pragma unroll
            for (int v = 0; v < NV; ++v) raw[v] = make_uint4(0u, 0u, 0u, 0u);
        }
    };
    fetch(0);
    for (int t0 = 0; t0 < kKmChunk; t0 += kKmTile) {
        __syncthreads();   // centres in place / the previous tile's u consumed
        {   // unit vectors of the tile's keys, transposed
#pragma unroll
            for (int v = 0; v < NV; ++v) {
                const uint32_t w[4] = {raw[v].x, raw[v].y, raw[v].z, raw[v].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) uT[(part * Q + v * 4 + e) * kKmTile + kk] = __uint_as_float(w[e]);
            }
        }
        __syncthreads();
        if (t0 + kKmTile < kKmChunk) fetch(t0 + kKmTile);
        float acc[8][8];
#pragma unroll
        for (int x = 0; x < 8; ++x)
#pragma unroll
            for (int y = 0; y < 8; ++y) acc[x][y] = 0.0f;
        const float *up = uT + warp * 8;
        const float *cp = cT + lane * 4;
#pragma unroll 4
        for (int d = 0; d < D; ++d) {
            const float4 u0 = *reinterpret_cast<const float4 *>(up + d * kKmTile);
            const float4 u1 = *reinterpret_cast<const float4 *>(up + d * kKmTile + 4);
            const float4 c0 = *reinterpret_cast<const float4 *>(cp + d * kKmTiledMaxK);
            const float4 c1 = *reinterpret_cast<const float4 *>(cp + d * kKmTiledMaxK + 128);
            const float uu[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            const float cc[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
            for (int x = 0; x < 8; ++x)
#pragma unroll
                for (int y = 0; y < 8; y += 2)
                    asm("{\n\t.reg .b64 pa, pb, pc;\n\t"
                        "mov.b64 pa, {%2, %2};\n\tmov.b64 pb, {%3, %4};\n\tmov.b64 pc, {%0, %1};\n\t"
                        "fma.rn.f32x2 pc, pa, pb, pc;\n\tmov.b64 {%0, %1}, pc;\n\t}"
                        : "+f"(acc[x][y]), "+f"(acc[x][y + 1])
                        : "f"(uu[x]), "f"(cc[y]), "f"(cc[y + 1]));
        }
#pragma unroll
        for (int x = 0; x < 8; ++x) {
            // this lane's best centre for key x (its centres in increasing order)
            float best = 0.0f;
            int lab = -1;
#pragma unroll
            for (int y = 0; y < 8; ++y) {
                const int j = (y < 4 ? 0 : 128) + lane * 4 + (y & 3);
                if (j < k && (lab < 0 || acc[x][y] > best)) { best = acc[x][y]; lab = j; }
            }
            const uint32_t ok = lab >= 0 ? f32_order_key(__fadd_rn(best, 0.0f)) : 0u;
            const uint32_t m = __reduce_max_sync(0xffffffffu, ok);
            const int win = __reduce_min_sync(0xffffffffu, ok == m && lab >= 0 ? lab : 0x7fffffff);
            const int64_t r = key0 + t0 + warp * 8 + x;
            if (lane == 0 && r < a.L) {
                a.labels[(int64_t)s * a.L + r] = win;
                atomicAdd(&hist[win], 1);
            }
        }
    }
    __syncthreads();
    int32_t *h = a.chist + ((int64_t)s * a.nchunk + c) * k;
    for (int j = tid; j < k; j += blockDim.x) h[j] = hist[j];
}

// Cluster sizes -> offsets; chist[c][j] becomes the first slot of chunk c's
// keys of cluster j.  One CTA per segment, thread j per cluster.
__global__ void __launch_bounds__(kKmMaxK) km_scan_kernel(KmArgs a) {
    __shared__ int wsum[32];
    const int s = blockIdx.x, j = threadIdx.x, k = a.k;
    const int lane = j & 31, warp = j >> 5;
    int32_t *h = a.chist + (int64_t)s * a.nchunk * k;
    int tot = 0;
    if (j < k) {
#pragma unroll 8
        for (int c = 0; c < a.nchunk; ++c) tot += h[(int64_t)c * k + j];
    }
    // exclusive scan of the sizes over j
    int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        int w = lane < nw ? wsum[lane] : 0, wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += v;
        }
        if (lane < nw) wsum[lane] = wi - w;
    }
    __syncthreads();
    const int excl = incl - tot + wsum[warp];
    int32_t *off = a.offsets + (int64_t)s * (k + 1);
    if (j < k) {
        off[j] = excl;
        if (j == k - 1) off[k] = excl + tot;
        int run = excl;
        for (int c = 0; c < a.nchunk; ++c) {
            const int v = h[(int64_t)c * k + j];
            h[(int64_t)c * k + j] = run;
            run += v;
        }
    }
}

// Stable slots for one chunk: warp w holds keys c*kKmChunk + 32 w + lane.
// Shared memory: per (warp, cluster) counts, then the warps' first slots.
__global__ void __launch_bounds__(kKmChunk) km_scatter_kernel(KmArgs a) {
    extern __shared__ int wcnt[];   // [32][k]
    const int s = blockIdx.y, c = blockIdx.x, k = a.k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int e = threadIdx.x; e < 32 * k; e += blockDim.x) wcnt[e] = 0;
    __syncthreads();
    const int64_t r = (int64_t)c * kKmChunk + threadIdx.x;
    const bool live = r < a.L;
    const int lab = live ? a.labels[(int64_t)s * a.L + r] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, lab);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (live && rank == 0) wcnt[warp * k + lab] = __popc(peers);
    __syncthreads();
    for (int j = threadIdx.x; j < k; j += blockDim.x) {   // warps' first slots, in warp order
        int run = a.chist[((int64_t)s * a.nchunk + c) * k + j];
        for (int w = 0; w < 32; ++w) {
            const int v = wcnt[w * k + j];
            wcnt[w * k + j] = run;
            run += v;
        }
    }
    __syncthreads();
    if (live) a.order[(int64_t)s * a.L + wcnt[warp * k + lab] + rank] = (int32_t)r;
}

// c_j = m / ||m||, m = mean of the cluster's unit keys summed in position
// order (block order); an empty cluster keeps its centre.  CTA (j, segment),
// thread i < D.
template <typename T>
__global__ void __launch_bounds__(128) km_update_kernel(KmArgs a) {
    __shared__ float m[128];
    __shared__ float nc_s;
    const int j = blockIdx.x, s = blockIdx.y, i = threadIdx.x, D = a.D;
    const int32_t *off = a.offsets + (int64_t)s * (a.k + 1);
    const int beg = off[j], end = off[j + 1];
    if (end <= beg) return;
    const int32_t *ord = a.order + (int64_t)s * a.L;
    const float *Us = a.U + (int64_t)s * a.L * D;
    float acc = 0.0f;
    if (i < D) {
        int p = beg;
        constexpr int kB = 64;   // rows in flight; the adds stay in order
        for (; p + kB <= end; p += kB) {
            int r[kB];
            float v[kB];
#pragma unroll
            for (int q = 0; q < kB; ++q) r[q] = ord[p + q];
#pragma unroll
            for (int q = 0; q < kB; ++q) v[q] = Us[(int64_t)r[q] * D + i];
#pragma unroll
            for (int q = 0; q < kB; ++q) acc = __fadd_rn(acc, v[q]);
        }
        for (; p < end; ++p) acc = __fadd_rn(acc, Us[(int64_t)ord[p] * D + i]);
        m[i] = __fdiv_rn(acc, (float)(end - beg));
    }
    __syncthreads();
    if (i == 0) {
        float q = 0.0f;
        for (int d = 0; d < D; ++d) q = __fmaf_rn(m[d], m[d], q);
        nc_s = __fsqrt_rn(q);
    }
    __syncthreads();
    if (i < D) {
        const float nc = nc_s;
        a.C[((int64_t)s * a.k + j) * D + i] = nc > 0.0f ? __fdiv_rn(m[i], nc) : 0.0f;
    }
}

size_t kmeans_ws_bytes(const bsa_kv_desc *d, int64_t L, int k) {
    const size_t nseg = (size_t)d->B * d->Hkv;
    const size_t nchunk = (size_t)div_up(L, kKmChunk);
    return align_up(nseg * (size_t)L * 4, 256) + align_up(nseg * nchunk * (size_t)k * 4, 256) +
           align_up(nseg * (size_t)L * d->D * 4, 256);
}

bool kmeans_supported(const bsa_kv_desc *d, int k) {
    return k >= 1 && k <= kKmMaxK && (size_t)((k + 3) & ~3) * d->D * 4 + (size_t)k * 4 <= 200 * 1024;
}

bsa_status launch_kmeans(const bsa_kv_desc *d, const void *K, int64_t L, int k, int iters,
                         const int32_t *init, float *C, int32_t *labels, int32_t *offsets,
                         int32_t *order, void *ws, cudaStream_t st) {
    KmArgs a;
    a.K = K;
    a.stride_b = d->stride_b; a.stride_h = d->stride_h; a.stride_t = d->stride_t;
    a.Hkv = d->Hkv; a.D = d->D; a.k = k; a.L = L;
    a.nchunk = (int)div_up(L, kKmChunk);
    a.init = init; a.C = C; a.labels = labels; a.offsets = offsets; a.order = order;
    const size_t nseg = (size_t)d->B * d->Hkv;
    a.norms = static_cast<float *>(ws);
    a.chist = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + align_up(nseg * (size_t)L * 4, 256));
    a.U = reinterpret_cast<float *>(static_cast<char *>(ws) + align_up(nseg * (size_t)L * 4, 256) +
                                    align_up(nseg * (size_t)a.nchunk * k * 4, 256));
    const dim3 gkeys((unsigned)div_up(L, 256), (unsigned)nseg);
    const dim3 gchunks((unsigned)a.nchunk, (unsigned)nseg), gclusters((unsigned)k, (unsigned)nseg);
    const size_t smem_assign = (size_t)((k + 3) & ~3) * d->D * 4 + (size_t)k * 4;
    const size_t smem_scatter = (size_t)32 * k * 4;
    auto run = [&](auto tag, auto dtag) -> bsa_status {
        using T = decltype(tag);
        constexpr int DD = decltype(dtag)::value;
        const bool tiled = k <= kKmTiledMaxK;
        auto assign = tiled ? km_assign_tiled_kernel<T, DD> : km_assign_kernel<T, DD>;
        const size_t smem_a = tiled ? (size_t)DD * (kKmTiledMaxK + kKmTile) * 4 + (size_t)k * 4 : smem_assign;
        BSA_CUDA_TRY(cudaFuncSetAttribute(assign, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_a));
        BSA_CUDA_TRY(cudaFuncSetAttribute(km_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem_scatter));
        km_norms_kernel<T><<<gkeys, 256, 0, st>>>(a);
        BSA_LAUNCH_CHECK();
        km_unit_kernel<T><<<dim3((unsigned)div_up(L * DD, 256), (unsigned)nseg), 256, 0, st>>>(a);
        BSA_LAUNCH_CHECK();
        km_init_kernel<T><<<gclusters, DD, 0, st>>>(a);
        BSA_LAUNCH_CHECK();
        for (int it = 0; it < iters; ++it) {
            assign<<<gchunks, kKmAssignThreads, smem_a, st>>>(a);
            BSA_LAUNCH_CHECK();
            km_scan_kernel<<<(unsigned)nseg, kKmMaxK, 0, st>>>(a);
            BSA_LAUNCH_CHECK();
            km_scatter_kernel<<<gchunks, kKmChunk, smem_scatter, st>>>(a);
            BSA_LAUNCH_CHECK();
            if (it + 1 < iters) {
                km_update_kernel<T><<<gclusters, 128, 0, st>>>(a);
                BSA_LAUNCH_CHECK();
            }
        }
        return BSA_OK;
    };
    if (d->kv_dtype == BSA_BF16)
        return d->D == 128 ? run(uint16_t{}, std::integral_constant<int, 128>())
                           : run(uint16_t{}, std::integral_constant<int, 64>());
    return d->D == 128 ? run(float{}, std::integral_constant<int, 128>())
                       : run(float{}, std::integral_constant<int, 64>());
}

// Row gather between two caches of the same geometry: row dst_row0 + i of
// each segment of the destination = row rows[seg][i] of the source.  A warp
// per row, 16-byte chunks.
__global__ void __launch_bounds__(256) gather_rows_kernel(const char *K, const char *V, char *Ko, char *Vo,
                                                           int64_t sb, int64_t sh, int64_t stt,
                                                           int64_t db, int64_t dh, int64_t dt, int Hkv,
                                                           int row_bytes, const int32_t *rows, int64_t n,
                                                           int64_t dst_row0, int64_t src_rows) {
    const int s = blockIdx.y;
    const int64_t i = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (i >= n) return;
    const int lane = threadIdx.x & 31, b = s / Hkv, g = s % Hkv;
    const int64_t r = rows[(int64_t)s * n + i];
    if (r < 0 || r >= src_rows) return;   // not a source row: the destination row is left alone
    const int64_t so = b * sb + g * sh + r * stt, dof = b * db + g * dh + (dst_row0 + i) * dt;
    for (int e = lane * 16; e < row_bytes; e += 512) {
        *reinterpret_cast<uint4 *>(Ko + dof + e) = *reinterpret_cast<const uint4 *>(K + so + e);
        *reinterpret_cast<uint4 *>(Vo + dof + e) = *reinterpret_cast<const uint4 *>(V + so + e);
    }
}

bsa_status launch_gather_rows(const bsa_kv_desc *src, const void *K, const void *V, const bsa_kv_desc *dst,
                              void *K_out, void *V_out, const int32_t *rows, int64_t n, int64_t dst_row0,
                              cudaStream_t st) {
    const int64_t es = src->kv_dtype == BSA_F32 ? 4 : src->kv_dtype == BSA_BF16 ? 2 : 1;
    const dim3 grid((unsigned)div_up(n, 8), (unsigned)(src->B * src->Hkv));
    gather_rows_kernel<<<grid, 256, 0, st>>>(
        static_cast<const char *>(K), static_cast<const char *>(V), static_cast<char *>(K_out),
        static_cast<char *>(V_out), src->stride_b * es, src->stride_h * es, src->stride_t * es,
        dst->stride_b * es, dst->stride_h * es, dst->stride_t * es, src->Hkv, (int)(src->D * es), rows, n,
        dst_row0, src->L_max);
    BSA_LAUNCH_CHECK();
    return BSA_OK;
}

}  // namespace bsa
