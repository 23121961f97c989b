// Per-block key summaries, computed by one CTA (shared by the summary build,
// the append step and the fused decode step).
//
// The arithmetic order is fixed so that the scores computed from these
// summaries, and hence the selected blocks, are reproducible bit for bit:
//   centroid       c[i] = (((0 + k_r0[i]) + k_r1[i]) + ...) / n   (rows in order)
//   centroid_norm  u_r = k_r / ||k_r|| (||.|| = sqrt of an fma chain over i),
//                  m = mean of u_r as above, c = m / ||m||
//   minmax         running min / max over rows in order (first wins on ties)
#pragma once
#include <type_traits>

#include "common.cuh"

namespace bsa {

constexpr int kNormChunk = 64;   // rows staged at once for the per-row norms

// fp32 norm of a row held in shared memory: fma chain over i, then sqrt.
__device__ __forceinline__ float row_norm_f32(const float *x, int D) {
    float acc = 0.0f;
    for (int i = 0; i < D; ++i) acc = __fmaf_rn(x[i], x[i], acc);
    return __fsqrt_rn(acc);
}

// Element i of logical row r of segment (b, g); zero for a row whose page
// is outside the pool.
template <typename T>
__device__ __forceinline__ float row_elem(const T *K, const KvRows &kr, int b, int g, int64_t r,
                                          int i) {
    const int64_t o = kr.off(b, g, r);
    return o < 0 ? 0.0f : load_elem(K, o + i);
}

// Element i of rows r .. r + 3 of segment (b, g), the loads issued together.
template <typename T>
__device__ __forceinline__ void row_elems4(const T *K, const KvRows &kr, int b, int g, int64_t r,
                                           int i, float (&v)[4]) {
    if (!kr.table) {   // contiguous: one base, a fixed row stride
        const T *p = K + b * kr.stride_b + g * kr.stride_h + r * kr.stride_t + i;
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = load_elem(p, e * kr.stride_t);
    } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = row_elem(K, kr, b, g, r + e, i);
    }
}

// Centroid of rows [r0, r1): thread i < D sums dimension i in row order.
template <typename T>
__device__ __forceinline__ void summarize_centroid(const T *K, const KvRows &kr, int b, int g, int D,
                                                   int64_t r0, int64_t r1, float *out) {
    const int i = threadIdx.x;
    const int64_t n = r1 - r0;
    if (i < D) {
        float acc = 0.0f;
        int64_t r = r0;
        for (; r + 4 <= r1; r += 4) {   // loads batched, adds stay in order
            float v[4];
            row_elems4(K, kr, b, g, r, i, v);
            acc = __fadd_rn(acc, v[0]);
            acc = __fadd_rn(acc, v[1]);
            acc = __fadd_rn(acc, v[2]);
            acc = __fadd_rn(acc, v[3]);
        }
        for (; r < r1; ++r) acc = __fadd_rn(acc, row_elem(K, kr, b, g, r, i));
        out[i] = n > 0 ? __fdiv_rn(acc, (float)n) : 0.0f;
    }
}

// Element type of MINMAX summaries for a cache of T: the cache dtype, bf16
// (exact) for an FP8 cache.
template <typename T>
using minmax_t = std::conditional_t<sizeof(T) == 4, float, uint16_t>;

// Min/max of rows [r0, r1), stored as (min, max) pairs per dimension (fp32
// or bf16 bits): thread i < D scans dimension i in row order.
template <typename T>
__device__ __forceinline__ void summarize_minmax(const T *K, const KvRows &kr, int b, int g, int D,
                                                 int64_t r0, int64_t r1, minmax_t<T> *o) {
    const int i = threadIdx.x;
    const int64_t n = r1 - r0;
    if (i < D) {
        float lo = __int_as_float(0x7f800000), hi = __int_as_float(0xff800000);  // +inf, -inf
        int64_t r = r0;
        for (; r + 4 <= r1; r += 4) {   // loads batched, rows scanned in order
            float v[4];
            row_elems4(K, kr, b, g, r, i, v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (v[e] < lo) lo = v[e];
                if (v[e] > hi) hi = v[e];
            }
        }
        for (; r < r1; ++r) {
            const float v = row_elem(K, kr, b, g, r, i);
            if (v < lo) lo = v;
            if (v > hi) hi = v;
        }
        if (n <= 0) lo = hi = 0.0f;
        if constexpr (sizeof(T) <= 2) {   // bf16 and FP8 values are bf16 values: exact
            o[2 * i] = static_cast<uint16_t>(__float_as_uint(lo) >> 16);
            o[2 * i + 1] = static_cast<uint16_t>(__float_as_uint(hi) >> 16);
        } else {
            o[2 * i] = lo;
            o[2 * i + 1] = hi;
        }
    }
}

// Summary of rows [r0, r1) of segment (b, g), computed by the whole CTA
// (blockDim.x >= D).  `out` points at this block's summary: D floats for the
// centroid kinds, D (min, max) pairs of cache elements for MINMAX.
// `sm` must hold kNormChunk*(D+1) + D + 1 floats.
template <typename T>
__device__ void summarize_rows(const T *K, const KvRows &kr, int b, int g, int D, int64_t r0,
                               int64_t r1, int kind, void *out, float *sm) {
    const int i = threadIdx.x;
    const int64_t n = r1 - r0;
    if (kind == BSA_SUM_CENTROID) {
        summarize_centroid<T>(K, kr, b, g, D, r0, r1, static_cast<float *>(out));
        return;
    }
    if (kind == BSA_SUM_MINMAX) {
        summarize_minmax<T>(K, kr, b, g, D, r0, r1, static_cast<minmax_t<T> *>(out));
        return;
    }
    // BSA_SUM_CENTROID_NORM
    float *rows = sm;                              // [kNormChunk][D+1]
    float *nrm = sm + kNormChunk * (D + 1);        // [kNormChunk] (aliases the tail)
    float acc = 0.0f;
    for (int64_t c0 = r0; c0 < r1; c0 += kNormChunk) {
        const int cn = (int)((r1 - c0) < kNormChunk ? (r1 - c0) : kNormChunk);
        __syncthreads();
        for (int e = threadIdx.x; e < cn * D; e += blockDim.x) {
            int rr = e / D, ii = e % D;
            rows[rr * (D + 1) + ii] = row_elem(K, kr, b, g, c0 + rr, ii);
        }
        __syncthreads();
        if (threadIdx.x < cn) nrm[threadIdx.x] = row_norm_f32(rows + threadIdx.x * (D + 1), D);
        __syncthreads();
        if (i < D) {
            for (int rr = 0; rr < cn; ++rr) {
                float nr = nrm[rr];
                acc = __fadd_rn(acc, nr > 0.0f ? __fdiv_rn(rows[rr * (D + 1) + i], nr) : 0.0f);
            }
        }
    }
    __syncthreads();
    float *mean = sm;   // reuse
    if (i < D) mean[i] = n > 0 ? __fdiv_rn(acc, (float)n) : 0.0f;
    __syncthreads();
    if (threadIdx.x == 0) mean[D] = row_norm_f32(mean, D);
    __syncthreads();
    if (i < D) {
        float nc = mean[D];
        static_cast<float *>(out)[i] = nc > 0.0f ? __fdiv_rn(mean[i], nc) : 0.0f;
    }
    __syncthreads();
}

__host__ __device__ inline size_t summary_row_bytes(int kind, int D, int kv_dtype) {
    return kind == BSA_SUM_MINMAX ? (size_t)2 * D * (kv_dtype == BSA_F32 ? 4 : 2)
                                  : (size_t)D * 4;
}

}  // namespace bsa
