// A1 (per-block key summaries) and A8 (decode-step append + incremental
// summary), sm_100a.
//
// Summaries ("Module 14: Sparse attention and long context", §14.3 MoBA,
// mean-pooled here; "Semantic blocks for sparse attention", normalised block
// centres; "Sparse attention in hybrid LLMs", Quest min/max page bounds).
// The arithmetic (fixed order, reproducible bit for bit) is in
// summary_rows.cuh.
#include "summary_rows.cuh"

namespace bsa {

struct SumArgs {
    const void *K;
    void *summ;
    const int32_t *offsets;   // variable blocks or nullptr
    KvRows rows;
    int Hkv, D, L_max, S, nb_total, first_block, kind;
    size_t row_bytes;
};

template <typename T>
__global__ void __launch_bounds__(128) build_summaries_kernel(SumArgs a) {
    extern __shared__ float sm[];
    const int j = a.first_block + blockIdx.x;
    const int s = blockIdx.y;
    const int b = s / a.Hkv, g = s % a.Hkv;
    int64_t r0, r1;
    if (a.offsets) {
        const int32_t *off = a.offsets + (int64_t)s * (a.nb_total + 1);
        r0 = min(max(off[j], 0), a.L_max);
        r1 = min(max(off[j + 1], (int32_t)r0), a.L_max);
    } else {
        r0 = (int64_t)j * a.S;
        r1 = r0 + a.S;
    }
    char *out = static_cast<char *>(a.summ) + ((int64_t)s * a.nb_total + j) * a.row_bytes;
    summarize_rows<T>(static_cast<const T *>(a.K), a.rows, b, g, a.D, r0, r1, a.kind, out, sm);
}

struct AppendArgs {
    void *K, *V;
    const void *k_new, *v_new;
    int32_t *cur_len;
    void *summ;
    KvRows rows;
    int Hkv, D, L_max, S, nb_total, kind;
    size_t row_bytes;
};

template <typename T>
__global__ void __launch_bounds__(256) append_kernel(AppendArgs a) {
    extern __shared__ float sm[];
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x;
    const int n = a.cur_len[b];
    if (n < 0 || n >= a.L_max) return;
    T *K = static_cast<T *>(a.K);
    T *V = static_cast<T *>(a.V);
    const T *kn = static_cast<const T *>(a.k_new) + (int64_t)b * a.Hkv * a.D;
    const T *vn = static_cast<const T *>(a.v_new) + (int64_t)b * a.Hkv * a.D;
    for (int e = threadIdx.x; e < a.Hkv * a.D; e += blockDim.x) {
        const int g = e / a.D, i = e % a.D;
        const int64_t o = a.rows.off(b, g, n);
        if (o < 0) continue;   // the row's page is outside the pool
        K[o + i] = kn[e];
        V[o + i] = vn[e];
    }
    __syncthreads();
    if (a.summ && a.S > 0 && (n + 1) % a.S == 0) {
        const int j = (n + 1) / a.S - 1;
        for (int g = 0; g < a.Hkv; ++g) {
            const int s = b * a.Hkv + g;
            char *out = static_cast<char *>(a.summ) + ((int64_t)s * a.nb_total + j) * a.row_bytes;
            summarize_rows<T>(K, a.rows, b, g, a.D, (int64_t)j * a.S, (int64_t)(j + 1) * a.S,
                              a.kind, out, sm);
            __syncthreads();
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) a.cur_len[b] = n + 1;
}

static size_t summary_smem(int kind, int D) {
    return kind == BSA_SUM_CENTROID_NORM ? (size_t)(kNormChunk * (D + 1) + D + 1) * 4 : 16;
}

bsa_status launch_build_summaries(const bsa_kv_desc *d, const void *K, const bsa_sel_params *p,
                                  int kind, int first_block, int n_blocks, int nb_total,
                                  void *summ, cudaStream_t st) {
    SumArgs a;
    a.K = K; a.summ = summ;
    a.offsets = p->block_size == 0 ? p->block_offsets : nullptr;
    a.rows = kv_rows(d);
    a.Hkv = d->Hkv; a.D = d->D; a.L_max = d->L_max; a.S = p->block_size;
    a.nb_total = nb_total; a.first_block = first_block; a.kind = kind;
    a.row_bytes = summary_row_bytes(kind, d->D, d->kv_dtype);
    dim3 grid(n_blocks, d->B * d->Hkv);
    size_t smem = summary_smem(kind, d->D);
    if (d->kv_dtype == BSA_BF16)
        build_summaries_kernel<uint16_t><<<grid, 128, smem, st>>>(a);
    else if (d->kv_dtype == BSA_FP8_E4M3)
        build_summaries_kernel<uint8_t><<<grid, 128, smem, st>>>(a);
    else
        build_summaries_kernel<float><<<grid, 128, smem, st>>>(a);
    BSA_LAUNCH_CHECK();
    return BSA_OK;
}

bsa_status launch_append(const bsa_kv_desc *d, void *K, void *V, const void *kn, const void *vn,
                         int32_t *cur_len, const bsa_sel_params *p, int kind, int nb_total,
                         void *summ, cudaStream_t st) {
    AppendArgs a;
    a.K = K; a.V = V; a.k_new = kn; a.v_new = vn; a.cur_len = cur_len;
    a.summ = (p && p->block_size > 0) ? summ : nullptr;
    a.rows = kv_rows(d);
    a.Hkv = d->Hkv; a.D = d->D; a.L_max = d->L_max; a.S = p ? p->block_size : 0;
    a.nb_total = nb_total; a.kind = kind;
    a.row_bytes = summary_row_bytes(kind, d->D, d->kv_dtype);
    size_t smem = summary_smem(kind, d->D);
    if (d->kv_dtype == BSA_BF16)
        BSA_CUDA_TRY(launch_pdl(append_kernel<uint16_t>, dim3(d->B), dim3(256), smem, st, a));
    else if (d->kv_dtype == BSA_FP8_E4M3)
        BSA_CUDA_TRY(launch_pdl(append_kernel<uint8_t>, dim3(d->B), dim3(256), smem, st, a));
    else
        BSA_CUDA_TRY(launch_pdl(append_kernel<float>, dim3(d->B), dim3(256), smem, st, a));
    BSA_LAUNCH_CHECK();
    return BSA_OK;
}

}  // namespace bsa
