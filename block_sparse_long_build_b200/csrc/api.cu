// C ABI of libbsa: argument validation, workspace layout and dispatch.
// Declarations and semantics: include/bsa.h.
#include <algorithm>
#include <mutex>

#include "summary_rows.cuh"

namespace bsa {

bsa_status launch_build_summaries(const bsa_kv_desc *, const void *, const bsa_sel_params *, int,
                                  int, int, int, void *, cudaStream_t);
bsa_status launch_append(const bsa_kv_desc *, void *, void *, const void *, const void *, int32_t *,
                         const bsa_sel_params *, int, int, void *, cudaStream_t);
bsa_status launch_select(const bsa_kv_desc *, const float *, const void *, int,
                         const bsa_sel_params *, const int32_t *, int, int, int32_t *, int32_t *,
                         int, int32_t *, int32_t *, uint32_t *, int32_t *, uint32_t *, uint32_t *,
                         cudaStream_t);
bsa_status launch_decode(const bsa_kv_desc *, const float *, const void *, const void *,
                         const int32_t *, const int32_t *, int, const int32_t *, int, float, float *,
                         float *, uint32_t *, uint32_t *, void *, cudaStream_t, const DecAppend *);
bool decode_can_fuse_append(const bsa_kv_desc *);
int decode_nsplit(const bsa_kv_desc *, int, int);
int decode_kernel_count(const bsa_kv_desc *, int, int);
size_t decode_scratch_bytes(const bsa_kv_desc *, int);
bsa_status launch_prefill(const bsa_kv_desc *, const void *, const void *, const bsa_sel_params *,
                          const void *, const bsa_kv_desc *, const void *, const void *, int,
                          const void *, int, int, float, float *, float *, uint32_t *, void *,
                          size_t, cudaStream_t);
size_t prefill_ws_bytes(const bsa_kv_desc *, const bsa_sel_params *, int);
size_t kmeans_ws_bytes(const bsa_kv_desc *, int64_t, int);
bool kmeans_supported(const bsa_kv_desc *, int);
bsa_status launch_kmeans(const bsa_kv_desc *, const void *, int64_t, int, int, const int32_t *, float *,
                         int32_t *, int32_t *, int32_t *, void *, cudaStream_t);
bsa_status launch_gather_rows(const bsa_kv_desc *, const void *, const void *, const bsa_kv_desc *, void *,
                              void *, const int32_t *, int64_t, int64_t, cudaStream_t);

int num_sms() {
    static int n = 0;
    static std::once_flag once;
    std::call_once(once, [] {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
            n = v;
        else
            n = 148;
        cudaGetLastError();
    });
    return n;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        cudaGetLastError();
    });
    return fn;
}

bool make_kv_tmap(CUtensorMap *map, const bsa_kv_desc *d, const void *base, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const bool paged = d->page_rows > 0;
    const cuuint64_t dims[4] = {(cuuint64_t)d->D, (cuuint64_t)(paged ? d->page_rows : d->L_max),
                                (cuuint64_t)d->Hkv, (cuuint64_t)(paged ? d->n_pages : d->B)};
    const cuuint64_t es = d->kv_dtype == BSA_FP8_E4M3 ? 1 : 2;   // bf16 or FP8 codes
    const cuuint64_t strides[3] = {(cuuint64_t)d->stride_t * es, (cuuint64_t)d->stride_h * es,
                                   (cuuint64_t)d->stride_b * es};
    const cuuint32_t box[4] = {(cuuint32_t)(128 / es), (cuuint32_t)box_rows, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, es == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                    const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_rows_tmap(CUtensorMap *map, CUtensorMapDataType dtype, int esize, const void *base,
                    int64_t cols, int64_t rows, int64_t row_bytes, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)(128 / esize), (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------- validation
static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

static int elem_size(const bsa_kv_desc *d) {
    return d->kv_dtype == BSA_F32 ? 4 : d->kv_dtype == BSA_BF16 ? 2 : 1;
}

static bool desc_ok(const bsa_kv_desc *d) {
    if (!d) return false;
    if (d->B < 1 || d->Hkv < 1 || d->Hq < d->Hkv || d->Hq % d->Hkv != 0) return false;
    if (d->D != 64 && d->D != 128) return false;
    if (d->kv_dtype != BSA_F32 && d->kv_dtype != BSA_BF16 && d->kv_dtype != BSA_FP8_E4M3) return false;
    if (d->L_max < 1) return false;
    if (d->stride_t < d->D || d->stride_h < 1 || d->stride_b < 1) return false;
    const int64_t es = elem_size(d);
    if ((d->stride_t * es) % 16 || (d->stride_h * es) % 16 || (d->stride_b * es) % 16) return false;
    if (d->page_rows < 0) return false;
    if (d->page_rows > 0) {   // paged pool
        if (d->page_rows % 16 || d->pages_per_seq < 1 || !d->page_table || d->n_pages < 1 ||
            d->n_pages > 0x7fffffffLL || (int64_t)d->pages_per_seq * d->page_rows != d->L_max)
            return false;
    }
    return true;
}

static bool sel_ok(const bsa_kv_desc *d, const bsa_sel_params *p) {
    if (!p || p->block_size < 0) return false;
    if (p->topk < 0 && p->budget_tokens < 0) return false;
    if (p->sink < 0 || p->window < 0) return false;
    if (p->block_size == 0) {
        if (p->n_blocks < 1 || !p->block_offsets || !p->kv_pos) return false;
        if (p->local_start < 0 || p->local_start > d->L_max) return false;
    }
    return true;
}

static int nb_total(const bsa_kv_desc *d, const bsa_sel_params *p) {
    return p->block_size > 0 ? (int)div_up(d->L_max, p->block_size) : p->n_blocks;
}

static int max_selected(const bsa_kv_desc *d, const bsa_sel_params *p) {
    const int nb = nb_total(d, p);
    if (p->topk >= 0) return std::max(1, std::min(p->topk, nb));
    if (p->block_size > 0) return std::max(1, std::min(p->budget_tokens / p->block_size, nb));
    return nb;
}

static int max_ranges(const bsa_kv_desc *d, const bsa_sel_params *p) {
    return max_selected(d, p) + 4;
}

// Workspace: [status u32][select counters: nseg][decode counters: nseg],
// padded to 256 bytes, then the op's scratch.
static size_t counters_bytes(const bsa_kv_desc *d) {
    return align_up((size_t)(1 + 2 * d->B * d->Hkv) * 4, 256);
}

static bool ws_ok(const void *ws, size_t have, size_t need) {
    return ws && aligned16(ws) && have >= need;
}

// Host-side checks shared by every decode entry point (bsa_decode,
// bsa_decode_step, bsa_decode_noalloc): BSA_OK or the error to return before
// anything touches device memory.
bsa_status decode_check_args(const bsa_kv_desc *d, const float *q, const void *K, const void *V,
                             const int32_t *ranges, const int32_t *n_ranges, int32_t max_r,
                             const int32_t *cur_len, int32_t tokens_hint, float scale,
                             const float *out) {
    if (!desc_ok(d)) return BSA_ERR_ARG;
    if (!q || !K || !V || !ranges || !n_ranges || !cur_len || !out) return BSA_ERR_ARG;
    if (!aligned16(K) || !aligned16(V) || !aligned16(q)) return BSA_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(ranges) % 8) return BSA_ERR_ARG;
    if (max_r < 1 || max_r > 4096 || tokens_hint < 0) return BSA_ERR_ARG;
    if (d->Hq / d->Hkv > kMaxG) return BSA_ERR_UNSUPPORTED;
    if (!(scale > 0.0f) || scale != scale) return BSA_ERR_ARG;
    return BSA_OK;
}

// Bytes of the status word + counters area at the start of a workspace.
size_t ws_counters_bytes(const bsa_kv_desc *d) { return counters_bytes(d); }

void *noalloc_scratch_on_current_context();
void arm_decode_wait_limit(uint32_t limit_ns);

}  // namespace bsa

using namespace bsa;

extern "C" {

int32_t bsa_version(void) { return 100; }

const char *bsa_status_string(bsa_status s) {
    switch (s) {
        case BSA_OK: return "ok";
        case BSA_ERR_ARG: return "invalid argument";
        case BSA_ERR_UNSUPPORTED: return "unsupported shape or option";
        case BSA_ERR_CUDA: return "CUDA error";
        case BSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case BSA_ERR_TIMEOUT: return "device-side wait timed out";
        case BSA_ERR_CAPACITY: return "a per-query limit was reached; result truncated";
    }
    return "unknown status";
}

bsa_status bsa_workspace_status(const void *ws, size_t ws_bytes, int32_t clear, uint32_t *bits,
                                bsa_stream_t stream) {
    void *word = const_cast<void *>(ws);
    if (!word) {
        word = noalloc_scratch_on_current_context();
        if (!word) return BSA_ERR_CUDA;
    } else if (ws_bytes < 4 || (reinterpret_cast<uintptr_t>(ws) & 3)) {
        return BSA_ERR_WORKSPACE;
    }
    const cudaStream_t st = (cudaStream_t)stream;
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, word, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        (clear && cudaMemsetAsync(word, 0, 4, st) != cudaSuccess) ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return BSA_ERR_CUDA;
    }
    if (bits) *bits = v;
    if (v & (1u | 2u | 8u)) return BSA_ERR_TIMEOUT;
    if (v) return BSA_ERR_CAPACITY;
    return BSA_OK;
}

bsa_status bsa_test_arm_wait_limit(int32_t limit_us) {
    if (limit_us < 0 || limit_us > 100000) return BSA_ERR_ARG;
    arm_decode_wait_limit((uint32_t)limit_us * 1000u);
    return BSA_OK;
}

int32_t bsa_summary_blocks(const bsa_kv_desc *d, const bsa_sel_params *p) {
    if (!desc_ok(d) || !sel_ok(d, p)) return -1;
    return nb_total(d, p);
}

size_t bsa_summary_bytes(const bsa_kv_desc *d, const bsa_sel_params *p, bsa_summary_kind kind) {
    if (!desc_ok(d) || !sel_ok(d, p)) return 0;
    if (kind < BSA_SUM_CENTROID || kind > BSA_SUM_MINMAX) return 0;
    // the row size the kernels write: bf16 bounds for bf16 and FP8 caches
    return (size_t)d->B * d->Hkv * nb_total(d, p) * summary_row_bytes(kind, d->D, d->kv_dtype);
}

int32_t bsa_max_selected(const bsa_kv_desc *d, const bsa_sel_params *p) {
    if (!desc_ok(d) || !sel_ok(d, p)) return -1;
    return max_selected(d, p);
}

int32_t bsa_max_ranges(const bsa_kv_desc *d, const bsa_sel_params *p) {
    if (!desc_ok(d) || !sel_ok(d, p)) return -1;
    return max_ranges(d, p);
}

size_t bsa_index_workspace_size(const bsa_kv_desc *d, int64_t L, int32_t k) {
    if (!desc_ok(d) || L < 1 || L > d->L_max || L > 0x7fffffffLL || k < 1 || k > L) return 0;
    return kmeans_ws_bytes(d, L, k);
}

bsa_status bsa_build_semantic_index(const bsa_kv_desc *d, const void *K, int64_t L, int32_t k,
                                    int32_t iters, const int32_t *init, float *centres, int32_t *labels,
                                    int32_t *offsets, int32_t *order, void *ws, size_t ws_bytes,
                                    bsa_stream_t stream) {
    if (!desc_ok(d) || !K || !init || !centres || !labels || !offsets || !order) return BSA_ERR_ARG;
    if (L < 1 || L > d->L_max || L > 0x7fffffffLL || k < 1 || k > L || iters < 1) return BSA_ERR_ARG;
    if (!aligned16(K) || !aligned16(centres)) return BSA_ERR_ARG;
    if (d->page_rows > 0 || d->kv_dtype == BSA_FP8_E4M3 || !kmeans_supported(d, k))
        return BSA_ERR_UNSUPPORTED;
    if (!ws_ok(ws, ws_bytes, kmeans_ws_bytes(d, L, k))) return BSA_ERR_WORKSPACE;
    return launch_kmeans(d, K, L, k, iters, init, centres, labels, offsets, order, ws, (cudaStream_t)stream);
}

bsa_status bsa_gather_rows(const bsa_kv_desc *src, const void *K, const void *V, const bsa_kv_desc *dst,
                           void *K_out, void *V_out, const int32_t *rows, int64_t n, int64_t dst_row0,
                           bsa_stream_t stream) {
    if (!desc_ok(src) || !desc_ok(dst) || !K || !V || !K_out || !V_out || !rows) return BSA_ERR_ARG;
    if (src->B != dst->B || src->Hkv != dst->Hkv || src->D != dst->D || src->kv_dtype != dst->kv_dtype)
        return BSA_ERR_ARG;
    if (!aligned16(K) || !aligned16(V) || !aligned16(K_out) || !aligned16(V_out)) return BSA_ERR_ARG;
    if (src->page_rows > 0 || dst->page_rows > 0) return BSA_ERR_UNSUPPORTED;
    if (n < 0 || dst_row0 < 0 || dst_row0 + n > dst->L_max) return BSA_ERR_ARG;
    if (n == 0) return BSA_OK;
    return launch_gather_rows(src, K, V, dst, K_out, V_out, rows, n, dst_row0, (cudaStream_t)stream);
}

int32_t bsa_decode_kernels(const bsa_kv_desc *d, const bsa_sel_params *p, int32_t tokens_hint) {
    if (!desc_ok(d) || !sel_ok(d, p) || tokens_hint < 0) return BSA_ERR_ARG;
    return decode_kernel_count(d, std::max(tokens_hint, 1), max_ranges(d, p));
}

size_t bsa_workspace_size(const bsa_kv_desc *d, const bsa_sel_params *p, int op, int32_t n_queries,
                          int32_t tokens_hint) {
    if (!desc_ok(d)) return 0;
    const size_t cb = counters_bytes(d);
    const size_t nseg = (size_t)d->B * d->Hkv;
    switch (op) {
        case BSA_OP_SELECT:
            if (!sel_ok(d, p)) return 0;
            return cb + align_up(nseg * nb_total(d, p) * 4, 256) * 2;
        case BSA_OP_DECODE: {
            const int mr = p && sel_ok(d, p) ? max_ranges(d, p) : 64;
            return cb + decode_scratch_bytes(d, decode_nsplit(d, std::max(tokens_hint, 1), mr));
        }
        case BSA_OP_APPEND:
            return cb;
        case BSA_OP_PREFILL:
            if (!sel_ok(d, p) || n_queries < 1) return 0;
            return cb + prefill_ws_bytes(d, p, n_queries);
    }
    return 0;
}

bsa_status bsa_build_summaries(const bsa_kv_desc *d, const void *K, const bsa_sel_params *p,
                               bsa_summary_kind kind, int32_t first_block, int32_t n_blocks,
                               void *summaries, bsa_stream_t stream) {
    if (!desc_ok(d) || !sel_ok(d, p) || !K || !summaries || !aligned16(K) || !aligned16(summaries))
        return BSA_ERR_ARG;
    if (kind < BSA_SUM_CENTROID || kind > BSA_SUM_MINMAX) return BSA_ERR_ARG;
    const int nb = nb_total(d, p);
    if (first_block < 0 || n_blocks < 0 || (int64_t)first_block + n_blocks > nb) return BSA_ERR_ARG;
    if (p->block_size > 0 && ((int64_t)first_block + n_blocks) * p->block_size > d->L_max)
        return BSA_ERR_ARG;
    if (n_blocks == 0) return BSA_OK;
    return launch_build_summaries(d, K, p, kind, first_block, n_blocks, nb, summaries,
                                  (cudaStream_t)stream);
}

bsa_status bsa_select(const bsa_kv_desc *d, const float *q, const void *summaries,
                      bsa_summary_kind kind, const bsa_sel_params *p, const int32_t *cur_len,
                      int32_t max_sel, int32_t *sel_blocks, int32_t *sel_count, int32_t max_r,
                      int32_t *ranges, int32_t *n_ranges, void *ws, size_t ws_bytes,
                      bsa_stream_t stream) {
    if (!desc_ok(d) || !sel_ok(d, p)) return BSA_ERR_ARG;
    if (!q || !summaries || !cur_len || !sel_blocks || !sel_count || !ranges || !n_ranges)
        return BSA_ERR_ARG;
    if (!aligned16(q) || !aligned16(summaries)) return BSA_ERR_ARG;
    if (kind < BSA_SUM_CENTROID || kind > BSA_SUM_MINMAX) return BSA_ERR_ARG;
    if (d->Hq / d->Hkv > 16) return BSA_ERR_UNSUPPORTED;
    if (max_sel < max_selected(d, p) || max_r < max_ranges(d, p)) return BSA_ERR_ARG;
    const size_t need = bsa_workspace_size(d, p, BSA_OP_SELECT, 0, 0);
    if (!ws_ok(ws, ws_bytes, need)) return BSA_ERR_WORKSPACE;
    const size_t nseg = (size_t)d->B * d->Hkv;
    const int nb = nb_total(d, p);
    uint32_t *cnt = static_cast<uint32_t *>(ws) + 1;
    char *scr = static_cast<char *>(ws) + counters_bytes(d);
    uint32_t *keys = reinterpret_cast<uint32_t *>(scr);
    int32_t *vis = reinterpret_cast<int32_t *>(scr + align_up(nseg * nb * 4, 256));
    return launch_select(d, q, summaries, kind, p, cur_len, nb, max_sel, sel_blocks, sel_count, max_r,
                         ranges, n_ranges, keys, vis, cnt, static_cast<uint32_t *>(ws),
                         (cudaStream_t)stream);
}

bsa_status bsa_decode(const bsa_kv_desc *d, const float *q, const void *K, const void *V,
                      const int32_t *ranges, const int32_t *n_ranges, int32_t max_r,
                      const int32_t *cur_len, int32_t tokens_hint, float scale, float *out,
                      float *lse, void *ws, size_t ws_bytes, bsa_stream_t stream) {
    const bsa_status chk =
        decode_check_args(d, q, K, V, ranges, n_ranges, max_r, cur_len, tokens_hint, scale, out);
    if (chk != BSA_OK) return chk;
    const int nsplit = decode_nsplit(d, std::max(tokens_hint, 1), max_r);
    const size_t need = counters_bytes(d) + decode_scratch_bytes(d, nsplit);
    if (!ws_ok(ws, ws_bytes, need)) return BSA_ERR_WORKSPACE;
    uint32_t *status = static_cast<uint32_t *>(ws);
    uint32_t *cnt = status + 1 + d->B * d->Hkv;
    void *scr = static_cast<char *>(ws) + counters_bytes(d);
    return launch_decode(d, q, K, V, ranges, n_ranges, max_r, cur_len, std::max(tokens_hint, 1),
                         scale, out, lse, status, cnt, scr, (cudaStream_t)stream, nullptr);
}

bsa_status bsa_decode_step(const bsa_kv_desc *d, const float *q, void *K, void *V,
                           const void *k_new, const void *v_new, int32_t *cur_len,
                           const bsa_sel_params *p, bsa_summary_kind kind, void *summaries,
                           const int32_t *ranges, const int32_t *n_ranges, int32_t max_r,
                           int32_t tokens_hint, float scale, float *out, float *lse, void *ws,
                           size_t ws_bytes, bsa_stream_t stream) {
    // the arguments of both halves, checked before anything is launched
    if (!desc_ok(d) || !K || !V || !k_new || !v_new || !cur_len) return BSA_ERR_ARG;
    if (p && !sel_ok(d, p)) return BSA_ERR_ARG;
    if (summaries && (!p || kind < BSA_SUM_CENTROID || kind > BSA_SUM_MINMAX)) return BSA_ERR_ARG;
    const bsa_status chk =
        decode_check_args(d, q, K, V, ranges, n_ranges, max_r, cur_len, tokens_hint, scale, out);
    if (chk != BSA_OK) return chk;
    const int nsplit = decode_nsplit(d, std::max(tokens_hint, 1), max_r);
    const size_t need = counters_bytes(d) + decode_scratch_bytes(d, nsplit);
    if (!ws_ok(ws, ws_bytes, need)) return BSA_ERR_WORKSPACE;
    const bool fixed_summ = summaries && p && p->block_size > 0;
    const bool fuse = decode_can_fuse_append(d) && aligned16(k_new) && aligned16(v_new) &&
                      (!fixed_summ || kind != BSA_SUM_CENTROID_NORM);
    if (!fuse) {   // the same two steps as separate launches
        const bsa_status r = bsa_append_kv(d, K, V, k_new, v_new, cur_len, p, kind, summaries, stream);
        if (r != BSA_OK) return r;
        return bsa_decode(d, q, K, V, ranges, n_ranges, max_r, cur_len, tokens_hint, scale, out, lse,
                          ws, ws_bytes, stream);
    }
    DecAppend app;
    app.k_new = k_new;
    app.v_new = v_new;
    app.cur_len = cur_len;
    app.summ = fixed_summ ? summaries : nullptr;
    app.S = p ? p->block_size : 0;
    app.nb_total = p ? nb_total(d, p) : 0;
    app.kind = kind;
    app.row_bytes = (int)summary_row_bytes(kind, d->D, d->kv_dtype);
    uint32_t *status = static_cast<uint32_t *>(ws);
    uint32_t *cnt = status + 1 + d->B * d->Hkv;
    void *scr = static_cast<char *>(ws) + counters_bytes(d);
    return launch_decode(d, q, K, V, ranges, n_ranges, max_r, cur_len, std::max(tokens_hint, 1),
                         scale, out, lse, status, cnt, scr, (cudaStream_t)stream, &app);
}

bsa_status bsa_append_kv(const bsa_kv_desc *d, void *K, void *V, const void *k_new,
                         const void *v_new, int32_t *cur_len, const bsa_sel_params *p,
                         bsa_summary_kind kind, void *summaries, bsa_stream_t stream) {
    if (!desc_ok(d) || !K || !V || !k_new || !v_new || !cur_len) return BSA_ERR_ARG;
    if (p && !sel_ok(d, p)) return BSA_ERR_ARG;
    if (summaries && (!p || kind < BSA_SUM_CENTROID || kind > BSA_SUM_MINMAX)) return BSA_ERR_ARG;
    const int nb = p ? nb_total(d, p) : 0;
    return launch_append(d, K, V, k_new, v_new, cur_len, p, kind, nb, summaries,
                         (cudaStream_t)stream);
}

bsa_status bsa_prefill_grouped(const bsa_kv_desc *d, const void *K, const void *V,
                               const bsa_sel_params *p, const void *summaries,
                               const bsa_kv_desc *pd, const void *K_pos, const void *V_pos,
                               int32_t pos_base, const void *Q, int32_t q_pos0, int32_t Tq,
                               float scale, float *out, float *lse, void *ws, size_t ws_bytes,
                               bsa_stream_t stream) {
    if (!desc_ok(d) || !desc_ok(pd) || !sel_ok(d, p)) return BSA_ERR_ARG;
    if (!K || !V || !summaries || !K_pos || !V_pos || !Q || !out) return BSA_ERR_ARG;
    if (!aligned16(K) || !aligned16(V) || !aligned16(K_pos) || !aligned16(V_pos) || !aligned16(Q) ||
        !aligned16(out) || !aligned16(summaries))
        return BSA_ERR_ARG;
    if (p->block_size != 0 || p->topk >= 0) return BSA_ERR_UNSUPPORTED;
    if (d->page_rows > 0 || pd->page_rows > 0) return BSA_ERR_UNSUPPORTED;
    if (d->B != 1 || pd->B != 1 || d->Hkv != pd->Hkv || d->Hq != pd->Hq || d->D != pd->D)
        return BSA_ERR_ARG;
    if (d->kv_dtype != BSA_BF16 || pd->kv_dtype != BSA_BF16 || d->D != 128) return BSA_ERR_UNSUPPORTED;
    if (d->stride_t != d->D || pd->stride_t != pd->D) return BSA_ERR_UNSUPPORTED;
    // the window K_pos/V_pos holds positions [pos_base, pos_base + pd->L_max): every
    // local key, [pos_limit, q_pos0 + Tq), must be in it
    if (Tq < 1 || q_pos0 < 0 || p->pos_limit < 0 || p->pos_limit > q_pos0 || pos_base < 0 ||
        pos_base > p->pos_limit || (int64_t)q_pos0 + Tq - pos_base > pd->L_max)
        return BSA_ERR_ARG;
    if (!(scale > 0.0f)) return BSA_ERR_ARG;
    const size_t need = bsa_workspace_size(d, p, BSA_OP_PREFILL, Tq, 0);
    if (!ws_ok(ws, ws_bytes, need)) return BSA_ERR_WORKSPACE;
    return launch_prefill(d, K, V, p, summaries, pd, K_pos, V_pos, pos_base, Q, q_pos0, Tq, scale, out, lse,
                          static_cast<uint32_t *>(ws), static_cast<char *>(ws) + counters_bytes(d),
                          ws_bytes - counters_bytes(d), (cudaStream_t)stream);
}

}  // extern "C"
