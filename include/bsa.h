/*
 * bsa.h -- C ABI of the block-sparse long-context attention library
 * (libbsa.so, CUDA for sm_100a).
 *
 * What the library computes (page title, section):
 *   1. Per-block key summaries: mean-pooled centroids ("Module 14: Sparse
 *      attention and long context", §14.3 MoBA -- the mean stands in for
 *      MoBA's learned gate key), normalised centres of normalised keys
 *      ("Semantic blocks for sparse attention", first section), or Quest-style
 *      elementwise min/max page bounds ("Sparse attention in hybrid LLMs",
 *      "Which parts of the context each layer reads").
 *   2. Block scores against the current query, summed over the G query heads
 *      of a KV head, and the top-k blocks or the blocks a token budget admits
 *      ("Sparse long-context inference with self-indexing attention",
 *      "Importance scores and block selection"), always with the attention
 *      sink (§14.2), the sliding window ("Sliding window") and, MoBA-style,
 *      the current block.
 *   3. Exact softmax attention with GQA over only the selected tokens
 *      (Module 14, Exercise 14.1), as split-K flash decoding with a
 *      log-sum-exp merge.
 *   4. Block-grouped prefill: queries that selected the same block are
 *      gathered and contracted against that block once ("Semantic blocks for
 *      sparse attention", "Large blocks make up for coarse selection with
 *      speed").
 *
 * Conventions (all entry points):
 *  - Pointers named d_* or documented "device" are CUDA device pointers;
 *    descriptors and parameter structs are host pointers read during the call
 *    only.  The caller owns every buffer, including the workspace; the
 *    library allocates nothing.  Between calls it keeps only per-process
 *    caches of device properties (SM count, cluster occupancy, the tensor-map
 *    encoder) and, for bsa_decode_noalloc, its built-in scratch array and
 *    that array's address per CUDA context.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  BSA_OK means "validated and launched"; a failed launch returns
 *    BSA_ERR_CUDA.  Results are ready when the stream reaches them.
 *  - Validation is host-side and touches no device memory: a bad argument
 *    returns BSA_ERR_ARG (or BSA_ERR_UNSUPPORTED for a valid but unbuilt
 *    case) and launches nothing.
 *  - KV caches are [B][Hkv][L_max][D] with element strides stride_b,
 *    stride_h, stride_t and D contiguous; the base must be 16-byte aligned
 *    and stride_t * element size a multiple of 16 bytes.  Query head h reads
 *    KV head h / G, G = Hq / Hkv.
 *  - A segment is one (batch b, KV head g) pair, index s = b * Hkv + g.
 *  - Token ranges are half-open [start, end) row indices into a segment.
 *  - Workspace: size from bsa_workspace_size(); it must be zero-filled once
 *    before its first use.  Every call leaves its counters at zero again, so
 *    one workspace can serve any sequence of calls on one stream.  Calls that
 *    may overlap on the GPU need separate workspaces.
 *  - Device-side errors: the first 4 bytes of a workspace are a sticky status
 *    word that kernels set and never clear: bit 0 a decode wait for a tile
 *    copy gave up, bit 1 a selection wait gave up (or a scoring CTA found
 *    its shared memory misaligned for the swizzled copies and scored
 *    nothing), bit 3 a prefill wait gave up (each BSA_ERR_TIMEOUT; the call
 *    finished with partial data), bit 2 a
 *    prefill query had more blocks within its budget than the 64 the library
 *    keeps (BSA_ERR_CAPACITY; that query's block list was cut at 64).  Read
 *    and clear it with bsa_workspace_status().
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BSA_API __attribute__((visibility("default")))
#else
#define BSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *bsa_stream_t;   /* == cudaStream_t */

typedef enum {
    BSA_OK = 0,
    BSA_ERR_ARG = -1,          /* invalid argument; nothing launched            */
    BSA_ERR_UNSUPPORTED = -2,  /* valid, but a shape the library does not cover */
    BSA_ERR_CUDA = -3,         /* a CUDA call or launch failed                  */
    BSA_ERR_WORKSPACE = -4,    /* workspace missing, misaligned or too small    */
    BSA_ERR_TIMEOUT = -5,      /* a bounded device-side wait gave up            */
    BSA_ERR_CAPACITY = -6      /* a per-query limit of the library was reached
                                  and the result was truncated                 */
} bsa_status;

typedef enum {
    BSA_SUM_CENTROID = 0,       /* fp32 mean of the block's keys                  */
    BSA_SUM_CENTROID_NORM = 1,  /* fp32 normalised mean of normalised keys        */
    BSA_SUM_MINMAX = 2          /* elementwise (min, max) pairs, cache dtype      */
} bsa_summary_kind;

/* Element types of K and V.  BSA_FP8_E4M3 ("Attention mechanisms in modern
 * LLMs", basic maths and the real cost: the cache may be kept in FP8):
 * 1 sign, 4 exponent (bias 7) and 3 mantissa bits, exponent 0 subnormal,
 * S.1111.111 NaN, no infinity (largest finite 448).  For an FP8 cache, MINMAX
 * summaries hold the bounds as bf16 (exact), and the decode reads 1 byte per
 * element; D must be 128 on the tensor-core path (D 64 runs on CUDA cores). */
typedef enum { BSA_F32 = 0, BSA_BF16 = 1, BSA_FP8_E4M3 = 2 } bsa_dtype;

typedef enum { BSA_OP_SELECT = 0, BSA_OP_DECODE = 1, BSA_OP_PREFILL = 2, BSA_OP_APPEND = 3 } bsa_op;

/* KV-cache geometry.
 *
 * Contiguous cache (page_rows = 0): K and V are [B][Hkv][L_max][D] with
 * element strides stride_b, stride_h, stride_t.
 *
 * Paged cache (page_rows > 0; "Sparse long-context inference with
 * self-indexing attention", "How much memory the KV cache takes": the cache
 * held as fixed-size pages): K and V point at a pool of n_pages pages,
 * [n_pages][Hkv][page_rows][D] with element strides stride_b (between
 * pages), stride_h, stride_t.  Logical row r of sequence b, KV head g lives in
 * page page_table[b * pages_per_seq + r / page_rows] at row r % page_rows.
 * page_rows is a multiple of 16, L_max = pages_per_seq * page_rows, and every
 * table entry a sequence's rows [0, L_max) can reach must be in
 * [0, n_pages): a decode reads zeros for rows whose entry is outside, and
 * appends skip them.  Sequences may share pages.  The page table is device
 * memory the caller owns; selection outputs stay in logical rows. */
typedef struct {
    int32_t B, Hq, Hkv, D;     /* D in {64, 128}; Hq a multiple of Hkv            */
    int32_t kv_dtype;          /* bsa_dtype of K and V                             */
    int32_t L_max;             /* rows per segment                                 */
    int64_t stride_b, stride_h, stride_t;   /* element strides of K and V          */
    int32_t page_rows;         /* 0: contiguous; else rows per page               */
    int32_t pages_per_seq;     /* paged: table entries per sequence               */
    const int32_t *page_table; /* paged: device int32 [B][pages_per_seq]          */
    int64_t n_pages;           /* paged: pages in the pool                        */
} bsa_kv_desc;

/* Selection parameters, in the pages' terms.
 *
 * Fixed blocks (block_size = S > 0): block j of a segment is rows
 * [j*S, (j+1)*S).  For a cache of n tokens (the newest, the current token,
 * is row n-1) the forced set is
 *     sink     [0, min(sink, n))
 *     window   [max(0, n - window), n)      -- the window counts the current token
 *     current  [floor((n-1)/S)*S, n)        -- when keep_current_block != 0
 * The candidates are the complete blocks ((j+1)*S <= n) not wholly inside the
 * forced set; k = topk, or budget_tokens / S when topk < 0.  The k candidates
 * with the highest scores are selected, the lower block index first among
 * equal fp32 scores.
 *
 * Variable blocks (block_size = 0): block j of segment s is rows
 * [block_offsets[s][j], block_offsets[s][j+1]) of a store whose rows are
 * sorted by original position inside each block (kv_pos[s][row]).  A block's
 * visible rows are those with kv_pos < pos_limit (a prefix of the block);
 * blocks with none are not candidates.  Blocks are taken greedily in rank
 * order while their visible rows fit in what is left of budget_tokens.  The
 * forced set is the position-ordered local part [local_start, n). */
typedef struct {
    int32_t block_size;
    int32_t n_blocks;               /* variable blocks: blocks per segment        */
    const int32_t *block_offsets;   /* device [B*Hkv][n_blocks+1]; variable only   */
    const int32_t *kv_pos;          /* device [B*Hkv][L_max]; variable only        */
    int32_t topk;                   /* >= 0: blocks; < 0: use budget_tokens        */
    int32_t budget_tokens;
    int32_t sink, window;
    int32_t keep_current_block;
    int32_t local_start;            /* variable only                               */
    int32_t pos_limit;              /* variable only                               */
} bsa_sel_params;

/* Blocks per segment the summaries buffer holds: ceil(L_max / S) for fixed
 * blocks, n_blocks for variable ones. */
BSA_API int32_t bsa_summary_blocks(const bsa_kv_desc *desc, const bsa_sel_params *sel);

/* Bytes of the summaries buffer: segments x blocks x (D fp32 for the centroid
 * kinds | D (min, max) pairs for MINMAX, in the cache dtype (bf16 for an FP8
 * cache): element 2i is the block's minimum of dimension i, element 2i + 1 its
 * maximum, so that one byte permute picks and widens the bound a query's sign
 * selects). */
BSA_API size_t bsa_summary_bytes(const bsa_kv_desc *desc, const bsa_sel_params *sel,
                         bsa_summary_kind kind);

/* Largest selected-block list and range list a segment can need. */
BSA_API int32_t bsa_max_selected(const bsa_kv_desc *desc, const bsa_sel_params *sel);
BSA_API int32_t bsa_max_ranges(const bsa_kv_desc *desc, const bsa_sel_params *sel);

/* Kernels one bsa_decode call launches for this geometry and tokens_hint
 * (the same values bsa_decode gets): 1 when the split-K partials merge
 * inside the decode grid (one thread-block cluster per segment, or a single
 * split), 2 when the merge kernel follows.  bsa_decode_step launches as many
 * when it runs fused (bf16 K/V, D 64 or 128, G <= 8), one more otherwise.
 * Reads the current device; a negative bsa_status on invalid arguments. */
BSA_API int32_t bsa_decode_kernels(const bsa_kv_desc *desc, const bsa_sel_params *sel,
                                   int32_t tokens_hint);

/* Workspace bytes for `op`.  n_queries: query rows per call for
 * BSA_OP_PREFILL (ignored otherwise); tokens_hint: for BSA_OP_DECODE, an
 * upper bound on the tokens any segment's ranges cover (sizes the split-K
 * grid; bsa_decode must get the same value).  0 on invalid arguments. */
BSA_API size_t bsa_workspace_size(const bsa_kv_desc *desc, const bsa_sel_params *sel, int op,
                          int32_t n_queries, int32_t tokens_hint);

/* Builds the summaries of blocks [first_block, first_block + n_blocks) of
 * every segment ("Module 14", §14.3; "Semantic blocks...", first section;
 * "Sparse attention in hybrid LLMs", "Which parts of the context each layer
 * reads").  K: device cache.  summaries: device buffer of
 * bsa_summary_bytes().  Fixed blocks must lie inside L_max; the centroid of
 * an empty variable block is zero.  Arithmetic: fp32 sums in row order,
 * then a correctly rounded division by the row count; the normalised kind
 * divides each key by its fp32 norm (fma chain over the dimensions, then a
 * correctly rounded square root) first and the mean by its norm after. */
BSA_API bsa_status bsa_build_summaries(const bsa_kv_desc *desc, const void *K,
                               const bsa_sel_params *sel, bsa_summary_kind kind,
                               int32_t first_block, int32_t n_blocks, void *summaries,
                               bsa_stream_t stream);

/* Scores every candidate block of every segment against the group's queries
 * and selects (rules above).  q: device fp32 [B][Hq][D].  cur_len: device
 * int32 [B], tokens in each sequence's cache.  Outputs, all device:
 *   sel_blocks [B*Hkv][max_selected]  selected block ids ascending
 *   sel_count  [B*Hkv]
 *   ranges     [B*Hkv][max_ranges][2] disjoint ascending token ranges that
 *                                     cover forced set and selected blocks
 *   n_ranges   [B*Hkv]
 * max_selected / max_ranges must be at least bsa_max_selected() /
 * bsa_max_ranges().  Score arithmetic (fixed, so that selections can be
 * compared bit for bit): per query head h an fp32 fma chain over
 * i = 0..D-1 of q_h[i] * x[i], x = the centroid, or for MINMAX
 * x[i] = q_h[i] >= 0 ? max[i] : min[i] (the larger of q*min and q*max);
 * head scores summed in head order. */
BSA_API bsa_status bsa_select(const bsa_kv_desc *desc, const float *q, const void *summaries,
                      bsa_summary_kind kind, const bsa_sel_params *sel, const int32_t *cur_len,
                      int32_t max_selected, int32_t *sel_blocks, int32_t *sel_count,
                      int32_t max_ranges, int32_t *ranges, int32_t *n_ranges,
                      void *ws, size_t ws_bytes, bsa_stream_t stream);

/* Exact softmax attention of every query head over its segment's ranges
 * (Module 14, Exercise 14.1, restricted to the selected tokens):
 *   out[b][h] = sum_j softmax_j(scale * q[b][h] . K[j]) V[j],
 *   lse[b][h] = log sum_j exp(scale * q[b][h] . K[j])      (natural log)
 * over the rows of ranges[s][0..n_ranges[s]), s = b*Hkv + h/G (ranges must
 * be 8-byte aligned; slots past n_ranges[s] may hold anything).  The last
 * range of each segment is extended to end at cur_len[b] when that is
 * larger: between selection refreshes the window keeps growing ("Sparse
 * attention in hybrid LLMs", refresh every 32 steps).  Rows are clamped to
 * [0, L_max).  q: device fp32 [B][Hq][D]; out: device fp32 [B][Hq][D];
 * lse: device fp32 [B][Hq] (may be NULL).  A segment with no rows gives
 * out = 0, lse = -inf.  tokens_hint: as for bsa_workspace_size(); any actual
 * count is handled, the hint only sizes the grid.  fp32 accumulation over
 * bf16 or fp32 K/V. */
BSA_API bsa_status bsa_decode(const bsa_kv_desc *desc, const float *q, const void *K, const void *V,
                      const int32_t *ranges, const int32_t *n_ranges, int32_t max_ranges,
                      const int32_t *cur_len, int32_t tokens_hint, float scale,
                      float *out, float *lse, void *ws, size_t ws_bytes, bsa_stream_t stream);

/* bsa_decode without a caller workspace.  The source pages have no
 * counterpart: this is a deployment convenience, not part of the method.
 *
 * For callers that cannot allocate device memory for a workspace -- code
 * embedded in an application that owns every device allocation and forbids
 * new ones once it is running (fixed budgets, pre-planned pools), or code
 * that cannot afford cudaMalloc's implicit synchronisation.  It computes
 * exactly what bsa_decode computes, with the same arguments minus ws and
 * ws_bytes, using a 4 MiB scratch array built into the library (a
 * file-scope device array: every GPU that loads the library holds it until
 * the process exits).  It allocates nothing.
 *  - The first call in each CUDA context (per device, and again after a
 *    device reset) looks up the array's device address with
 *    cudaGetSymbolAddress, with that device current, and caches it under the
 *    context's unique id; make that first call before any stream capture.
 *  - Every call shares the one array and zeroes its status word and counters
 *    first, on `stream`, after its arguments have been checked (a rejected
 *    call touches nothing).  Calls that may overlap on the GPU (other
 *    streams, other host threads) race on it and give wrong results:
 *    serialise them.
 *  - The status word of a call (a timed-out wait) stays readable until the
 *    next call zeroes it: bsa_workspace_status(NULL, 0, ...).
 *  - A problem that needs more scratch than 4 MiB (what bsa_workspace_size
 *    reports for BSA_OP_DECODE with these sizes and the selection parameters
 *    whose bsa_max_ranges() is max_ranges) is rejected with BSA_ERR_WORKSPACE
 *    before anything is launched. */
BSA_API bsa_status bsa_decode_noalloc(const bsa_kv_desc *desc, const float *q, const void *K,
                                      const void *V, const int32_t *ranges,
                                      const int32_t *n_ranges, int32_t max_ranges,
                                      const int32_t *cur_len, int32_t tokens_hint, float scale,
                                      float *out, float *lse, bsa_stream_t stream);

/* One decode step's cache bookkeeping: writes k_new, v_new (device,
 * [B][Hkv][D] in the cache dtype) at row cur_len[b] of every segment, and
 * when that row completes a fixed block, builds that block's summary with the
 * same arithmetic as bsa_build_summaries (summaries may be NULL to skip);
 * then increments cur_len[b].  Sequences whose cache is full (cur_len[b] ==
 * L_max) are left unchanged. */
BSA_API bsa_status bsa_append_kv(const bsa_kv_desc *desc, void *K, void *V, const void *k_new,
                         const void *v_new, int32_t *cur_len, const bsa_sel_params *sel,
                         bsa_summary_kind kind, void *summaries, bsa_stream_t stream);

/* One whole decode step after the selection: exactly bsa_append_kv(desc, K,
 * V, k_new, v_new, cur_len, sel, kind, summaries) followed by bsa_decode(desc,
 * q, K, V, ranges, n_ranges, max_ranges, cur_len, tokens_hint, scale, out,
 * lse, ws, ws_bytes), with the arguments and the results of those two calls
 * ("Sparse attention in hybrid LLMs": between selection refreshes a step
 * appends its token and attends over the kept pages plus the grown window).
 * On the tensor-core path (bf16 cache, D in {64, 128}, Hq/Hkv <= 8, rows
 * contiguous, k_new and v_new 16-byte aligned) both run in one launch: the
 * CTA whose tile holds row cur_len[b] writes that row before loading the
 * tile, builds the summary of a fixed block the row completes (CENTROID or
 * MINMAX summaries), and the last CTA of each sequence increments cur_len.
 * Elsewhere (and for CENTROID_NORM summaries of fixed blocks) it issues the
 * two launches.  A step that refreshes the selection must append before
 * selecting: use bsa_append_kv, bsa_select, bsa_decode there.  Workspace:
 * bsa_workspace_size(BSA_OP_DECODE). */
BSA_API bsa_status bsa_decode_step(const bsa_kv_desc *desc, const float *q, void *K, void *V,
                                   const void *k_new, const void *v_new, int32_t *cur_len,
                                   const bsa_sel_params *sel, bsa_summary_kind kind,
                                   void *summaries, const int32_t *ranges,
                                   const int32_t *n_ranges, int32_t max_ranges,
                                   int32_t tokens_hint, float scale, float *out, float *lse,
                                   void *ws, size_t ws_bytes, bsa_stream_t stream);

/* Block-grouped prefill for variable (semantic) blocks, batch 1.
 * Query row i sits at position q_pos0 + i and reads
 *   (a) the positions [pos_limit, q_pos0 + i] densely and causally from the
 *       position-ordered keys and values K_pos / V_pos (pos_desc geometry),
 *       whose row r holds position pos_base + r -- for a chunk past the dense
 *       limit (pos_limit = q_pos0) just the chunk's own rows, pos_base =
 *       q_pos0; it must cover [pos_limit, q_pos0 + Tq), and
 *   (b) the visible prefixes (kv_pos < pos_limit) of the blocks its group
 *       selects from the block-ordered store K / V (desc geometry) with the
 *       variable-block rules above (budget_tokens, CENTROID_NORM summaries).
 * Selection is per (query row, KV head); the queries that selected one block
 * are gathered and contracted against it together on the tensor cores, and
 * the partial results are merged per query by log-sum-exp.
 * Q: device bf16 [Tq][Hq][D]; out: device fp32 [Tq][Hq][D]; lse: device fp32
 * [Tq][Hq] (may be NULL).  K, V, K_pos, V_pos, Q, out and the CENTROID_NORM
 * summaries must be 16-byte aligned (BSA_ERR_ARG otherwise).  pos_limit = 0
 * makes the call dense causal attention over [0, q_pos0 + i]. */
BSA_API bsa_status bsa_prefill_grouped(const bsa_kv_desc *desc, const void *K, const void *V,
                               const bsa_sel_params *sel, const void *summaries,
                               const bsa_kv_desc *pos_desc, const void *K_pos, const void *V_pos,
                               int32_t pos_base, const void *Q, int32_t q_pos0, int32_t Tq,
                               float scale, float *out, float *lse, void *ws, size_t ws_bytes,
                               bsa_stream_t stream);

/* The semantic index ("Semantic blocks for sparse attention", first section:
 * similar keys from anywhere in the request form one block, stored together
 * and scored through its centre): spherical k-means over rows [0, L) of each
 * segment of K (desc geometry, bf16 or fp32, D 64 or 128), then the
 * block-ordered store.  Arithmetic, fixed so that labels compare bit for bit:
 *   u_r = k_r / ||k_r|| (fp32; ||.|| = sqrt of an fma chain over i; a zero
 *         key stays zero); c_j = u_{init[j]} to start;
 *   `iters` assignment rounds: label_r = argmax_j of the fp32 fma chain over
 *         i of u_r[i] * c_j[i], the lowest j on equal values; between rounds
 *         c_j = m / ||m||, m = (u summed over cluster j in position order) /
 *         n_j (the CENTROID_NORM arithmetic); an empty cluster keeps c_j.
 * Outputs (device, [B*Hkv] segments each): centres [k][D] fp32 (those of the
 * last assignment), labels [L], offsets [k+1] (cluster j is rows
 * offsets[j] .. offsets[j+1] of the block-ordered store) and order [L] (the
 * original position of block-ordered row i: clusters in index order,
 * positions ascending), which is the kv_pos a grouped prefill takes and the
 * row list bsa_gather_rows takes.  init [B*Hkv][k]: starting rows (entries
 * outside [0, L) are clamped).  1 <= k <= min(L, 1024) and k * D <= 49,152;
 * the workspace (bsa_index_workspace_size bytes, 16-byte aligned; it holds
 * every key's unit vector in fp32, L * D * 4 bytes per segment, computed once
 * per call) needs no zeroing.  BSA_ERR_ARG / BSA_ERR_UNSUPPORTED / BSA_ERR_WORKSPACE before any
 * launch. */
BSA_API size_t bsa_index_workspace_size(const bsa_kv_desc *desc, int64_t L, int32_t n_clusters);
BSA_API bsa_status bsa_build_semantic_index(const bsa_kv_desc *desc, const void *K, int64_t L,
                                            int32_t n_clusters, int32_t iters, const int32_t *init,
                                            float *centres, int32_t *labels, int32_t *offsets,
                                            int32_t *order, void *ws, size_t ws_bytes,
                                            bsa_stream_t stream);

/* Row gather between two caches of the same B, Hkv, D and dtype (strides may
 * differ): for every segment, rows dst_row0 + i of K_out / V_out take rows
 * rows[seg][i] of K / V, i < n (rows: device int32 [B*Hkv][n]; an entry
 * outside [0, src L_max) leaves its destination row as it was; rows past the
 * destination's L_max are BSA_ERR_ARG).  Builds the
 * block-ordered store from `order`.  All four caches 16-byte aligned. */
BSA_API bsa_status bsa_gather_rows(const bsa_kv_desc *src, const void *K, const void *V,
                                   const bsa_kv_desc *dst, void *K_out, void *V_out,
                                   const int32_t *rows, int64_t n, int64_t dst_row0,
                                   bsa_stream_t stream);

/* Reads the sticky device-side status word of a workspace (see the
 * conventions above) once the work enqueued on `stream` so far has finished:
 * the call waits for the stream, so it must not be made while the stream is
 * being captured into a CUDA graph (it then returns BSA_ERR_CUDA).
 * ws == NULL reads the scratch built into the library for
 * bsa_decode_noalloc on the current device (ws_bytes is then ignored).
 * When clear != 0 the word is reset to zero afterwards.  bits (host, may be
 * NULL) receives the raw word.  Returns BSA_OK when no bit is set,
 * BSA_ERR_TIMEOUT when a wait bit (0, 1 or 3) is set, otherwise
 * BSA_ERR_CAPACITY; BSA_ERR_WORKSPACE for a workspace smaller than 4 bytes or
 * misaligned; BSA_ERR_CUDA when the stream or the copy fails. */
BSA_API bsa_status bsa_workspace_status(const void *ws, size_t ws_bytes, int32_t clear,
                                        uint32_t *bits, bsa_stream_t stream);

/* Test hook, not part of the method: the next decode launch of this process
 * (bsa_decode, bsa_decode_step or bsa_decode_noalloc on the tensor-core path)
 * makes one warp of its first CTA wait, before any tile copy is issued, on a
 * barrier that nothing completes, giving up after limit_us microseconds
 * (1 <= limit_us <= 100,000; 0 disarms).  The wait ends by its limit, sets
 * the timeout bit of the status word as a real stalled copy would, and the
 * launch then runs to completion with correct results, so a caller can check
 * that a wait which gives up is reported (bsa_workspace_status returns
 * BSA_ERR_TIMEOUT) without stalling anything.  BSA_ERR_ARG for a limit out of
 * range. */
BSA_API bsa_status bsa_test_arm_wait_limit(int32_t limit_us);

/* Static text for a status code. */
BSA_API const char *bsa_status_string(bsa_status status);

/* Library ABI version (major * 100 + minor). */
BSA_API int32_t bsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H */
