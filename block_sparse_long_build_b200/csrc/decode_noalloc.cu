// bsa_decode_noalloc: the split-K decode with the library's own scratch.
//
// Some callers cannot hand the library a workspace: code embedded in a host
// application that owns every device allocation and forbids new ones after
// start-up (fixed memory budgets, pre-planned pools), or paths where the
// implicit synchronisation of cudaMalloc is not acceptable.  For them this
// entry point uses a buffer that lives in the library image itself: a
// file-scope device array, created when the library's module is loaded on a
// GPU and held until the process exits.  Nothing here allocates device
// memory.
//
// Host code cannot use the array's name as a device address, so the address
// is looked up with cudaGetSymbolAddress, with the device current, on the
// first call made in a CUDA context, and cached under that context's unique
// id: a device reset or another context on the same device gets a fresh
// lookup instead of a stale pointer.
#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"

namespace bsa {

int decode_nsplit(const bsa_kv_desc *, int, int);
size_t decode_scratch_bytes(const bsa_kv_desc *, int);
size_t ws_counters_bytes(const bsa_kv_desc *);
bsa_status decode_check_args(const bsa_kv_desc *, const float *, const void *, const void *,
                             const int32_t *, const int32_t *, int32_t, const int32_t *, int32_t,
                             float, const float *);

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB

// The scratch: status word, split counters and split partials of one call.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Unique id of the CUDA context current on this thread (0 if none is
// current yet or it cannot be read).
static unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
        cudaGetLastError();
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of g_noalloc_scratch in the current context, or nullptr.
void *noalloc_scratch_on_current_context() {
    static std::mutex mu;
    static std::vector<std::pair<unsigned long long, void *>> cache;
    std::lock_guard<std::mutex> lock(mu);
    unsigned long long id = current_context_id();
    if (id)
        for (auto &e : cache)
            if (e.first == id) return e.second;
    // the lookup binds the device's primary context if none is current yet
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return nullptr;
    }
    if (!id) id = current_context_id();
    if (id) cache.emplace_back(id, p);
    return p;
}

}  // namespace bsa

extern "C" bsa_status bsa_decode_noalloc(const bsa_kv_desc *d, const float *q, const void *K,
                                         const void *V, const int32_t *ranges,
                                         const int32_t *n_ranges, int32_t max_ranges,
                                         const int32_t *cur_len, int32_t tokens_hint, float scale,
                                         float *out, float *lse, bsa_stream_t stream) {
    using namespace bsa;
    // Every check bsa_decode makes, before the shared array is touched: a
    // rejected call must not clear the counters of a call in flight.
    const bsa_status chk = decode_check_args(d, q, K, V, ranges, n_ranges, max_ranges, cur_len,
                                             tokens_hint, scale, out);
    if (chk != BSA_OK) return chk;
    const size_t zero_bytes = ws_counters_bytes(d);
    const size_t need =
        zero_bytes + decode_scratch_bytes(d, decode_nsplit(d, std::max(tokens_hint, 1), max_ranges));
    if (need > kNoAllocScratchBytes) return BSA_ERR_WORKSPACE;
    void *scratch = noalloc_scratch_on_current_context();
    if (!scratch) return BSA_ERR_CUDA;
    // The array keeps the previous call's contents: zero the status word and
    // the counters, which the split-K merge needs to start at zero.
    if (cudaMemsetAsync(scratch, 0, zero_bytes, (cudaStream_t)stream) != cudaSuccess)
        return BSA_ERR_CUDA;
    return bsa_decode(d, q, K, V, ranges, n_ranges, max_ranges, cur_len, tokens_hint, scale, out,
                      lse, scratch, kNoAllocScratchBytes, stream);
}
