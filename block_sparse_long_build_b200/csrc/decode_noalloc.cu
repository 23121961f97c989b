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
// is looked up once per device with cudaGetSymbolAddress, with that device
// current, on the first call made on it, and cached.
#include <mutex>

#include "common.cuh"

namespace bsa {

int decode_nsplit(const bsa_kv_desc *, int, int);
size_t decode_scratch_bytes(const bsa_kv_desc *, int);

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB

// The scratch: status word, split counters and split partials of one call.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch on the current device, or nullptr.
static void *noalloc_scratch_on_current_device() {
    static std::mutex mu;
    static void *addr[kMaxDevices] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return nullptr;
        }
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace bsa

extern "C" bsa_status bsa_decode_noalloc(const bsa_kv_desc *d, const float *q, const void *K,
                                         const void *V, const int32_t *ranges,
                                         const int32_t *n_ranges, int32_t max_ranges,
                                         const int32_t *cur_len, int32_t tokens_hint, float scale,
                                         float *out, float *lse, bsa_stream_t stream) {
    using namespace bsa;
    // bsa_workspace_size() is 0 for an invalid descriptor; the size this call
    // needs is the one bsa_decode() will check for the same arguments.
    if (bsa_workspace_size(d, nullptr, BSA_OP_DECODE, 0, tokens_hint) == 0) return BSA_ERR_ARG;
    if (max_ranges < 1 || max_ranges > 4096 || tokens_hint < 0) return BSA_ERR_ARG;
    const size_t zero_bytes = align_up((size_t)(1 + 2 * d->B * d->Hkv) * 4, 256);
    const size_t need =
        zero_bytes + decode_scratch_bytes(d, decode_nsplit(d, std::max(tokens_hint, 1), max_ranges));
    if (need > kNoAllocScratchBytes) return BSA_ERR_WORKSPACE;
    void *scratch = noalloc_scratch_on_current_device();
    if (!scratch) return BSA_ERR_CUDA;
    // The array keeps the previous call's contents: zero the status word and
    // the counters, which the split-K merge needs to start at zero.
    if (cudaMemsetAsync(scratch, 0, zero_bytes, (cudaStream_t)stream) != cudaSuccess)
        return BSA_ERR_CUDA;
    return bsa_decode(d, q, K, V, ranges, n_ranges, max_ranges, cur_len, tokens_hint, scale, out,
                      lse, scratch, kNoAllocScratchBytes, stream);
}
