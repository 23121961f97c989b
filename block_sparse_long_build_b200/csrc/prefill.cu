// A6/A7: block-grouped prefill (placeholder until the tensor-core kernels land).
#include "common.cuh"

namespace bsa {

size_t prefill_ws_bytes(const bsa_kv_desc *, const bsa_sel_params *, int) { return 256; }

bsa_status launch_prefill(const bsa_kv_desc *, const void *, const void *, const bsa_sel_params *,
                          const void *, const bsa_kv_desc *, const void *, const void *,
                          const void *, int, int, float, float *, float *, void *, size_t,
                          cudaStream_t) {
    return BSA_ERR_UNSUPPORTED;
}

}  // namespace bsa
