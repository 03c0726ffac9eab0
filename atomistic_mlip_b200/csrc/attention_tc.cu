// Tensor-core (tcgen05 / TMEM) fused attention -- not built yet; the bf16
// path runs on the SIMT kernel until this reports availability.
#include "common.cuh"

namespace e2f {

e2f_status attention_tc_available(const e2f_weights *) { return E2F_ERR_UNSUPPORTED; }

e2f_status attention_tc_impl(const void *, const void *, const void *, const float *, const e2f_csr *,
                             const e2f_weights *, float *, cudaStream_t, cudaEvent_t, cudaEvent_t) {
  return E2F_ERR_UNSUPPORTED;
}

}  // namespace e2f
