// Tensor-core SGMM (tcgen05) for long segments: not built yet.
#include "apr_internal.cuh"

namespace apr {

bool sgmm_tensor_supported(const SgmmArgs& a, int dtype) {
  (void)a;
  (void)dtype;
  return false;
}

cudaError_t launch_sgmm_tensor(const SgmmArgs& a, cudaStream_t s) {
  (void)a;
  (void)s;
  return cudaErrorNotSupported;
}

}  // namespace apr
