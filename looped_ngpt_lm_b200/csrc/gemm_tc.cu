#include "gemm_tc.cuh"

namespace dory {

cudaError_t launch_gemm_tc(int, int, int, const bf16*, int, const bf16*, float*, int, size_t, int*, int* S,
                           size_t* ps, cudaStream_t) {
  *S = 1;
  *ps = 0;
  return cudaErrorNotSupported;
}

}  // namespace dory
