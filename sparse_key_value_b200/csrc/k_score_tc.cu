// k_score_tc.cu -- sub-key scoring on the tensor cores (tcgen05): placeholder
// until the kernel lands; the SIMT path serves every shape meanwhile.
#include "kernels.h"

namespace pkm {

bool score_tc_supported(pkm_dtype, int, int, int) { return false; }
int score_tc_splits(int64_t, int, int) { return 1; }
cudaError_t launch_score_topk_tc(const void*, const void*, int64_t, int, int, int, int, int,
                                 const float*, const float*, float*, int32_t*, int32_t*,
                                 cudaStream_t) {
  return cudaErrorNotSupported;
}

bool gemm_tc_supported(int64_t, int, int) { return false; }
cudaError_t launch_gemm_tc(const void*, const void*, int64_t, int, int, int, void*, int32_t*,
                           cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace pkm
