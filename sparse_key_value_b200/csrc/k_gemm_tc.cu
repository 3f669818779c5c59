// k_gemm_tc.cu -- tensor-core GEMM for the Memory+ block (placeholder: the
// SIMT GEMM in k_gemm.cu serves every shape until this kernel lands).
#include "kernels.h"

namespace pkm {

bool gemm_tc_supported(int64_t, int, int) { return false; }
cudaError_t launch_gemm_tc(const void*, const void*, int64_t, int, int, int, void*, int32_t*,
                           cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace pkm
