// pkm_capi_bwd.cu -- backward entry points (placeholder).
#include "kernels.h"

extern "C" {

size_t pkm_backward_workspace_size(const pkm_bwd_args*) { return 0; }
pkm_status pkm_backward(const pkm_bwd_args*, pkm_stream_t) { return PKM_ERR_UNSUPPORTED; }
size_t embbag_backward_workspace_size(int64_t, int32_t, int32_t, int64_t) { return 0; }
pkm_status embbag_backward(const void*, const int32_t*, const float*, int64_t, int32_t, int32_t,
                           pkm_dtype, const void*, int64_t, float*, int32_t*, float*, int64_t*,
                           int64_t, float*, void*, size_t, pkm_stream_t) {
  return PKM_ERR_UNSUPPORTED;
}

}
