// a7: backward of the hybrid block-sparse attention (placeholder until the
// tensor-core backward lands).
#include <cuda_runtime.h>

#include "common.cuh"

extern "C" size_t pbsa_attn_bwd_workspace(const pbsa_dims* d, int Tq, int NB, int Amax) {
  if (d == nullptr || Tq < 1 || NB < 1 || Amax < 1) return 0;
  return 256;
}

extern "C" int pbsa_attn_bwd(const pbsa_dims* d, const void*, int, int, const void*, const void*,
                             int, const int32_t*, const int32_t*, const int32_t*, const int32_t*,
                             int, int, const void*, const float*, const void*, float*, float*,
                             float*, void*, size_t, void*) {
  int rc = pbsa::common_dims_check(d);
  if (rc) return rc;
  pbsa::set_error("attn_bwd: not built yet");
  return PBSA_ERR_ARG;
}
