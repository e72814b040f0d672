// tc_bwd.cu -- tcgen05 tensor-core recompute backward (bf16).
#include <cuda_runtime.h>

#include "kernels.h"

namespace cpattn {

bool tc_bwd_supported(const AttnShape& sh) {
  (void)sh;
  return false;
}

int launch_tc_bwd(const AttnShape& sh, const void* q, const void* k, const void* v,
                  const void* o, const float* lse, const void* dout, void* dq, void* dk,
                  void* dv, float* ws_dq, float* ws_delta, unsigned* err, cudaStream_t stream) {
  (void)sh; (void)q; (void)k; (void)v; (void)o; (void)lse; (void)dout; (void)dq; (void)dk;
  (void)dv; (void)ws_dq; (void)ws_delta; (void)err; (void)stream;
  return -1;
}

}  // namespace cpattn
