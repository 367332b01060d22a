// Tensor-core (tcgen05) FiX kernels: not yet available; every problem runs on
// the exact CUDA-core kernels.
#include "fix_internal.h"

namespace fix {

bool tc_fwd_supported(const Dims&) { return false; }
fix_status tc_fwd(const Dims&, const Chunk*, const void*, const void*, const __nv_bfloat16*,
                  const void*, const float*, const float*, const void*, void*, bool, float*,
                  float*, float*, int*, cudaStream_t) {
  return FIX_ERR_CUDA;
}
int tc_fwd_kernel_count(const Dims&) { return 0; }
bool tc_bwd_supported(const Dims&) { return false; }
int tc_bwd_kernel_count(const Dims&) { return 0; }
fix_status tc_bwd(const fix_attn_problem*, const Dims&, const Chunk*, const void*, const void*, const void*,
                  const __nv_bfloat16*, const float*, const float*, const float*, const float*,
                  const float*, void*, void*, void*, float*, int*, cudaStream_t) {
  return FIX_ERR_CUDA;
}

}  // namespace fix
