// Tensor-core (tcgen05) FiX backward: not yet available; the backward runs on
// the exact CUDA-core kernels.
#include "fix_internal.h"

namespace fix {

bool tc_bwd_supported(const Dims&) { return false; }
int tc_bwd_kernel_count(const Dims&) { return 0; }
fix_status tc_bwd(const fix_attn_problem*, const Dims&, const Chunk*, const void*, const void*, const void*,
                  const uint16_t*, const float*, const float*, const float*, const float*,
                  const float*, void*, void*, void*, float*, int*, cudaStream_t) {
  return FIX_ERR_CUDA;
}

}  // namespace fix
