// Test hooks, compiled only into the test build of the library
// (libfixattn_test.so, -DFIX_TEST_HOOKS); the product library has none.
//
// fix_attn_test_stall_forward(1) makes every following tensor-core forward
// launch run "stalled": its producer warp issues no loads, so nothing is ever
// in flight, and every bounded wait gives up after 1 ms instead of 1 s.  The
// kernel must then take its abort path -- record FIX_ERR_DEVICE_TIMEOUT in the
// status word, leave every role, release TMEM -- and the next ordinary call
// must succeed.  This exercises the device-side failure detection without a
// GPU fault or a hang.
//
// fix_attn_test_exp2_poly(x, out, n, stream) and its packed-pair form
// fix_attn_test_exp2_poly_x2 evaluate the forward's polynomial 2^x on n
// device floats, so that a test can hold them to their error bound against
// exact powers of two.
#ifdef FIX_TEST_HOOKS
#include <cuda_runtime.h>

#include <atomic>

#include "fix_internal.h"
#include "fix_sm100.cuh"

namespace fix {
static std::atomic<int> g_stall{0};
int test_stall_forward() { return g_stall.load(); }
}  // namespace fix

extern "C" void fix_attn_test_stall_forward(int on) { fix::g_stall.store(on ? 1 : 0); }

// The last CUDA error a launch in the library reported (cudaError_t), for
// diagnosing FIX_ERR_CUDA in tests.
namespace fix {
extern int g_test_last_cuda_error;
}
extern "C" int fix_attn_test_last_cuda_error(void) { return fix::g_test_last_cuda_error; }

namespace {
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = fix::sm100::exp2_poly3(x[i]);
}

// The packed-pair form: elements 2i and 2i + 1 as one f32x2 pair.
__global__ void exp2_poly_x2_kernel(const float* __restrict__ x, float* __restrict__ out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (2 * i + 1 < n) {
    float a, b;
    fix::sm100::f2_unpack(fix::sm100::exp2_poly3_x2(fix::sm100::f2_pack(x[2 * i], x[2 * i + 1])), a, b);
    out[2 * i] = a;
    out[2 * i + 1] = b;
  } else if (2 * i < n) {
    out[2 * i] = fix::sm100::exp2_poly3(x[2 * i]);
  }
}
}  // namespace

extern "C" int fix_attn_test_exp2_poly(const float* x, float* out, int n, void* stream) {
  if (n <= 0) return 0;
  exp2_poly_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, out, n);
  return cudaGetLastError() == cudaSuccess ? 0 : 1;
}

extern "C" int fix_attn_test_exp2_poly_x2(const float* x, float* out, int n, void* stream) {
  if (n <= 0) return 0;
  const int pairs = (n + 1) / 2;
  exp2_poly_x2_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, out, n);
  return cudaGetLastError() == cudaSuccess ? 0 : 1;
}
#endif
