// Internal declarations shared by the host API and the kernel translation units.
#pragma once
#include "fix_attn.h"
#include "fix_common.cuh"

namespace fix {

constexpr int ST_ROWS = 32;  // rows per CTA of the exact (SIMT) kernels

// Validates a problem descriptor and fills the kernel-side dims (fix_api.cu).
fix_status validate_problem(const fix_attn_problem* p, Dims* d);

// Sizes of one decode call (fix_decode.cu).
struct DecodeDims {
  int B, Tmax, Hq, Hkv, Dk, Dv, grp;
  int R;        // keys per range of the split
  int nsplit;   // ranges over Tmax
  float scale, eps;
  int no_norm, scalar_gate;
};

// fix_prefix.cu
template <int NW>
__global__ void upload_kernel(const __grid_constant__ Blob<NW> b, uint32_t* dst, int nwords);
__global__ void prefix_kernel(Dims d, const Chunk* chunks, const float* g, const __nv_bfloat16* v,
                              float* L, float* Lt, uint16_t* vt, __nv_bfloat16* vm, __nv_bfloat16* vml,
                              float* tot, float* rho, float* hr, float* lvt, int* safe,
                              int* badflag, int* hmax);
// Launch shape of prefix_kernel: grid (nchunks, Hkv, prefix_slices(Dv)), 256
// threads, prefix_smem_bytes(Dv, lt) of dynamic shared memory (lt: the
// channel-major copy of L is written).
int prefix_slices(int Dv);
size_t prefix_smem_bytes(int Dv, bool lt);
__global__ void chunk_total_kernel(Dims d, const Chunk* chunks, const float* x, float* tot);
__global__ void channel_sum_kernel(const float* x, long long rows, int D, float* out);
__global__ void reverse_cumsum_kernel(Dims d, const Chunk* chunks, const float* x,
                                      const float* tot, float* out);

// fix_simt.cu
__global__ void fwd_simt_kernel(Dims d, const Chunk* chunks, const __nv_bfloat16* q,
                                const __nv_bfloat16* k, const __nv_bfloat16* v, const float* L,
                                const float* tot, const __nv_bfloat16* w,
                                const __nv_bfloat16* z, void* y, int y_f32, float* o_s,
                                float* m_s, float* rstd_s);
__global__ void bwd_pre_kernel(Dims d, const Chunk* chunks, const __nv_bfloat16* q,
                               const __nv_bfloat16* k, const __nv_bfloat16* v, const float* o_s,
                               const float* m_s, const float* rstd_s, const __nv_bfloat16* dy,
                               const __nv_bfloat16* w, const __nv_bfloat16* z,
                               __nv_bfloat16* dz, float* do_ws, float* A, float* delta,
                               float* dwpart, int* hmax_g, float* ptt);
size_t bwd_pre_smem_bytes(int grp);   // dynamic shared memory of bwd_pre_kernel
__global__ void bwd_pre_ops_kernel(Dims d, const Chunk* chunks, const float* L, const float* rho,
                                   const float* hr, const int* safe, const float* do_ws,
                                   const int* hmax_g, uint16_t* dot, __nv_bfloat16* domh,
                                   __nv_bfloat16* doml, int* dsafe);
__global__ void dw_reduce_kernel(const float* parts, int nparts, int Dv, __nv_bfloat16* dw);
__global__ void dq_simt_kernel(Dims d, const Chunk* chunks, const __nv_bfloat16* q,
                               const __nv_bfloat16* k, const __nv_bfloat16* v, const float* L,
                               const float* tot, const float* m_s, const float* do_ws,
                               const float* delta, __nv_bfloat16* dq, const int* gate);
__global__ void dkv_simt_kernel(Dims d, const Chunk* chunks, const __nv_bfloat16* q,
                                const __nv_bfloat16* k, const __nv_bfloat16* v, const float* L,
                                const float* tot, const float* m_s, const float* do_ws,
                                const float* delta, const float* A, __nv_bfloat16* dk,
                                __nv_bfloat16* dv, float* dG, const int* gate);

// Tensor-core (tcgen05) kernels.
// Raises a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device.  The attribute is set once per (kernel, device) and size
// increase, so the launch path makes no further runtime calls for it (which
// keeps the calls cheap and lets a stream capture record the launches).
bool set_smem_limit(const void* func, int bytes);
// FIX_OK if no launch error is pending, else FIX_ERR_CUDA (test builds
// record the error for fix_attn_test_last_cuda_error).
fix_status launch_status();
bool tc_fwd_supported(const Dims& d);
fix_status tc_fwd(const Dims& d, const Chunk* chunks, const int* order, const void* q,
                  const void* k, const uint16_t* vt, const __nv_bfloat16* vm,
                  const __nv_bfloat16* vml, const void* v,
                  const float* L, const float* Lt, const float* tot, const float* rho, const float* hr,
                  const float* lvt, const int* safe,
                  const void* w, const void* z, void* y, bool y_f32, float* o_s, float* m_s,
                  float* rstd_s, int* status, cudaStream_t st);
int tc_fwd_kernel_count(const Dims& d);
#ifdef FIX_TEST_HOOKS
// Test builds (libfixattn_test.so) only: whether the tensor-core forward runs
// stalled (no loads issued, every wait gives up after 1 ms).
int test_stall_forward();
#endif
bool tc_bwd_supported(const Dims& d);
int tc_bwd_kernel_count(const Dims& d, long long nslots);

// Device buffers of one backward call for the tensor-core kernels.
struct TcBwdArgs {
  const Chunk* chunks;
  const int* order;
  const void* q;
  const void* k;
  const void* v;
  const uint16_t* vt;
  const __nv_bfloat16* vm;
  const float* L;
  const float* tot;
  const float* rho;
  const float* hr;
  const float* lvt;      // log2 of the largest |Vt| per (chunk, kv head, channel)
  const int* safe;
  const int* dsafe;
  const float* m_s;
  const float* do_ws;
  const uint16_t* dot;
  const __nv_bfloat16* domh;
  const __nv_bfloat16* doml;
  const float* A;
  const float* ptt;      // P_tt per (token, q head), from the preprocess
  const float* delta;    // without the norm: sum_c do_t o_t per (token, q head); else NULL
  const int* badflag;
  const Part* parts;
  const int2* cpart;
  int tiles_per_part;
  long long nparts;
  long long nslots;
  float* partial;
  void* dq;
  void* dk;
  void* dv;
  float* dG;
  int* status;
};
// which = 0: dq kernel, 1: dk/dv kernel, 2: combine of the dk/dv partials
fix_status tc_bwd(const fix_attn_problem* p, const Dims& d, const TcBwdArgs& a, int which,
                  cudaStream_t st);

}  // namespace fix
