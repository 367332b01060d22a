// Shared device-side definitions of the FiX attention library.
//
// Chunking.  Every sequence is cut into chunks of FIX_CHUNK = 128 tokens that
// start at the sequence's first token (the last chunk may be short).  The
// gate prefix sums are kept chunk-local: L_t[c] = sum of g over the chunk's
// rows up to and including t, plus one total per chunk, tot_j[c].  For t in
// chunk i and s in chunk j <= i the decay exponent is
//     G_t - G_s = (L_t - L_s) + sum_{j <= j' < i} tot_j'
// which never subtracts two large prefix sums (better fp32 accuracy than one
// global cumsum) and lets the prefix pass run with no carry between chunks.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#define FIX_CHUNK 128
// CTAs per chunk in the backward preprocess (FIX_CHUNK / kPreSplit rows each).
constexpr int kPreSplit = 2;
// CTAs per chunk in the preprocess's second pass (its items are smaller, so
// more CTAs keep enough loads in flight)
constexpr int kPreOpsSplit = 8;
// Largest schedule piece one upload launch carries in its parameter block
// (31 KB of the 32 KB that kernel parameters may take).
constexpr int kBlobMaxWords = 7936;

// e^x for the 16-bit tensor-core operands (pre-decayed values and gradients)
// that the prefix pass and the backward preprocess produce: the MUFU 2^x
// approximation of x log2(e) (relative error about 2^-22, far below their 8-
// or 11-bit significands and the ~16 bits of a hi/lo pair; results below
// fp32's normal range become 0, which every 16-bit store does anyway).  The
// exact CUDA-core kernels keep expf.
__device__ __forceinline__ float exp_op(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x * 1.4426950408889634f));
  return y;
}
// Largest half-range of a chunk's prefix sums that the in-chunk split
// exp(L_t - rho) * exp(rho - L_s) keeps inside float range (e^80 ~ 5.5e34),
// and the largest |rho| for which the forward's column factor exp(rho) stays
// a normal float.  A channel outside either bound is "out of range": its
// rho is 0, its hr is stored as FIX_HR_BAD, its Vm is 0, and its diagonal
// block is summed exactly in fp32.
#define FIX_HR_MAX 80.0f
#define FIX_RHO_MAX 80.0f
#define FIX_HR_BAD 1e30f
// Pre-decayed values Vt (key blocks before the query chunk) are stored as
// fp16 scaled by 2^-e per (chunk, kv head, channel), e = vt_exponent(lvt)
// from lvt = log2 of the column's largest |Vt|, so that every stored value
// is at most 2^15 in magnitude (e = 0 whenever that already holds).
__host__ __device__ __forceinline__ float vt_exponent(float lvt) {
  return lvt > 15.0f ? ceilf(lvt - 15.0f) : 0.0f;
}
// Largest |v| for which the fp16 operand path is used (fp16 max is 65504;
// every scaled value on that path is <= |v| when g <= 0).
#define FIX_F16_VMAX 30000.0f

namespace fix {

// One chunk of the schedule (built on the host from the sequence lengths):
// first token (index into the packed token stream), number of valid rows,
// chunk index within its sequence and the sequence's chunk count.  Chunks of
// a sequence are consecutive in the table, so the sequence's first chunk has
// id (this id - j).
struct Chunk {
  int tok0;
  int len;
  int j;
  int nch;
};

// One CTA's share of a key chunk's backward work: the key chunk, the kind of
// query tiles (diag = 1: those of the chunk itself, else those of later
// chunks), the index p of its run of (at most `tiles_per_part`) 64-row tiles
// of that kind, and the slot of its fp32 partial sums in the partial buffer.
struct Part {
  int ci;
  int p;
  int slot;
  int diag;
};

// 64-row halves of chunk j of a sequence of L tokens.
__device__ __host__ inline int fix_halves(int L, int j) {
  const int len = L - j * FIX_CHUNK < FIX_CHUNK ? L - j * FIX_CHUNK : FIX_CHUNK;
  return (len + 63) / 64;
}

// A schedule table carried in a kernel's parameter block.
template <int NW>
struct Blob {
  uint32_t w[NW];
};

struct Dims {
  int N;          // total tokens
  int B, T;       // dense batch / length (T = N when packed)
  int Hq, Hkv;    // heads
  int Dk, Dv;     // head dims
  int grp;        // Hq / Hkv
  int nseq;       // sequences (B, or packed count)
  int nchunks;    // chunks over all sequences
  float scale;    // logit scale
  float eps;      // RMSNorm epsilon
  int no_norm;    // FIX_FLAG_NO_NORM: y = o / l, no RMSNorm
  int scalar_gate;  // FIX_FLAG_SCALAR_GATE: g is [N, Hkv]
};

__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }

// The output gate's activation, swish(z) = z sigmoid(z), and its derivative
// sigmoid(z) (1 + z (1 - sigmoid(z))).
__device__ __forceinline__ float swish(float z) { return z / (1.0f + __expf(-z)); }
__device__ __forceinline__ float swish_grad(float z) {
  const float sg = 1.0f / (1.0f + __expf(-z));
  return sg * (1.0f + z * (1.0f - sg));
}
__device__ __forceinline__ __nv_bfloat16 f2bf(float x) { return __float2bfloat16_rn(x); }

// 4 consecutive values from an 8-byte (bf16) or 16-byte (fp32) aligned
// address into floats; zeros for a null address.
__device__ __forceinline__ void ld4b(const __nv_bfloat16* p, float* x) {
  if (!p) {
    x[0] = x[1] = x[2] = x[3] = 0.f;
    return;
  }
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  x[0] = __uint_as_float(u.x << 16);
  x[1] = __uint_as_float(u.x & 0xFFFF0000u);
  x[2] = __uint_as_float(u.y << 16);
  x[3] = __uint_as_float(u.y & 0xFFFF0000u);
}
__device__ __forceinline__ void ld4f(const float* p, float* x) {
  if (!p) {
    x[0] = x[1] = x[2] = x[3] = 0.f;
    return;
  }
  const float4 u = *reinterpret_cast<const float4*>(p);
  x[0] = u.x;
  x[1] = u.y;
  x[2] = u.z;
  x[3] = u.w;
}
// 4 floats to 4 consecutive bf16 (round to nearest) at an 8-byte aligned address.
__device__ __forceinline__ void st4b(__nv_bfloat16* p, const float* x) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]), b = __floats2bfloat162_rn(x[2], x[3]);
  *reinterpret_cast<uint2*>(p) =
      make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
}

// Asynchronous copy of N (4, 8 or 16) bytes from global to shared memory,
// cached in L1; with valid false nothing is read and the N bytes are zeroed.
template <int N>
__device__ __forceinline__ void cp_async(void* sdst, const void* gsrc, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(sdst));
  asm volatile("cp.async.ca.shared.global [%0], [%1], %2, %3;" ::"r"(d), "l"(gsrc), "n"(N),
               "r"(valid ? N : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Waits until at most N of this thread's committed copy groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Status word at the head of the workspace.
enum { FIX_DEV_OK = 0, FIX_DEV_TIMEOUT = 10 };

}  // namespace fix
