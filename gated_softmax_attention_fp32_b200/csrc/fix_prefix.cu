// Gate prefix pass, schedule upload and the reverse cumsum of dG.
//
// FiX README, "Code Structure": intra_chunk_preprocess_fwd ("Intra-chunk
// forward preprocessing") and inter_chunk_scale_v ("Inter-chunk scaling for
// V").  Here one HBM-bound pass reads g and v once per chunk of 128 tokens and
// writes
//   L_t[c]  = sum_{r in chunk, r <= t} g_r[c]         chunk-local prefix (f32)
//   tot[c]  = L_last[c]                                chunk total (f32)
//   Vt_s[c] = v_s[c] * exp(L_last[c] - L_s[c])         values pre-decayed to the
//                                                      chunk's last row (bf16)
// For g <= 0 every factor exp(L_last - L_s) is <= 1, so Vt never overflows.
// The backward reuses the same kernels for its reverse cumsum of dG.
#include "fix_common.cuh"

namespace fix {

// Copies a schedule table built on the host (chunk table, longest-first
// order, dk/dv work split) from the launch's parameter block into the
// workspace: the tables are small, and a parameter copy needs no host
// synchronisation and no allocation, and is captured by a CUDA graph.
template <int NW>
__global__ void __launch_bounds__(256) upload_kernel(const __grid_constant__ Blob<NW> b,
                                                     uint32_t* __restrict__ dst, int nwords) {
  for (int i = threadIdx.x; i < nwords; i += blockDim.x) dst[i] = b.w[i];
}
template __global__ void upload_kernel<256>(const __grid_constant__ Blob<256>, uint32_t*, int);
template __global__ void upload_kernel<1024>(const __grid_constant__ Blob<1024>, uint32_t*, int);
template __global__ void upload_kernel<4096>(const __grid_constant__ Blob<4096>, uint32_t*, int);
template __global__ void upload_kernel<kBlobMaxWords>(const __grid_constant__ Blob<kBlobMaxWords>,
                                                      uint32_t*, int);

// grid (nchunks, Hkv, ceil(Dv / 32)), block 256: a CTA takes 32 channels of
// one chunk and kv head, thread = (row group of 16 rows, channel); the eight
// groups are scanned in parallel and joined through shared memory.  Few
// registers per thread keep many warps per SM, so that many loads are in
// flight and one CTA's loads overlap another's scan and stores.
//
// Besides L and tot, the tensor-core path needs:
//   Vt_s[c] = v_s[c] * exp(tot[c] - L_s[c])     values pre-decayed to the chunk's
//             last row, for key blocks strictly before a query chunk, stored
//             as fp16 times 2^-e (e = vt_exponent(lvt), lvt[c] = log2 of the
//             column's largest |Vt|), so that no stored value exceeds 2^15;
//   safe[ci * Hkv + kv] = every g of the chunk is <= 0 and every |v| <=
//             FIX_F16_VMAX (then e = 0 and every later scaling is <= 1); the
//             schedule upload sets it to 1 and every CTA of the chunk ANDs
//             its part in;
//   rho[c] = (min_t L_t[c] + max_t L_t[c]) / 2,  hr[c] = (max - min) / 2,
//   Vm_s[c] = v_s[c] * exp(rho[c] - L_s[c])       (|exponent| <= hr), stored as
//             a pair of bf16 (hi, lo = bf16(Vm - hi)) for a near-exact
//             diagonal block,
// so that exp(G_t - G_s) = exp(L_t - rho) * exp(rho - L_s) with both factors
// inside [e^-hr, e^hr].  Channels with hr > FIX_HR_MAX or |rho| > FIX_RHO_MAX
// are out of range (see fix_common.cuh): Vm = 0, rho = 0, hr = FIX_HR_BAD.
constexpr int kPrefixThreads = 256;
constexpr int kPrefixGroups = kPrefixThreads / 32;        // row groups of 32 channels
constexpr int kPrefixRows = FIX_CHUNK / kPrefixGroups;    // rows per thread

__global__ void __launch_bounds__(kPrefixThreads, 4) prefix_kernel(
    Dims d, const Chunk* __restrict__ chunks, const float* __restrict__ g,
    const __nv_bfloat16* __restrict__ v, float* __restrict__ L, float* __restrict__ Lt,
    uint16_t* __restrict__ vt,
    __nv_bfloat16* __restrict__ vm, __nv_bfloat16* __restrict__ vml, float* __restrict__ tot,
    float* __restrict__ rho, float* __restrict__ hr, float* __restrict__ lvt,
    int* __restrict__ safe, int* __restrict__ badflag, int* __restrict__ hmax) {
  __shared__ float part[kPrefixThreads], pmin[kPrefixThreads], pmax[kPrefixThreads];
  __shared__ float tr[32][FIX_CHUNK + 1];   // the slab of L, channel-major (for Lt)
  const int Dv = d.Dv;
  const int cl = threadIdx.x & 31, grp = threadIdx.x >> 5;
  const int c = blockIdx.z * 32 + cl;
  const bool act = c < Dv;
  const int ci = blockIdx.x, kv = blockIdx.y;
  const Chunk ch = chunks[ci];
  // the backward's per-(chunk, q head) max |do|, raised by its preprocess
  if (hmax && blockIdx.z == 0 && threadIdx.x < d.grp)
    hmax[(size_t)ci * d.Hq + kv * d.grp + threadIdx.x] = 0;
  const size_t rs = (size_t)d.Hkv * Dv;
  const size_t base = (size_t)ch.tok0 * rs + (size_t)kv * Dv + (act ? c : 0);
  const int r0 = grp * kPrefixRows;
  const int nr = act ? max(0, min(kPrefixRows, ch.len - r0)) : 0;
  float lv[kPrefixRows], vv[kPrefixRows];
  float acc = 0.f, lmin = INFINITY, lmax = -INFINITY;
  bool nonpos = true;
  // g and v in one round trip (v only on the tensor-core path); a scalar gate
  // ([N, Hkv]) is the same for every channel of the token
  const size_t gbase = d.scalar_gate ? (size_t)ch.tok0 * d.Hkv + kv : base;
  const size_t grs = d.scalar_gate ? (size_t)d.Hkv : rs;
#pragma unroll
  for (int u = 0; u < kPrefixRows; ++u)
    if (u < nr) lv[u] = g[gbase + (size_t)(r0 + u) * grs];
  if (vt) {
#pragma unroll
    for (int u = 0; u < kPrefixRows; ++u)
      if (u < nr) vv[u] = bf2f(v[base + (size_t)(r0 + u) * rs]);
  }
#pragma unroll
  for (int u = 0; u < kPrefixRows; ++u) {
    if (u < nr) {
      nonpos = nonpos && lv[u] <= 0.f;
      acc += lv[u];
      lv[u] = acc;
      lmin = fminf(lmin, acc);
      lmax = fmaxf(lmax, acc);
    }
  }
  part[threadIdx.x] = acc;
  pmin[threadIdx.x] = lmin;
  pmax[threadIdx.x] = lmax;
  __syncthreads();
  float off = 0.f, total = 0.f, cmin = INFINITY, cmax = -INFINITY;
#pragma unroll
  for (int q = 0; q < kPrefixGroups; ++q) {
    const float pq = part[q * 32 + cl];
    if (q < grp) off += pq;
    cmin = fminf(cmin, total + pmin[q * 32 + cl]);
    cmax = fmaxf(cmax, total + pmax[q * 32 + cl]);
    total += pq;
  }
#pragma unroll
  for (int u = 0; u < kPrefixRows; ++u)
    if (u < nr) {
      lv[u] += off;
      L[base + (size_t)(r0 + u) * rs] = lv[u];
      if (Lt) tr[cl][r0 + u] = lv[u];
    }
  const size_t ti = ((size_t)ci * d.Hkv + kv) * Dv + c;
  if (grp == 0 && act) tot[ti] = total;
  if (Lt) {
    // L channel-major: a warp writes 32 consecutive tokens of one channel
    __syncthreads();
    const int lane = threadIdx.x & 31;
    for (int j = grp; j < 32; j += kPrefixGroups) {
      const int cj = blockIdx.z * 32 + j;
      if (cj >= Dv) break;
      float* dst = Lt + ((size_t)kv * Dv + cj) * d.N + ch.tok0;
      for (int r = lane; r < ch.len; r += 32) dst[r] = tr[j][r];
    }
  }
  if (!vt) return;  // uniform: the exact kernels need only L and tot
  float vmax = 0.f, xmax = 0.f;
#pragma unroll
  for (int u = 0; u < kPrefixRows; ++u)
    if (u < nr) {
      vmax = fmaxf(vmax, fabsf(vv[u]));
      xmax = fmaxf(xmax, fabsf(vv[u] * exp_op(total - lv[u])));
    }
  const int f16 = __syncthreads_and(nonpos && vmax <= FIX_F16_VMAX);   // part[] free after this
  if (threadIdx.x == 0 && !f16) atomicAnd(safe + (size_t)ci * d.Hkv + kv, 0);
  part[threadIdx.x] = xmax;
  const float half = 0.5f * (cmax - cmin);
  const float mid = 0.5f * (cmax + cmin);
  const bool good = !act || (half <= FIX_HR_MAX && fabsf(mid) <= FIX_RHO_MAX);
  const float ref = good ? mid : 0.f;
  if (__syncthreads_or(!good) && threadIdx.x == 0) atomicOr(badflag, 1);
  float cx = 0.f;
#pragma unroll
  for (int q = 0; q < kPrefixGroups; ++q) cx = fmaxf(cx, part[q * 32 + cl]);
  const float lg = cx > 0.f ? log2f(cx) : -1e30f;
  const float sc = exp2f(-vt_exponent(lg));
  if (grp == 0 && act) {
    rho[ti] = ref;
    hr[ti] = ch.len > 0 ? (good ? half : FIX_HR_BAD) : 0.f;
    lvt[ti] = lg;
  }
#pragma unroll
  for (int u = 0; u < kPrefixRows; ++u)
    if (u < nr) {
      const size_t a = base + (size_t)(r0 + u) * rs;
      const float xt = vv[u] * exp_op(total - lv[u]);
      vt[a] = __half_as_ushort(__float2half_rn(xt * sc));
      const float xm = good ? vv[u] * exp_op(ref - lv[u]) : 0.f;
      const __nv_bfloat16 xm_hi = f2bf(xm);
      vm[a] = xm_hi;
      vml[a] = f2bf(xm - bf2f(xm_hi));   // Vm = hi + lo to ~16 bits
    }
}

// Reverse cumsum of dG within each sequence (dg_r = sum_{t >= r} dG_t), in two
// launches over the same chunk table: chunk totals, then local reverse scans
// plus the totals of the later chunks of the same sequence.  Both use the
// prefix pass's block shape: grid (nchunks, Hkv, ceil(Dv / 32)), 256 threads =
// (row group, channel), every row of a group loaded up front, groups joined
// through shared memory.
__global__ void __launch_bounds__(kPrefixThreads) chunk_total_kernel(Dims d,
                                                                     const Chunk* __restrict__ chunks,
                                                                     const float* __restrict__ x,
                                                                     float* __restrict__ tot) {
  __shared__ float part[kPrefixThreads];
  const int Dv = d.Dv;
  const int cl = threadIdx.x & 31, grp = threadIdx.x >> 5;
  const int c = blockIdx.z * 32 + cl;
  const bool act = c < Dv;
  const int ci = blockIdx.x, kv = blockIdx.y;
  const Chunk ch = chunks[ci];
  const size_t rs = (size_t)d.Hkv * Dv;
  const size_t base = (size_t)ch.tok0 * rs + (size_t)kv * Dv + (act ? c : 0);
  const int r0 = grp * kPrefixRows;
  const int nr = act ? max(0, min(kPrefixRows, ch.len - r0)) : 0;
  float xv[kPrefixRows];
#pragma unroll
  for (int u = 0; u < kPrefixRows; ++u) xv[u] = u < nr ? x[base + (size_t)(r0 + u) * rs] : 0.f;
  float acc = 0.f;
#pragma unroll
  for (int u = 0; u < kPrefixRows; ++u) acc += xv[u];
  part[threadIdx.x] = acc;
  __syncthreads();
  if (grp == 0 && act) {
    float t = 0.f;
#pragma unroll
    for (int q = 0; q < kPrefixGroups; ++q) t += part[q * 32 + cl];
    tot[((size_t)ci * d.Hkv + kv) * Dv + c] = t;
  }
}

// out[r] = sum of the D values of row r (a warp per row, fixed order).
__global__ void __launch_bounds__(256) channel_sum_kernel(const float* __restrict__ x,
                                                          long long rows, int D,
                                                          float* __restrict__ out) {
  const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float s = 0.f;
  for (int c = lane; c < D; c += 32) s += x[r * D + c];
  s = warp_sum(s);
  if (lane == 0) out[r] = s;
}

__global__ void __launch_bounds__(kPrefixThreads) reverse_cumsum_kernel(
    Dims d, const Chunk* __restrict__ chunks, const float* __restrict__ x,
    const float* __restrict__ tot, float* __restrict__ out) {
  __shared__ float part[kPrefixThreads];
  const int Dv = d.Dv;
  const int cl = threadIdx.x & 31, grp = threadIdx.x >> 5;
  const int c = blockIdx.z * 32 + cl;
  const bool act = c < Dv;
  const int ci = blockIdx.x, kv = blockIdx.y;
  const Chunk ch = chunks[ci];
  const size_t rs = (size_t)d.Hkv * Dv;
  const size_t base = (size_t)ch.tok0 * rs + (size_t)kv * Dv + (act ? c : 0);
  const int r0 = grp * kPrefixRows;
  const int nr = act ? max(0, min(kPrefixRows, ch.len - r0)) : 0;
  float xv[kPrefixRows];
#pragma unroll
  for (int u = 0; u < kPrefixRows; ++u) xv[u] = u < nr ? x[base + (size_t)(r0 + u) * rs] : 0.f;
  // the later chunks of the sequence, in order
  float acc = 0.f;
  const int first = ci - ch.j;
  if (act)
    for (int jj = ch.nch - 1; jj > ch.j; --jj) acc += tot[((size_t)(first + jj) * d.Hkv + kv) * Dv + c];
  float own = 0.f;
#pragma unroll
  for (int u = 0; u < kPrefixRows; ++u) own += xv[u];
  part[threadIdx.x] = own;
  __syncthreads();
  // then the later row groups of this chunk, from the last one down
  for (int q = kPrefixGroups - 1; q > grp; --q) acc += part[q * 32 + cl];
#pragma unroll
  for (int u = kPrefixRows - 1; u >= 0; --u)
    if (u < nr) {
      acc += xv[u];
      out[base + (size_t)(r0 + u) * rs] = acc;
    }
}

}  // namespace fix
