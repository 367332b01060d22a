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

// grid (nchunks, Hkv, channel slices of 64), block 256: a CTA takes one
// chunk of one kv head and up to 64 of its channels; a half-warp covers a
// row of the slice (a lane per 4 consecutive channels: 16-byte g and L, and
// 8-byte v and 16-bit output accesses), so a warp covers two rows and every
// row group (a half-warp) 8 rows.  The sixteen row groups are scanned in
// parallel and joined through shared memory.  Slicing the channels gives
// two CTAs per (chunk, kv head) at Dv = 128 and several CTAs per SM.
//
// Besides L and tot, the tensor-core path needs:
//   Lt = L channel-major [Hkv][Dv][N] (forward only), written through a
//             shared-memory transpose so that a warp stores 32 consecutive
//             tokens of one channel;
//   Vt_s[c] = v_s[c] * exp(tot[c] - L_s[c])     values pre-decayed to the chunk's
//             last row, for key blocks strictly before a query chunk, stored
//             as fp16 times 2^-e (e = vt_exponent(lvt), lvt[c] = log2 of the
//             column's largest |Vt|), so that no stored value exceeds 2^15;
//   safe[ci * Hkv + kv] = every g of the chunk is <= 0 and every |v| <=
//             FIX_F16_VMAX (then e = 0 and every later scaling is <= 1); the
//             schedule upload sets it to 1 and the CTA ANDs its result in;
//   rho[c] = (min_t L_t[c] + max_t L_t[c]) / 2,  hr[c] = (max - min) / 2,
//   Vm_s[c] = v_s[c] * exp(rho[c] - L_s[c])       (|exponent| <= hr), stored as
//             a pair of bf16 (hi, lo = bf16(Vm - hi)) for a near-exact
//             diagonal block,
// so that exp(G_t - G_s) = exp(L_t - rho) * exp(rho - L_s) with both factors
// inside [e^-hr, e^hr].  Channels with hr > FIX_HR_MAX or |rho| > FIX_RHO_MAX
// are out of range (see fix_common.cuh): Vm = 0, rho = 0, hr = FIX_HR_BAD.
// the dG scans: the same slicing as the prefix pass (64-channel slices, a
// half-warp per row, 16 row groups of 8 rows)
constexpr int kPrefixThreads = 256;
constexpr int kPrefixGroups = kPrefixThreads / 16;        // row groups
constexpr int kPrefixRows = FIX_CHUNK / kPrefixGroups;    // rows per thread
// the prefix pass itself: channel slices of 64, a half-warp per row
constexpr int kPfxThreads = 256;
constexpr int kPfxLanes = 16;                             // lanes per row
constexpr int kPfxSlice = 4 * kPfxLanes;                  // channels per CTA
constexpr int kPfxGroups = kPfxThreads / kPfxLanes;       // row groups
constexpr int kPfxRows = FIX_CHUNK / kPfxGroups;

int prefix_slices(int Dv) { return Dv > kPfxSlice ? Dv / kPfxSlice : 1; }

size_t prefix_smem_bytes(int Dv, bool lt) {
  const int sl = Dv < kPfxSlice ? Dv : kPfxSlice;
  return (size_t)4 * kPfxGroups * sl * sizeof(float) +
         (lt ? (size_t)sl * (FIX_CHUNK + 1) * sizeof(float) : 0);
}

namespace {
__device__ __forceinline__ float4 f4_add(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}
__device__ __forceinline__ float4 f4_min(float4 a, float4 b) {
  return make_float4(fminf(a.x, b.x), fminf(a.y, b.y), fminf(a.z, b.z), fminf(a.w, b.w));
}
__device__ __forceinline__ float4 f4_max(float4 a, float4 b) {
  return make_float4(fmaxf(a.x, b.x), fmaxf(a.y, b.y), fmaxf(a.z, b.z), fmaxf(a.w, b.w));
}
__device__ __forceinline__ float f4_get(const float4& a, int k) {
  return k == 0 ? a.x : k == 1 ? a.y : k == 2 ? a.z : a.w;
}
__device__ __forceinline__ void bf4_unpack(uint2 u, float* x) {
  x[0] = __uint_as_float(u.x << 16);
  x[1] = __uint_as_float(u.x & 0xFFFF0000u);
  x[2] = __uint_as_float(u.y << 16);
  x[3] = __uint_as_float(u.y & 0xFFFF0000u);
}
}  // namespace

__global__ void __launch_bounds__(kPfxThreads, 2) prefix_kernel(
    Dims d, const Chunk* __restrict__ chunks, const float* __restrict__ g,
    const __nv_bfloat16* __restrict__ v, float* __restrict__ L, float* __restrict__ Lt,
    uint16_t* __restrict__ vt, __nv_bfloat16* __restrict__ vm, __nv_bfloat16* __restrict__ vml,
    float* __restrict__ tot, float* __restrict__ rho, float* __restrict__ hr,
    float* __restrict__ lvt, int* __restrict__ safe, int* __restrict__ badflag,
    int* __restrict__ hmax) {
  extern __shared__ float psm[];
  const int Dv = d.Dv;
  const int sl = Dv < kPfxSlice ? Dv : kPfxSlice;   // channels of this CTA
  const int cb = blockIdx.z * sl;                    // its first channel
  const int nq = sl / 4;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int qd = lane % kPfxLanes;                   // channel quad in the slice
  const int grp = warp * (32 / kPfxLanes) + lane / kPfxLanes;   // row group
  const bool act = qd < nq;
  const int cl = 4 * (act ? qd : 0);                 // channel in the slice
  const int c0 = cb + cl;
  const int ci = blockIdx.x, kv = blockIdx.y;
  const Chunk ch = chunks[ci];
  float* part = psm;                     // [groups][sl] group totals
  float* pmin = part + kPfxGroups * sl;  // [groups][sl] group minima of L
  float* pmax = pmin + kPfxGroups * sl;  // [groups][sl] group maxima
  float* pxm = pmax + kPfxGroups * sl;   // [groups][sl] group max |Vt|
  float* tr = pxm + kPfxGroups * sl;     // [sl][FIX_CHUNK + 1] L, channel-major
  // the backward's per-(chunk, q head) max |do|, raised by its preprocess
  if (hmax && blockIdx.z == 0 && threadIdx.x < d.grp)
    hmax[(size_t)ci * d.Hq + kv * d.grp + threadIdx.x] = 0;
  const size_t rs = (size_t)d.Hkv * Dv;
  const size_t base = (size_t)ch.tok0 * rs + (size_t)kv * Dv + c0;
  const int r0 = grp * kPfxRows;
  const int nr = act ? max(0, min(kPfxRows, ch.len - r0)) : 0;
  float4 lv[kPfxRows];
  uint2 vv[kPfxRows];
  // g and v in one round trip (v only on the tensor-core path); a scalar gate
  // ([N, Hkv]) is the same for every channel of the token
#pragma unroll
  for (int u = 0; u < kPfxRows; ++u) {
    if (u < nr) {
      if (d.scalar_gate) {
        const float x = g[((size_t)ch.tok0 + r0 + u) * d.Hkv + kv];
        lv[u] = make_float4(x, x, x, x);
      } else {
        lv[u] = *reinterpret_cast<const float4*>(g + base + (size_t)(r0 + u) * rs);
      }
    }
  }
  if (vt) {
#pragma unroll
    for (int u = 0; u < kPfxRows; ++u)
      if (u < nr) vv[u] = *reinterpret_cast<const uint2*>(v + base + (size_t)(r0 + u) * rs);
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 lmin = make_float4(INFINITY, INFINITY, INFINITY, INFINITY);
  float4 lmax = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
  bool nonpos = true;
#pragma unroll
  for (int u = 0; u < kPfxRows; ++u) {
    if (u < nr) {
      nonpos = nonpos && lv[u].x <= 0.f && lv[u].y <= 0.f && lv[u].z <= 0.f && lv[u].w <= 0.f;
      acc = f4_add(acc, lv[u]);
      lv[u] = acc;
      lmin = f4_min(lmin, acc);
      lmax = f4_max(lmax, acc);
    }
  }
  if (act) {
    *reinterpret_cast<float4*>(part + grp * sl + cl) = acc;
    *reinterpret_cast<float4*>(pmin + grp * sl + cl) = lmin;
    *reinterpret_cast<float4*>(pmax + grp * sl + cl) = lmax;
  }
  __syncthreads();
  float4 off = make_float4(0.f, 0.f, 0.f, 0.f), total = off;
  float4 cmin = make_float4(INFINITY, INFINITY, INFINITY, INFINITY);
  float4 cmax = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
  if (act) {
#pragma unroll
    for (int q = 0; q < kPfxGroups; ++q) {
      const float4 pq = *reinterpret_cast<const float4*>(part + q * sl + cl);
      if (q < grp) off = f4_add(off, pq);
      cmin = f4_min(cmin, f4_add(total, *reinterpret_cast<const float4*>(pmin + q * sl + cl)));
      cmax = f4_max(cmax, f4_add(total, *reinterpret_cast<const float4*>(pmax + q * sl + cl)));
      total = f4_add(total, pq);
    }
  }
#pragma unroll
  for (int u = 0; u < kPfxRows; ++u)
    if (u < nr) {
      lv[u] = f4_add(lv[u], off);
      *reinterpret_cast<float4*>(L + base + (size_t)(r0 + u) * rs) = lv[u];
      if (Lt) {
#pragma unroll
        for (int k = 0; k < 4; ++k) tr[(cl + k) * (FIX_CHUNK + 1) + r0 + u] = f4_get(lv[u], k);
      }
    }
  const size_t ti = ((size_t)ci * d.Hkv + kv) * Dv + c0;
  if (grp == 0 && act) *reinterpret_cast<float4*>(tot + ti) = total;
  if (Lt) {
    // L channel-major: a warp stores 32 consecutive tokens of one channel
    __syncthreads();
    for (int c = warp; c < sl; c += kPfxThreads / 32) {
      float* dst = Lt + ((size_t)kv * Dv + cb + c) * d.N + ch.tok0;
      for (int r = lane; r < ch.len; r += 32) dst[r] = tr[c * (FIX_CHUNK + 1) + r];
    }
  }
  if (!vt) return;  // uniform: the exact kernels need only L and tot
  float vmax = 0.f;
  float4 xmax = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int u = 0; u < kPfxRows; ++u)
    if (u < nr) {
      float x[4];
      bf4_unpack(vv[u], x);
#pragma unroll
      for (int k = 0; k < 4; ++k) vmax = fmaxf(vmax, fabsf(x[k]));
      xmax.x = fmaxf(xmax.x, fabsf(x[0] * exp_op(total.x - lv[u].x)));
      xmax.y = fmaxf(xmax.y, fabsf(x[1] * exp_op(total.y - lv[u].y)));
      xmax.z = fmaxf(xmax.z, fabsf(x[2] * exp_op(total.z - lv[u].z)));
      xmax.w = fmaxf(xmax.w, fabsf(x[3] * exp_op(total.w - lv[u].w)));
    }
  if (act) *reinterpret_cast<float4*>(pxm + grp * sl + cl) = xmax;
  const int f16 = __syncthreads_and(nonpos && vmax <= FIX_F16_VMAX);
  if (threadIdx.x == 0 && !f16) atomicAnd(safe + (size_t)ci * d.Hkv + kv, 0);
  float ref[4], hrng[4], lg[4], sc[4];
  bool good[4];
  bool any_bad = false;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    hrng[k] = 0.5f * (f4_get(cmax, k) - f4_get(cmin, k));
    const float mid = 0.5f * (f4_get(cmax, k) + f4_get(cmin, k));
    good[k] = !act || ch.len <= 0 || (hrng[k] <= FIX_HR_MAX && fabsf(mid) <= FIX_RHO_MAX);
    ref[k] = good[k] ? mid : 0.f;
    any_bad = any_bad || !good[k];
    float cx = 0.f;
    if (act) {
#pragma unroll
      for (int q = 0; q < kPfxGroups; ++q) cx = fmaxf(cx, pxm[q * sl + cl + k]);
    }
    lg[k] = cx > 0.f ? log2f(cx) : -1e30f;
    sc[k] = exp2f(-vt_exponent(lg[k]));
  }
  if (__syncthreads_or(any_bad) && threadIdx.x == 0) atomicOr(badflag, 1);
  if (grp == 0 && act) {
    *reinterpret_cast<float4*>(rho + ti) = make_float4(ref[0], ref[1], ref[2], ref[3]);
    float h4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) h4[k] = ch.len > 0 ? (good[k] ? hrng[k] : FIX_HR_BAD) : 0.f;
    *reinterpret_cast<float4*>(hr + ti) = make_float4(h4[0], h4[1], h4[2], h4[3]);
    *reinterpret_cast<float4*>(lvt + ti) = make_float4(lg[0], lg[1], lg[2], lg[3]);
  }
#pragma unroll
  for (int u = 0; u < kPfxRows; ++u)
    if (u < nr) {
      float x[4], xt[4], xm[4], hi[4], lo[4];
      bf4_unpack(vv[u], x);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float lk = f4_get(lv[u], k);
        xt[k] = x[k] * exp_op(f4_get(total, k) - lk) * sc[k];
        xm[k] = good[k] ? x[k] * exp_op(ref[k] - lk) : 0.f;
        hi[k] = __bfloat162float(__float2bfloat16_rn(xm[k]));
        lo[k] = xm[k] - hi[k];   // Vm = hi + lo to ~16 bits
      }
      const size_t a = base + (size_t)(r0 + u) * rs;
      const __half2 t01 = __floats2half2_rn(xt[0], xt[1]), t23 = __floats2half2_rn(xt[2], xt[3]);
      const __nv_bfloat162 h01 = __floats2bfloat162_rn(hi[0], hi[1]), h23 = __floats2bfloat162_rn(hi[2], hi[3]);
      const __nv_bfloat162 l01 = __floats2bfloat162_rn(lo[0], lo[1]), l23 = __floats2bfloat162_rn(lo[2], lo[3]);
      *reinterpret_cast<uint2*>(vt + a) =
          make_uint2(*reinterpret_cast<const uint32_t*>(&t01), *reinterpret_cast<const uint32_t*>(&t23));
      *reinterpret_cast<uint2*>(vm + a) =
          make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
      *reinterpret_cast<uint2*>(vml + a) =
          make_uint2(*reinterpret_cast<const uint32_t*>(&l01), *reinterpret_cast<const uint32_t*>(&l23));
    }
}

// Reverse cumsum of dG within each sequence (dg_r = sum_{t >= r} dG_t), in two
// launches over the same chunk table: chunk totals, then local reverse scans
// plus the totals of the later chunks of the same sequence.  Both use the
// prefix pass's block shape: grid (nchunks, Hkv), 256 threads = (row group,
// 4 channels), every row of a group loaded up front as 16-byte vectors,
// groups joined through shared memory.
__global__ void __launch_bounds__(kPrefixThreads) chunk_total_kernel(Dims d,
                                                                     const Chunk* __restrict__ chunks,
                                                                     const float* __restrict__ x,
                                                                     float* __restrict__ tot) {
  __shared__ float4 part[kPrefixGroups][16];
  const int Dv = d.Dv;
  const int sl = Dv < kPfxSlice ? Dv : kPfxSlice;
  const int nq = sl / 4;
  const int lane = threadIdx.x & 31, qd = lane & 15;
  const int grp = (threadIdx.x >> 5) * 2 + (lane >> 4);
  const bool act = qd < nq;
  const int c0 = blockIdx.z * sl + 4 * (act ? qd : 0);
  const int ci = blockIdx.x, kv = blockIdx.y;
  const Chunk ch = chunks[ci];
  const size_t rs = (size_t)d.Hkv * Dv;
  const size_t base = (size_t)ch.tok0 * rs + (size_t)kv * Dv + c0;
  const int r0 = grp * kPrefixRows;
  const int nr = act ? max(0, min(kPrefixRows, ch.len - r0)) : 0;
  float4 xv[kPrefixRows];
#pragma unroll
  for (int u = 0; u < kPrefixRows; ++u)
    if (u < nr) xv[u] = *reinterpret_cast<const float4*>(x + base + (size_t)(r0 + u) * rs);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int u = 0; u < kPrefixRows; ++u)
    if (u < nr) acc = f4_add(acc, xv[u]);
  part[grp][qd] = acc;
  __syncthreads();
  if (grp == 0 && act) {
    float4 t = part[0][qd];
#pragma unroll
    for (int q = 1; q < kPrefixGroups; ++q) t = f4_add(t, part[q][qd]);
    *reinterpret_cast<float4*>(tot + ((size_t)ci * d.Hkv + kv) * Dv + c0) = t;
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
  __shared__ float4 part[kPrefixGroups][16], later[kPrefixGroups][16];
  const int Dv = d.Dv;
  const int sl = Dv < kPfxSlice ? Dv : kPfxSlice;
  const int nq = sl / 4;
  const int lane = threadIdx.x & 31, qd = lane & 15;
  const int grp = (threadIdx.x >> 5) * 2 + (lane >> 4);
  const bool act = qd < nq;
  const int c0 = blockIdx.z * sl + 4 * (act ? qd : 0);
  const int ci = blockIdx.x, kv = blockIdx.y;
  const Chunk ch = chunks[ci];
  const size_t rs = (size_t)d.Hkv * Dv;
  const size_t base = (size_t)ch.tok0 * rs + (size_t)kv * Dv + c0;
  const int r0 = grp * kPrefixRows;
  const int nr = act ? max(0, min(kPrefixRows, ch.len - r0)) : 0;
  float4 xv[kPrefixRows];
#pragma unroll
  for (int u = 0; u < kPrefixRows; ++u)
    if (u < nr) xv[u] = *reinterpret_cast<const float4*>(x + base + (size_t)(r0 + u) * rs);
  // the totals of the sequence's later chunks: row group q takes chunks
  // j + 1 + q, j + 1 + q + 16, ... (two accumulators, so that the loads
  // overlap); the groups' sums are then added in group order
  const int first = ci - ch.j;
  float4 la = make_float4(0.f, 0.f, 0.f, 0.f), lb = la;
  if (act) {
    int jj = ch.j + 1 + grp;
    for (; jj + kPrefixGroups < ch.nch; jj += 2 * kPrefixGroups) {
      la = f4_add(la, *reinterpret_cast<const float4*>(tot + ((size_t)(first + jj) * d.Hkv + kv) * Dv + c0));
      lb = f4_add(lb, *reinterpret_cast<const float4*>(
                          tot + ((size_t)(first + jj + kPrefixGroups) * d.Hkv + kv) * Dv + c0));
    }
    if (jj < ch.nch)
      la = f4_add(la, *reinterpret_cast<const float4*>(tot + ((size_t)(first + jj) * d.Hkv + kv) * Dv + c0));
  }
  float4 own = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int u = 0; u < kPrefixRows; ++u)
    if (u < nr) own = f4_add(own, xv[u]);
  part[grp][qd] = own;
  later[grp][qd] = f4_add(la, lb);
  __syncthreads();
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int q = 0; q < kPrefixGroups; ++q) acc = f4_add(acc, later[q][qd]);
  // then the later row groups of this chunk, from the last one down
  for (int q = kPrefixGroups - 1; q > grp; --q) acc = f4_add(acc, part[q][qd]);
#pragma unroll
  for (int u = kPrefixRows - 1; u >= 0; --u)
    if (u < nr) {
      acc = f4_add(acc, xv[u]);
      *reinterpret_cast<float4*>(out + base + (size_t)(r0 + u) * rs) = acc;
    }
}

}  // namespace fix
