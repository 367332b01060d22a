// Gate prefix pass and packed-sequence schedule.
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

// order[] lists chunk ids by decreasing chunk index j (the number of key
// blocks before the diagonal), so that grids walking order[] start the
// longest causal rows first.  maxj is an upper bound on j + 1; if it exceeds
// the histogram, order[] is the identity.  Run by one whole CTA.
__device__ void order_chunks(const Chunk* __restrict__ chunks, int nchunks, int maxj,
                             int* __restrict__ order) {
  constexpr int kBins = 4096;
  __shared__ int hist[kBins];
  if (maxj > kBins) {
    for (int i = threadIdx.x; i < nchunks; i += blockDim.x) order[i] = i;
    return;
  }
  for (int b = threadIdx.x; b < maxj; b += blockDim.x) hist[b] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < nchunks; i += blockDim.x)
    atomicAdd(&hist[min(max(chunks[i].j, 0), maxj - 1)], 1);
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int b = maxj - 1; b >= 0; --b) {
      const int c = hist[b];
      hist[b] = acc;
      acc += c;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nchunks; i += blockDim.x)
    order[atomicAdd(&hist[min(max(chunks[i].j, 0), maxj - 1)], 1)] = i;
}

// Single CTA: turns sequence lengths (device cu_seqlens, or B sequences of T
// tokens when cu is NULL) into the chunk table, sequences in order.  The table
// has `cap` entries (the count the host derived from its cu_seqlens mirror);
// every entry is first set empty, writes past `cap` are dropped and lengths
// are clamped to the N tokens, so a device array that disagrees with the host
// mirror cannot send any kernel outside its buffers.
// Exclusive prefix sum over the threads of a CTA (blockDim a multiple of 32):
// warp shuffles, then the warp totals through `scan`; *total gets the sum.
__device__ int block_excl_scan(int v, int* scan, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scan[w] = x;
  __syncthreads();
  int off = 0, tot = 0;
  for (int i = 0; i < nw; ++i) {
    const int t = scan[i];
    if (i < w) off += t;
    tot += t;
  }
  __syncthreads();   // scan[] is reused by the next call
  *total = tot;
  return off + x - v;
}

// Number of 64-row query tiles from chunk j to the end of a sequence of L
// tokens (every chunk but the last is a whole number of tiles).
__device__ __host__ inline int tiles64_from(int L, int j) {
  return (L - j * FIX_CHUNK + 63) / 64;
}

__global__ void __launch_bounds__(kScheduleThreads) schedule_kernel(const int64_t* __restrict__ cu, int nseq,
                                                        int T, int N, int cap,
                                                        Chunk* __restrict__ out, int maxj,
                                                        int* __restrict__ order, PartSpec ps) {
  __shared__ int scan[kScheduleThreads / 32];
  for (int i = threadIdx.x; i < cap; i += blockDim.x) out[i] = Chunk{0, 0, 0, 0};
  __syncthreads();
  int carry = 0;
  for (int first = 0; first < nseq; first += blockDim.x) {
    const int i = first + threadIdx.x;
    long long s0 = 0;
    int L = 0;
    if (i < nseq) {
      if (cu) {
        s0 = cu[i];
        const long long e = cu[i + 1];
        s0 = s0 < 0 ? 0 : (s0 > N ? N : s0);
        L = (int)((e > N ? N : e) - s0);
        if (L < 0) L = 0;
      } else {
        s0 = (long long)i * T;
        L = T;
      }
    }
    const int nc = (L + FIX_CHUNK - 1) / FIX_CHUNK;
    int tot;
    const int excl = carry + block_excl_scan(nc, scan, &tot);
    const int ncw = max(0, min(nc, cap - excl));   // chunks that fit the table
    for (int j = 0; j < ncw; ++j) {
      Chunk c;
      c.tok0 = (int)(s0 + (long long)j * FIX_CHUNK);
      c.len = min(FIX_CHUNK, L - j * FIX_CHUNK);
      c.j = j;
      c.nch = ncw;
      out[excl + j] = c;
    }
    carry += tot;
  }
  if (order) {
    __threadfence_block();
    __syncthreads();
    order_chunks(out, cap, maxj, order);
  }
  if (!ps.parts) return;
  // dk/dv work split: key chunk j of a sequence of L tokens has grp * h_j
  // diagonal tiles (h_j = its 64-row halves) and grp * (tiles64_from(L, j) -
  // h_j) later ones, each kind cut into runs of at most P tiles.  parts[]
  // holds every later-block part first (the long ones start first), then the
  // diagonal parts; a key chunk's slots are consecutive, diagonal parts first.
  auto seq_len = [&](int i) -> int {
    if (i >= nseq) return 0;
    if (!cu) return T;
    long long s0 = cu[i];
    const long long e = cu[i + 1];
    s0 = s0 < 0 ? 0 : (s0 > N ? N : s0);
    const long long L = (e > N ? N : e) - s0;
    return L < 0 ? 0 : (int)L;
  };
  const int P = ps.tiles_per_part;
  auto n_diag = [&](int L, int j) { return (ps.grp * fix_halves(L, j) + P - 1) / P; };
  auto n_off = [&](int L, int j) {
    return (ps.grp * (tiles64_from(L, j) - fix_halves(L, j)) + P - 1) / P;
  };
  int total_off = 0;
  for (int first = 0; first < nseq; first += blockDim.x) {
    const int L = seq_len(first + threadIdx.x);
    const int nc = (L + FIX_CHUNK - 1) / FIX_CHUNK;
    int no = 0;
    for (int j = 0; j < nc; ++j) no += n_off(L, j);
    int t;
    block_excl_scan(no, scan, &t);
    total_off += t;
  }
  int cbase = 0, obase = 0, dbase = 0, sbase = 0;
  for (int first = 0; first < nseq; first += blockDim.x) {
    const int L = seq_len(first + threadIdx.x);
    const int nc = (L + FIX_CHUNK - 1) / FIX_CHUNK;
    int no = 0, nd = 0;
    for (int j = 0; j < nc; ++j) {
      no += n_off(L, j);
      nd += n_diag(L, j);
    }
    int ctot, otot, dtot, stot;
    const int c0 = cbase + block_excl_scan(nc, scan, &ctot);
    int o = obase + block_excl_scan(no, scan, &otot);
    int e = total_off + dbase + block_excl_scan(nd, scan, &dtot);
    int s0 = sbase + block_excl_scan(no + nd, scan, &stot);
    for (int j = 0; j < nc && c0 + j < cap; ++j) {
      const int ndj = n_diag(L, j), noj = n_off(L, j);
      ps.cpart[c0 + j] = make_int2(ndj + noj, s0);
      for (int p = 0; p < ndj; ++p, ++e)
        if (e < ps.cap_parts) ps.parts[e] = Part{c0 + j, p, s0 + p, 1};
      for (int p = 0; p < noj; ++p, ++o)
        if (o < ps.cap_parts) ps.parts[o] = Part{c0 + j, p, s0 + ndj + p, 0};
      s0 += ndj + noj;
    }
    cbase += ctot;
    obase += otot;
    dbase += dtot;
    sbase += stot;
  }
}

// grid (nchunks, Hkv), block 512: thread = (row group, channel); the chunk's
// 128 rows are split into 512 / Dv groups scanned in parallel and joined
// through shared memory.
//
// Besides L and tot, the tensor-core path needs:
//   Vt_s[c] = v_s[c] * exp(tot[c] - L_s[c])     values pre-decayed to the chunk's
//             last row, for key blocks strictly before a query chunk.  Stored
//             as fp16 when the chunk is "fp16-safe" (every g <= 0 and every
//             |v| <= FIX_F16_VMAX, so that all later scalings stay <= |v|),
//             else as bf16; safe[ci * Hkv + kv] records which.
//   rho[c] = (min_t L_t[c] + max_t L_t[c]) / 2,  hr[c] = (max - min) / 2,
//   Vm_s[c] = v_s[c] * exp(rho[c] - L_s[c])       (|exponent| <= hr), stored as
//             a pair of bf16 (hi, lo = bf16(Vm - hi)) for a near-exact
//             diagonal block,
// so that exp(G_t - G_s) = exp(L_t - rho) * exp(rho - L_s) with both factors
// inside [e^-hr, e^hr].  Channels with hr > FIX_HR_MAX cannot be split this
// way in float range; for them Vm = 0 and rho = 0, and the kernels handle the
// diagonal block of that channel exactly in fp32.
constexpr int kPrefixThreads = 512;

__global__ void __launch_bounds__(kPrefixThreads) prefix_kernel(
    Dims d, const Chunk* __restrict__ chunks, const float* __restrict__ g,
    const __nv_bfloat16* __restrict__ v, float* __restrict__ L, uint16_t* __restrict__ vt,
    __nv_bfloat16* __restrict__ vm, __nv_bfloat16* __restrict__ vml, float* __restrict__ tot,
    float* __restrict__ rho, float* __restrict__ hr, int* __restrict__ safe,
    int* __restrict__ badflag, int* __restrict__ hmax) {
  constexpr int kMaxRows = FIX_CHUNK * 128 / kPrefixThreads;  // rows per thread at Dv = 128
  __shared__ float part[kPrefixThreads], pmin[kPrefixThreads], pmax[kPrefixThreads];
  const int Dv = d.Dv;
  const int groups = kPrefixThreads / Dv;
  const int rows = FIX_CHUNK / groups;                       // rows per group
  const int c = threadIdx.x % Dv, grp = threadIdx.x / Dv;
  const int ci = blockIdx.x, kv = blockIdx.y;
  const Chunk ch = chunks[ci];
  // the backward's per-(chunk, q head) max |do|, raised by its preprocess
  if (hmax && threadIdx.x < d.grp) hmax[(size_t)ci * d.Hq + kv * d.grp + threadIdx.x] = 0;
  const size_t rs = (size_t)d.Hkv * Dv;
  const size_t base = (size_t)ch.tok0 * rs + (size_t)kv * Dv + c;
  const int r0 = grp * rows;
  const int nr = max(0, min(rows, ch.len - r0));
  float lv[kMaxRows], vv[kMaxRows];
  float acc = 0.f, lmin = INFINITY, lmax = -INFINITY;
  bool nonpos = true;
  // g and v in one round trip (v only on the tensor-core path)
#pragma unroll
  for (int u = 0; u < kMaxRows; ++u)
    if (u < nr) lv[u] = g[base + (size_t)(r0 + u) * rs];
  if (vt) {
#pragma unroll
    for (int u = 0; u < kMaxRows; ++u)
      if (u < nr) vv[u] = bf2f(v[base + (size_t)(r0 + u) * rs]);
  }
#pragma unroll
  for (int u = 0; u < kMaxRows; ++u) {
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
  for (int q = 0; q < groups; ++q) {
    const float pq = part[q * Dv + c];
    if (q < grp) off += pq;
    cmin = fminf(cmin, total + pmin[q * Dv + c]);
    cmax = fmaxf(cmax, total + pmax[q * Dv + c]);
    total += pq;
  }
#pragma unroll
  for (int u = 0; u < kMaxRows; ++u)
    if (u < nr) {
      lv[u] += off;
      L[base + (size_t)(r0 + u) * rs] = lv[u];
    }
  const size_t ti = ((size_t)ci * d.Hkv + kv) * Dv + c;
  if (grp == 0) tot[ti] = total;
  if (!vt) return;  // uniform: the exact kernels need only L and tot
  float vmax = 0.f;
#pragma unroll
  for (int u = 0; u < kMaxRows; ++u)
    if (u < nr) vmax = fmaxf(vmax, fabsf(vv[u]));
  const int f16 = __syncthreads_and(nonpos && vmax <= FIX_F16_VMAX);
  if (threadIdx.x == 0) safe[(size_t)ci * d.Hkv + kv] = f16;
  const float half = 0.5f * (cmax - cmin);
  const bool good = half <= FIX_HR_MAX;
  const float ref = good ? 0.5f * (cmax + cmin) : 0.f;
  if (__syncthreads_or(!good) && threadIdx.x == 0) atomicOr(badflag, 1);
  if (grp == 0) {
    rho[ti] = ref;
    hr[ti] = ch.len > 0 ? half : 0.f;
  }
#pragma unroll
  for (int u = 0; u < kMaxRows; ++u)
    if (u < nr) {
      const size_t a = base + (size_t)(r0 + u) * rs;
      const float xt = vv[u] * exp_op(total - lv[u]);
      vt[a] = f16 ? __half_as_ushort(__float2half_rn(xt)) : __bfloat16_as_ushort(f2bf(xt));
      const float xm = good ? vv[u] * exp_op(ref - lv[u]) : 0.f;
      const __nv_bfloat16 xm_hi = f2bf(xm);
      vm[a] = xm_hi;
      vml[a] = f2bf(xm - bf2f(xm_hi));   // Vm = hi + lo to ~16 bits
    }
}

// Reverse cumsum of dG within each sequence (dg_r = sum_{t >= r} dG_t), in two
// launches over the same chunk table: chunk totals, then local reverse scans
// plus the totals of the later chunks of the same sequence.  Both use the
// prefix pass's block shape: 512 threads = (row group, channel), every row of
// a group loaded up front, groups joined through shared memory.
__global__ void __launch_bounds__(kPrefixThreads) chunk_total_kernel(Dims d,
                                                                     const Chunk* __restrict__ chunks,
                                                                     const float* __restrict__ x,
                                                                     float* __restrict__ tot) {
  constexpr int kMaxRows = FIX_CHUNK * 128 / kPrefixThreads;
  __shared__ float part[kPrefixThreads];
  const int Dv = d.Dv;
  const int groups = kPrefixThreads / Dv, rows = FIX_CHUNK / groups;
  const int c = threadIdx.x % Dv, grp = threadIdx.x / Dv;
  const int ci = blockIdx.x, kv = blockIdx.y;
  const Chunk ch = chunks[ci];
  const size_t rs = (size_t)d.Hkv * Dv;
  const size_t base = (size_t)ch.tok0 * rs + (size_t)kv * Dv + c;
  const int r0 = grp * rows;
  const int nr = max(0, min(rows, ch.len - r0));
  float xv[kMaxRows];
#pragma unroll
  for (int u = 0; u < kMaxRows; ++u) xv[u] = u < nr ? x[base + (size_t)(r0 + u) * rs] : 0.f;
  float acc = 0.f;
#pragma unroll
  for (int u = 0; u < kMaxRows; ++u) acc += xv[u];
  part[threadIdx.x] = acc;
  __syncthreads();
  if (grp == 0) {
    float t = 0.f;
    for (int q = 0; q < groups; ++q) t += part[q * Dv + c];
    tot[((size_t)ci * d.Hkv + kv) * Dv + c] = t;
  }
}

__global__ void __launch_bounds__(kPrefixThreads) reverse_cumsum_kernel(
    Dims d, const Chunk* __restrict__ chunks, const float* __restrict__ x,
    const float* __restrict__ tot, float* __restrict__ out) {
  constexpr int kMaxRows = FIX_CHUNK * 128 / kPrefixThreads;
  __shared__ float part[kPrefixThreads];
  const int Dv = d.Dv;
  const int groups = kPrefixThreads / Dv, rows = FIX_CHUNK / groups;
  const int c = threadIdx.x % Dv, grp = threadIdx.x / Dv;
  const int ci = blockIdx.x, kv = blockIdx.y;
  const Chunk ch = chunks[ci];
  const size_t rs = (size_t)d.Hkv * Dv;
  const size_t base = (size_t)ch.tok0 * rs + (size_t)kv * Dv + c;
  const int r0 = grp * rows;
  const int nr = max(0, min(rows, ch.len - r0));
  float xv[kMaxRows];
#pragma unroll
  for (int u = 0; u < kMaxRows; ++u) xv[u] = u < nr ? x[base + (size_t)(r0 + u) * rs] : 0.f;
  // the later chunks of the sequence, in order
  float acc = 0.f;
  const int first = ci - ch.j;
  for (int jj = ch.nch - 1; jj > ch.j; --jj) acc += tot[((size_t)(first + jj) * d.Hkv + kv) * Dv + c];
  float own = 0.f;
#pragma unroll
  for (int u = 0; u < kMaxRows; ++u) own += xv[u];
  part[threadIdx.x] = own;
  __syncthreads();
  // then the later row groups of this chunk, from the last one down
  for (int q = groups - 1; q > grp; --q) acc += part[q * Dv + c];
#pragma unroll
  for (int u = kMaxRows - 1; u >= 0; --u)
    if (u < nr) {
      acc += xv[u];
      out[base + (size_t)(r0 + u) * rs] = acc;
    }
}

}  // namespace fix
