// FiX decode: one new query per sequence against the cache of its earlier
// keys, values and gates.
//
// The FiX poster abstract names inference memory as one of the challenges FiX
// addresses; the pages give no decode algorithm, so this is the definition
// evaluated for the last row t = L - 1 of each sequence:
//   o_t[c] = sum_{s<=t} exp(S_ts - m_t) exp(G_t[c] - G_s[c]) v_s[c]
// followed by the same RMSNorm / no-norm output and output gate as the
// forward.  The cache holds k, v and the log forget gates g (element-wise
// [Tmax, Hkv, Dv] or scalar [Tmax, Hkv]) of tokens 0..L-1, the new token's
// included; no cumulative gate is stored, so its precision does not degrade
// with position.
//
// Split over keys (memory bound: every cached byte is read once):
//   decode_partial_kernel, grid (B * Hkv, nsplit): a CTA takes one range of
//     R keys of one kv head, for all q heads of its group, walking the range
//     from its last key backwards so that the decay to the range's last key,
//     exp(sum_{r=s+1..e} g_r), is a running suffix sum (every factor <= 1 for
//     g <= 0).  It writes the range's row maximum m_i and sum l_i per head,
//     its partial o_i[c], and the range's gate total tot_i[c].
//   decode_combine_kernel, one CTA per (sequence, q head): the decay from a
//     range's last key to t is exp(sum of the later ranges' totals); with the
//     maxima M = max m_i: o = sum_i exp(m_i - M) D_i o_i, l = sum_i exp(m_i -
//     M) l_i, then the norm (or o / l) and the gate.
#include "fix_internal.h"

#define FIX_DECODE_TRY(expr)          \
  do {                                \
    fix_status _s = (expr);           \
    if (_s != FIX_OK) return _s;      \
  } while (0)

namespace fix {

constexpr int kDecThreads = 256;
constexpr int kDecTile = 32;      // keys per shared-memory tile

// grid (B * Hkv, nsplit), block 256.  Shared memory: q of the group [grp][Dk],
// one tile of k [32][Dk + 1], v [32][Dv], the tile's decay [32][Dv], the
// logits [grp][32] and the heads' rescale factors [grp].
__global__ void __launch_bounds__(kDecThreads) decode_partial_kernel(
    DecodeDims dd, const int* __restrict__ seqlens, const __nv_bfloat16* __restrict__ q,
    const __nv_bfloat16* __restrict__ kc, const __nv_bfloat16* __restrict__ vc,
    const float* __restrict__ gc, float* __restrict__ part_m, float* __restrict__ part_l,
    float* __restrict__ part_o, float* __restrict__ part_tot) {
  extern __shared__ float sm[];
  const int Dk = dd.Dk, Dv = dd.Dv, grp = dd.grp;
  const int b = blockIdx.x / dd.Hkv, kv = blockIdx.x % dd.Hkv, sp = blockIdx.y;
  float* sq = sm;                              // [grp][Dk]
  float* sk = sq + grp * Dk;                   // [32][Dk + 1]
  float* sv = sk + kDecTile * (Dk + 1);        // [32][Dv]
  float* sdec = sv + kDecTile * Dv;            // [32][Dv]
  float* ss = sdec + kDecTile * Dv;            // [grp][32]
  const int tid = threadIdx.x;
  const int L = min(max(seqlens[b], 0), dd.Tmax);
  const int s0 = sp * dd.R, s1 = min(L, s0 + dd.R);
  const size_t pi = ((size_t)b * dd.Hkv + kv) * dd.nsplit + sp;     // (b, kv, split)
  if (s0 >= s1) {
    // an empty range: contributes nothing
    for (int h = tid; h < grp; h += blockDim.x) {
      part_m[pi * grp + h] = -INFINITY;
      part_l[pi * grp + h] = 0.f;
    }
    for (int e = tid; e < grp * Dv; e += blockDim.x) part_o[pi * grp * Dv + e] = 0.f;
    for (int c = tid; c < Dv; c += blockDim.x) part_tot[pi * Dv + c] = 0.f;
    return;
  }
  const size_t krs = (size_t)dd.Hkv * Dk, vrs = (size_t)dd.Hkv * Dv;
  const size_t tok0 = (size_t)b * dd.Tmax;
  for (int e = tid; e < grp * Dk; e += blockDim.x) {
    const int h = e / Dk, c = e % Dk;
    sq[e] = bf2f(q[((size_t)b * dd.Hq + kv * grp + h) * Dk + c]) * dd.scale;
  }
  // accumulators: thread owns (head, channel) pairs e = tid + 256 i
  constexpr int kMaxPairs = 16 * 128 / kDecThreads;
  float acc[kMaxPairs];
#pragma unroll
  for (int i = 0; i < kMaxPairs; ++i) acc[i] = 0.f;
  float mrun = -INFINITY, lrun = 0.f;     // thread h < grp: its head's running max / sum
  float suf = 0.f;                        // thread c < Dv: sum of g after the current tile
  for (int te = s1; te > s0; te -= kDecTile) {
    const int tb = max(s0, te - kDecTile), nk = te - tb;
    __syncthreads();
    for (int e = tid; e < kDecTile * Dk; e += blockDim.x) {
      const int s = e / Dk, c = e % Dk;
      sk[s * (Dk + 1) + c] = s < nk ? bf2f(kc[(tok0 + tb + s) * krs + (size_t)kv * Dk + c]) : 0.f;
    }
    for (int e = tid; e < kDecTile * Dv; e += blockDim.x) {
      const int s = e / Dv, c = e % Dv;
      sv[e] = s < nk ? bf2f(vc[(tok0 + tb + s) * vrs + (size_t)kv * Dv + c]) : 0.f;
    }
    // decay of each key of the tile to the range's last key, from the running
    // suffix sum of g (keys walked backwards)
    if (tid < Dv) {
      const int c = tid;
      for (int s = nk - 1; s >= 0; --s) {
        sdec[s * Dv + c] = __expf(suf);
        const size_t gi = dd.scalar_gate ? (tok0 + tb + s) * dd.Hkv + kv
                                         : (tok0 + tb + s) * vrs + (size_t)kv * Dv + c;
        suf += gc[gi];
      }
    }
    __syncthreads();
    // logits of the tile for every head of the group
    for (int e = tid; e < grp * kDecTile; e += blockDim.x) {
      const int h = e / kDecTile, s = e % kDecTile;
      float a = -INFINITY;
      if (s < nk) {
        a = 0.f;
        for (int c = 0; c < Dk; ++c) a += sq[h * Dk + c] * sk[s * (Dk + 1) + c];
      }
      ss[e] = a;
    }
    __syncthreads();
    // per head: tile max, rescale factor, P (in place of the logits), sum
    if (tid < grp) {
      const int h = tid;
      float mx = mrun;
      for (int s = 0; s < nk; ++s) mx = fmaxf(mx, ss[h * kDecTile + s]);
      const float alpha = __expf(mrun - mx);   // 0 on the first tile (mrun = -inf)
      float lt = 0.f;
      for (int s = 0; s < kDecTile; ++s) {
        const float p = s < nk ? __expf(ss[h * kDecTile + s] - mx) : 0.f;
        ss[h * kDecTile + s] = p;
        lt += p;
      }
      lrun = lrun * alpha + lt;
      mrun = mx;
      ss[grp * kDecTile + h] = alpha;          // rescale factor for the accumulators
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kMaxPairs; ++i) {
      const int e = tid + kDecThreads * i;
      if (e >= grp * Dv) break;
      const int h = e / Dv, c = e % Dv;
      float a = acc[i] * ss[grp * kDecTile + h];
      for (int s = 0; s < nk; ++s) a += ss[h * kDecTile + s] * sdec[s * Dv + c] * sv[s * Dv + c];
      acc[i] = a;
    }
  }
  for (int i = 0; i < kMaxPairs; ++i) {
    const int e = tid + kDecThreads * i;
    if (e >= grp * Dv) break;
    part_o[pi * grp * Dv + e] = acc[i];
  }
  if (tid < grp) {
    part_m[pi * grp + tid] = mrun;
    part_l[pi * grp + tid] = lrun;
  }
  if (tid < Dv) part_tot[pi * Dv + tid] = suf;
}

// One CTA (128 threads) per (sequence, q head): thread c < Dv owns channel c.
__global__ void __launch_bounds__(128) decode_combine_kernel(
    DecodeDims dd, const float* __restrict__ part_m, const float* __restrict__ part_l,
    const float* __restrict__ part_o, const float* __restrict__ part_tot,
    const __nv_bfloat16* __restrict__ w, const __nv_bfloat16* __restrict__ z, void* __restrict__ y,
    int y_f32) {
  __shared__ float red[4];
  const int b = blockIdx.x / dd.Hq, h = blockIdx.x % dd.Hq, kv = h / dd.grp, hh = h % dd.grp;
  const int c = threadIdx.x, lane = c & 31, warp = c >> 5;
  const size_t pb = ((size_t)b * dd.Hkv + kv) * dd.nsplit;
  float M = -INFINITY;
  for (int i = 0; i < dd.nsplit; ++i) M = fmaxf(M, part_m[(pb + i) * dd.grp + hh]);
  const bool none = M == -INFINITY;              // an empty sequence: y = 0
  // later ranges first: the running total is the decay from range i's last
  // key to the query
  float o = 0.f, l = 0.f, after = 0.f;
  for (int i = dd.nsplit - 1; i >= 0; --i) {
    const float mi = part_m[(pb + i) * dd.grp + hh];
    if (mi == -INFINITY) continue;                 // empty range
    const float a = __expf(mi - M);
    l += a * part_l[(pb + i) * dd.grp + hh];
    if (c < dd.Dv) {
      o += a * __expf(after) * part_o[((pb + i) * dd.grp + hh) * dd.Dv + c];
      after += part_tot[(pb + i) * dd.Dv + c];
    }
  }
  float sq = c < dd.Dv ? o * o : 0.f;
  sq = warp_sum(sq);
  if (lane == 0) red[warp] = sq;
  __syncthreads();
  const float tot = red[0] + red[1] + red[2] + red[3];
  if (c >= dd.Dv) return;
  float yv = dd.no_norm ? o / l : o / sqrtf(tot / (float)dd.Dv + dd.eps) * bf2f(w[c]);
  if (none) yv = 0.f;
  const size_t a0 = ((size_t)b * dd.Hq + h) * dd.Dv + c;
  if (z) yv *= swish(bf2f(z[a0]));
  if (y_f32) reinterpret_cast<float*>(y)[a0] = yv;
  else reinterpret_cast<__nv_bfloat16*>(y)[a0] = f2bf(yv);
}

}  // namespace fix

// ---------------------------------------------------------------- host side

namespace fix {

static size_t decode_smem(const DecodeDims& dd) {
  return sizeof(float) * ((size_t)dd.grp * dd.Dk + kDecTile * (dd.Dk + 1) + 2 * kDecTile * dd.Dv +
                          (size_t)dd.grp * (kDecTile + 1));
}

// Split of the cache into ranges of R keys: about four CTAs per SM of a
// 148-SM B200 over the batch's kv heads, R a multiple of 32 in [64, 4096].
static fix_status decode_dims(const fix_attn_problem* p, DecodeDims* dd) {
  Dims d;
  FIX_DECODE_TRY(validate_problem(p, &d));
  if (p->cu_seqlens || p->num_seqs) return FIX_ERR_CU_SEQLENS;   // lengths come per sequence
  if (d.grp * d.Dv > 2048) return FIX_ERR_GQA;
  dd->B = d.B;
  dd->Tmax = d.T;
  dd->Hq = d.Hq;
  dd->Hkv = d.Hkv;
  dd->Dk = d.Dk;
  dd->Dv = d.Dv;
  dd->grp = d.grp;
  dd->scale = d.scale;
  dd->eps = d.eps;
  dd->no_norm = d.no_norm;
  dd->scalar_gate = d.scalar_gate;
  const long long keys = (long long)d.B * d.Hkv * (d.T > 0 ? d.T : 1);
  long long R = (keys + 4 * 148 - 1) / (4 * 148);
  R = (R + 31) / 32 * 32;
  R = R < 64 ? 64 : (R > 4096 ? 4096 : R);
  dd->R = (int)R;
  dd->nsplit = (int)(((d.T > 0 ? d.T : 1) + R - 1) / R);
  return FIX_OK;
}

struct DecodeWs {
  size_t m, l, o, tot, total;
};

static DecodeWs decode_layout(const DecodeDims& dd) {
  DecodeWs w{};
  const size_t np = (size_t)dd.B * dd.Hkv * dd.nsplit;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = (o + bytes + 255) / 256 * 256;
    return at;
  };
  w.m = take(np * dd.grp * 4);
  w.l = take(np * dd.grp * 4);
  w.o = take(np * dd.grp * dd.Dv * 4);
  w.tot = take(np * dd.Dv * 4);
  w.total = o;
  return w;
}

}  // namespace fix

using namespace fix;

extern "C" size_t fix_attn_decode_workspace_bytes(const fix_attn_problem* p) {
  DecodeDims dd;
  if (decode_dims(p, &dd) != FIX_OK) return 0;
  return decode_layout(dd).total;
}

extern "C" fix_status fix_attn_decode(const fix_attn_problem* p, const int32_t* seqlens,
                                      const void* q, const void* k_cache, const void* v_cache,
                                      const float* g_cache, const void* o_norm_weight,
                                      const void* o_gate, void* y, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  DecodeDims dd;
  FIX_DECODE_TRY(decode_dims(p, &dd));
  if (!seqlens || !q || !k_cache || !v_cache || !g_cache || (!o_norm_weight && !dd.no_norm) ||
      !y || !workspace)
    return FIX_ERR_NULL;
  for (const void* ptr : {(const void*)seqlens, q, k_cache, v_cache, (const void*)g_cache,
                          o_norm_weight, o_gate, (const void*)y, (const void*)workspace})
    if (ptr && (reinterpret_cast<uintptr_t>(ptr) & 15u)) return FIX_ERR_ALIGN;
  const DecodeWs ws = decode_layout(dd);
  if (workspace_bytes < ws.total) return FIX_ERR_WORKSPACE;
  if (dd.B == 0 || dd.Tmax == 0) return FIX_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(workspace);
  const size_t smem = decode_smem(dd);
  if (!set_smem_limit(reinterpret_cast<const void*>(decode_partial_kernel), (int)smem))
    return FIX_ERR_CUDA;
  decode_partial_kernel<<<dim3(dd.B * dd.Hkv, dd.nsplit), kDecThreads, smem, st>>>(
      dd, seqlens, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k_cache),
      static_cast<const __nv_bfloat16*>(v_cache), g_cache, reinterpret_cast<float*>(base + ws.m),
      reinterpret_cast<float*>(base + ws.l), reinterpret_cast<float*>(base + ws.o),
      reinterpret_cast<float*>(base + ws.tot));
  if (cudaGetLastError() != cudaSuccess) return FIX_ERR_CUDA;
  decode_combine_kernel<<<dd.B * dd.Hq, 128, 0, st>>>(
      dd, reinterpret_cast<const float*>(base + ws.m), reinterpret_cast<const float*>(base + ws.l),
      reinterpret_cast<const float*>(base + ws.o), reinterpret_cast<const float*>(base + ws.tot),
      static_cast<const __nv_bfloat16*>(o_norm_weight), static_cast<const __nv_bfloat16*>(o_gate),
      y, p->y_dtype == FIX_DTYPE_F32);
  return launch_status();
}
