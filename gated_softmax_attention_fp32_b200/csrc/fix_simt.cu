// Exact fp32 CUDA-core kernels for FiX attention (FIX_ALGO_SIMT).
//
// Every decay factor exp(G_t[c] - G_s[c]) is formed element by element from
// the chunk-local prefix sums (no factorisation through a reference row), so
// these kernels are slow but follow the definition directly:
//   o_t[c] = sum_{s<=t} exp(S_ts - m_t) exp(G_t[c] - G_s[c]) v_s[c]
// (FiX poster abstract: element-wise forgetting on the values, softmax
// denominator dropped under the RMSNorm).  They are a second GPU path that the
// tensor-core kernels are cross-checked against.
//
// Tiling: a CTA owns 32 rows (query rows for fwd / dq, key rows for dk/dv) of
// one 128-token chunk; keys (or queries) stream through shared memory in
// tiles of 32.  Decay exponents across chunks add the chunk totals between
// the two chunks (see fix_common.cuh).
#include "fix_common.cuh"

namespace fix {

constexpr int ST = 32;          // rows per CTA and per streamed tile
constexpr unsigned FULL = 0xffffffffu;

// ---------------------------------------------------------------------------
// Forward.  grid (nchunks * 4, Hq), block 256 (8 warps x 4 query rows).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) fwd_simt_kernel(
    Dims d, const Chunk* __restrict__ chunks, const __nv_bfloat16* __restrict__ q,
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const float* __restrict__ L, const float* __restrict__ tot,
    const __nv_bfloat16* __restrict__ w, const __nv_bfloat16* __restrict__ z,
    void* __restrict__ y, int y_f32, float* __restrict__ o_s, float* __restrict__ m_s,
    float* __restrict__ rstd_s) {
  extern __shared__ float sm[];
  const int Dk = d.Dk, Dv = d.Dv;
  float* sQ = sm;                       // [ST][Dk]
  float* sLq = sQ + ST * Dk;            // [ST][Dv]
  float* sK = sLq + ST * Dv;            // [ST][Dk+1]
  float* sV = sK + ST * (Dk + 1);       // [ST][Dv]
  float* sLk = sV + ST * Dv;            // [ST][Dv]

  const int ci = blockIdx.x >> 2, r0 = (blockIdx.x & 3) * ST;
  const int h = blockIdx.y, kv = h / d.grp;
  const Chunk ch = chunks[ci];
  if (r0 >= ch.len) return;
  const int nrows = min(ST, ch.len - r0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t qrs = (size_t)d.Hq * Dk, krs = (size_t)d.Hkv * Dk;
  const size_t vrs = (size_t)d.Hkv * Dv, ors = (size_t)d.Hq * Dv;
  const int seq0 = ch.tok0 - ch.j * FIX_CHUNK;
  const int first = ci - ch.j;

  for (int e = threadIdx.x; e < ST * Dk; e += blockDim.x) {
    const int r = e / Dk, dd = e % Dk;
    sQ[e] = r < nrows ? bf2f(q[(size_t)(ch.tok0 + r0 + r) * qrs + (size_t)h * Dk + dd]) : 0.f;
  }
  for (int e = threadIdx.x; e < ST * Dv; e += blockDim.x) {
    const int r = e / Dv, c = e % Dv;
    sLq[e] = r < nrows ? L[(size_t)(ch.tok0 + r0 + r) * vrs + (size_t)kv * Dv + c] : 0.f;
  }

  float o[4][4], mrow[4], lrow[4], delta[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    mrow[a] = -INFINITY;
    lrow[a] = 0.f;
    delta[a] = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) o[a][u] = 0.f;
  }

  for (int jj = ch.j; jj >= 0; --jj) {
    if (jj < ch.j) {  // delta = sum of chunk totals from jj up to (not incl.) this chunk
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = lane + 32 * u;
        if (c < Dv) delta[u] += tot[((size_t)(first + jj) * d.Hkv + kv) * Dv + c];
      }
    }
    const int klen = (jj == ch.j) ? (r0 + nrows) : FIX_CHUNK;
    for (int kt = 0; kt < klen; kt += ST) {
      const int nk = min(ST, klen - kt);
      const int ktok = seq0 + jj * FIX_CHUNK + kt;
      __syncthreads();
      for (int e = threadIdx.x; e < ST * Dk; e += blockDim.x) {
        const int s = e / Dk, dd = e % Dk;
        sK[s * (Dk + 1) + dd] = s < nk ? bf2f(k[(size_t)(ktok + s) * krs + (size_t)kv * Dk + dd]) : 0.f;
      }
      for (int e = threadIdx.x; e < ST * Dv; e += blockDim.x) {
        const int s = e / Dv, c = e % Dv;
        const size_t a = (size_t)(ktok + s) * vrs + (size_t)kv * Dv + c;
        sV[e] = s < nk ? bf2f(v[a]) : 0.f;
        sLk[e] = s < nk ? L[a] : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const int r = warp * 4 + rr;
        if (r >= nrows) break;
        const int tpos = ch.j * FIX_CHUNK + r0 + r;
        const int spos = jj * FIX_CHUNK + kt + lane;
        const bool valid = lane < nk && spos <= tpos;
        float acc = 0.f;
        for (int dd = 0; dd < Dk; ++dd) acc += sQ[r * Dk + dd] * sK[lane * (Dk + 1) + dd];
        const float sv = valid ? acc * d.scale : -INFINITY;
        const float mnew = fmaxf(mrow[rr], warp_max(sv));
        if (mnew == -INFINITY) continue;
        const float alpha = (mrow[rr] == mnew) ? 1.f : expf(mrow[rr] - mnew);
        mrow[rr] = mnew;
        float lq[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          o[rr][u] *= alpha;
          const int c = lane + 32 * u;
          lq[u] = c < Dv ? sLq[r * Dv + c] + delta[u] : 0.f;
        }
        const float p = valid ? expf(sv - mnew) : 0.f;
        lrow[rr] = lrow[rr] * alpha + warp_sum(p);   // softmax denominator (no norm)
        for (int s = 0; s < nk; ++s) {
          const float ps = __shfl_sync(FULL, p, s);
          if (ps == 0.f) continue;  // masked key: its factor may be out of range
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int c = lane + 32 * u;
            if (c < Dv) o[rr][u] += ps * expf(lq[u] - sLk[s * Dv + c]) * sV[s * Dv + c];
          }
        }
      }
    }
  }

#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int r = warp * 4 + rr;
    if (r >= nrows) break;
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) ss += o[rr][u] * o[rr][u];
    ss = warp_sum(ss);
    // RMSNorm, or (no norm) the softmax denominator; the saved tensors are
    // then o / l, the log-sum-exp and ones
    const float rstd = d.no_norm ? 1.f / lrow[rr] : 1.f / sqrtf(ss / (float)Dv + d.eps);
    const size_t tok = (size_t)(ch.tok0 + r0 + r);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = lane + 32 * u;
      if (c >= Dv) continue;
      const size_t a = tok * ors + (size_t)h * Dv + c;
      float yv = o[rr][u] * rstd * (d.no_norm ? 1.f : bf2f(w[c]));
      if (z) yv *= swish(bf2f(z[a]));
      if (y_f32) reinterpret_cast<float*>(y)[a] = yv;
      else reinterpret_cast<__nv_bfloat16*>(y)[a] = f2bf(yv);
      if (o_s) o_s[a] = d.no_norm ? o[rr][u] * rstd : o[rr][u];
    }
    if (lane == 0 && m_s) {
      m_s[tok * d.Hq + h] = d.no_norm ? mrow[rr] + logf(lrow[rr]) : mrow[rr];
      rstd_s[tok * d.Hq + h] = d.no_norm ? 1.f : rstd;
    }
  }
}

// ---------------------------------------------------------------------------
// Backward preprocess (shared by all kernel families).  Pass 1, grid
// (nchunks * kPreSplit, Hkv), 8 warps: a CTA takes half of a chunk's rows
// for one kv head, a warp a row at a time over the kv group's q heads:
//   RMSNorm backward   n = o rstd,  dn = dy w,  do = rstd (dn - n mean(dn n))
//   A_t[c]  = sum_{h in group} do_t[c] (o_t[c] - P_tt v_t[c])
//             the row part of dG_t without the s = t pair, whose counterpart
//             the dk/dv kernels leave out of dv as well, so that
//             dG = A - v dv_strict carries no cancelling diagonal terms
//             (P_tt = exp(S_tt - m_t), S_tt recomputed from q_t, k_t)
//   dw partials        sum_t dy_t n_t per CTA
//   hmax[ci * Hq + h]  max |do| over the chunk (float bits, atomicMax; zeroed
//                      by the prefix pass), only for the tensor-core kernels;
//   ptt[t * Hq + h]    P_tt, for the tensor-core dk/dv combine (optional).
// A warp's (row, q head) items arrive through a ring of kPreStages stages in
// shared memory (cp.async, each lane copying its own 4 channels), so that
// kPreStages - 1 items are in flight beside the one computed without
// holding registers.  Dynamic shared memory: bwd_pre_smem_bytes(grp).
// ---------------------------------------------------------------------------
constexpr int kPreWarps = 8;
constexpr int kPreStages = 4;
// one stage of a warp: q (32 x 8 B), o (32 x 16), dy, z, v, k (32 x 8 each),
// rstd and m (32 x 4 each: every lane copies the row's scalar)
constexpr int kPreStageBytes = 2048;
constexpr int kPsQ = 0, kPsO = 256, kPsDy = 768, kPsZ = 1024, kPsV = 1280, kPsK = 1536,
              kPsRs = 1792, kPsM = 1920;

size_t bwd_pre_smem_bytes(int grp) {
  return (size_t)(grp + 3) / 4 * 16 + (size_t)kPreWarps * grp * 32 * sizeof(float) +
         (size_t)kPreWarps * kPreStages * kPreStageBytes;
}

__global__ void __launch_bounds__(kPreWarps * 32, 3) bwd_pre_kernel(
    Dims d, const Chunk* __restrict__ chunks, const __nv_bfloat16* __restrict__ q,
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const float* __restrict__ o_s, const float* __restrict__ m_s,
    const float* __restrict__ rstd_s, const __nv_bfloat16* __restrict__ dy,
    const __nv_bfloat16* __restrict__ w, const __nv_bfloat16* __restrict__ z,
    __nv_bfloat16* __restrict__ dz, float* __restrict__ do_ws, float* __restrict__ A,
    float* __restrict__ delta_out, float* __restrict__ dwpart, int* __restrict__ hmax_g,
    float* __restrict__ ptt_out) {
  __shared__ float red[kPreWarps][128];
  extern __shared__ __align__(16) float pre_smem[];
  float* hmax = pre_smem;   // [grp] max |do| per head
  // [warps][grp][32] each lane's running max |do| per head, joined once at
  // the end instead of a warp reduction per item
  float* lmax = pre_smem + (d.grp + 3) / 4 * 4 + (size_t)(threadIdx.x >> 5) * d.grp * 32;
  uint8_t* ring = reinterpret_cast<uint8_t*>(pre_smem + (d.grp + 3) / 4 * 4 + kPreWarps * d.grp * 32) +
                  (size_t)(threadIdx.x >> 5) * kPreStages * kPreStageBytes;
  const int Dv = d.Dv, Dk = d.Dk, kv = blockIdx.y;
  const int ci = blockIdx.x / kPreSplit, sub = blockIdx.x % kPreSplit;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Chunk ch = chunks[ci];
  for (int i = threadIdx.x; i < d.grp; i += blockDim.x) hmax[i] = 0.f;
  __syncthreads();
  // lane = 4 consecutive channels (16-byte fp32 / 8-byte bf16 accesses)
  const int c0 = 4 * lane;
  const bool cv = c0 < Dv, ck = c0 < Dk;
  float wv[4], dwl[4];
  ld4b(w && cv ? w + c0 : nullptr, wv);
#pragma unroll
  for (int u = 0; u < 4; ++u) dwl[u] = 0.f;
  const size_t ors = (size_t)d.Hq * Dv, vrs = (size_t)d.Hkv * Dv;
  const size_t qrs = (size_t)d.Hq * Dk, krs = (size_t)d.Hkv * Dk;
  constexpr int kRows = FIX_CHUNK / kPreSplit;
  const int rend = min(ch.len, (sub + 1) * kRows);
  const int r0 = sub * kRows + warp;
  const int nrows = rend > r0 ? (rend - r0 + kPreWarps - 1) / kPreWarps : 0;
  const int grp = d.grp, nitems = nrows * grp;
  // The warp's (row, q head) items in order, through the stage ring.
  struct In {
    float rs, mt, q[4], o[4], dy[4], z[4], vr[4], kr[4];
  };
  auto issue = [&](int it) {
    uint8_t* sb = ring + (it % kPreStages) * kPreStageBytes;
    const int i = it / grp, hh = it % grp;
    const size_t t = (size_t)ch.tok0 + r0 + i * kPreWarps;
    const int h = kv * grp + hh;
    const size_t a = t * ors + (size_t)h * Dv + c0;
    cp_async<4>(sb + kPsRs + lane * 4, rstd_s + t * d.Hq + h, true);
    cp_async<4>(sb + kPsM + lane * 4, m_s + t * d.Hq + h, true);
    cp_async<8>(sb + kPsQ + lane * 8, ck ? q + t * qrs + (size_t)h * Dk + c0 : q, ck);
    cp_async<16>(sb + kPsO + lane * 16, cv ? o_s + a : o_s, cv);
    cp_async<8>(sb + kPsDy + lane * 8, cv ? dy + a : dy, cv);
    if (z) cp_async<8>(sb + kPsZ + lane * 8, cv ? z + a : z, cv);
    if (hh == 0) {
      cp_async<8>(sb + kPsV + lane * 8, cv ? v + t * vrs + (size_t)kv * Dv + c0 : v, cv);
      cp_async<8>(sb + kPsK + lane * 8, ck ? k + t * krs + (size_t)kv * Dk + c0 : k, ck);
    }
  };
  auto unpack_bf4 = [](const uint8_t* p, float* x) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    x[0] = __uint_as_float(u.x << 16);
    x[1] = __uint_as_float(u.x & 0xFFFF0000u);
    x[2] = __uint_as_float(u.y << 16);
    x[3] = __uint_as_float(u.y & 0xFFFF0000u);
  };
  auto fetch = [&](int it, In& in) {
    const uint8_t* sb = ring + (it % kPreStages) * kPreStageBytes;
    const int hh = it % grp;
    in.rs = *reinterpret_cast<const float*>(sb + kPsRs + lane * 4);
    in.mt = *reinterpret_cast<const float*>(sb + kPsM + lane * 4);
    unpack_bf4(sb + kPsQ + lane * 8, in.q);
    const float4 o4 = *reinterpret_cast<const float4*>(sb + kPsO + lane * 16);
    in.o[0] = o4.x;
    in.o[1] = o4.y;
    in.o[2] = o4.z;
    in.o[3] = o4.w;
    unpack_bf4(sb + kPsDy + lane * 8, in.dy);
    if (z) unpack_bf4(sb + kPsZ + lane * 8, in.z);
    else in.z[0] = in.z[1] = in.z[2] = in.z[3] = 0.f;
    if (hh == 0) {
      unpack_bf4(sb + kPsV + lane * 8, in.vr);
      unpack_bf4(sb + kPsK + lane * 8, in.kr);
    }
  };
  float acc[4] = {0.f, 0.f, 0.f, 0.f}, vr[4] = {0.f, 0.f, 0.f, 0.f}, kr[4] = {0.f, 0.f, 0.f, 0.f};
  auto process = [&](int it, const In& cur) {
    const int i = it / grp, hh = it % grp;
    const size_t t = (size_t)ch.tok0 + r0 + i * kPreWarps;
    const int h = kv * grp + hh;
    if (hh == 0) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        vr[u] = cur.vr[u];
        kr[u] = cur.kr[u];
        acc[u] = 0.f;
      }
    }
    float sdot = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) sdot += cur.q[u] * kr[u];
    const float ptt = expf(warp_sum(sdot) * d.scale - cur.mt);
    if (ptt_out && lane == 0) ptt_out[t * d.Hq + h] = ptt;
    // output gate: y = u swish(z) with u the normed (or, without the norm,
    // the averaged) output; du = dy swish(z), dz = dy u swish'(z)
    float du[4], dn[4], n[4], dot_ = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      du[u] = z ? cur.dy[u] * swish(cur.z[u]) : cur.dy[u];
      n[u] = d.no_norm ? cur.o[u] : cur.o[u] * cur.rs;
      dn[u] = d.no_norm ? du[u] : du[u] * wv[u];
      dot_ += dn[u] * n[u];
      if (!d.no_norm) dwl[u] += du[u] * n[u];
    }
    dot_ = warp_sum(dot_) / (float)Dv;
    // without the norm: do = du, and sum_c do o (the softmax-denominator
    // term of dS) goes to the dq and dk/dv kernels
    if (d.no_norm && lane == 0) delta_out[t * d.Hq + h] = dot_ * (float)Dv;
    float dov[4], mx = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      dov[u] = d.no_norm ? du[u] : cur.rs * (dn[u] - n[u] * dot_);
      acc[u] += dov[u] * (cur.o[u] - ptt * vr[u]);
      mx = fmaxf(mx, fabsf(dov[u]));
    }
    if (cv) {
      const size_t a = t * ors + (size_t)h * Dv + c0;
      *reinterpret_cast<float4*>(do_ws + a) = make_float4(dov[0], dov[1], dov[2], dov[3]);
      if (z) {
        float g4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float uo = d.no_norm ? cur.o[u] : n[u] * wv[u];
          g4[u] = cur.dy[u] * uo * swish_grad(cur.z[u]);
        }
        st4b(dz + a, g4);
      }
    }
    if (hmax_g) lmax[hh * 32 + lane] = fmaxf(lmax[hh * 32 + lane], mx);
    if (hh == grp - 1 && cv)
      *reinterpret_cast<float4*>(A + t * vrs + (size_t)kv * Dv + c0) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  };
  if (hmax_g)
    for (int hh = 0; hh < grp; ++hh) lmax[hh * 32 + lane] = 0.f;   // lane-private slots
  // each lane reads back only what it copied itself: its own wait is enough
#pragma unroll
  for (int p = 0; p < kPreStages - 1; ++p) {
    if (p < nitems) issue(p);
    cp_async_commit();
  }
  for (int it = 0; it < nitems; ++it) {
    if (it + kPreStages - 1 < nitems) issue(it + kPreStages - 1);   // over item it - 1's stage
    cp_async_commit();
    cp_async_wait<kPreStages - 1>();
    In cur;
    fetch(it, cur);
    process(it, cur);
  }

  if (hmax_g)
    for (int hh = 0; hh < grp; ++hh) {
      const float mx = warp_max(lmax[hh * 32 + lane]);
      if (lane == 0) atomicMax(reinterpret_cast<int*>(&hmax[hh]), __float_as_int(mx));
    }
#pragma unroll
  for (int u = 0; u < 4; ++u) red[warp][c0 + u] = cv ? dwl[u] : 0.f;
  __syncthreads();
  const int cw = threadIdx.x;
  if (cw < Dv) {
    float sm = 0.f;
#pragma unroll
    for (int i = 0; i < kPreWarps; ++i) sm += red[i][cw];
    dwpart[((size_t)blockIdx.x * d.Hkv + kv) * Dv + cw] = sm;
  }
  if (hmax_g)
    for (int i = threadIdx.x; i < d.grp; i += blockDim.x)
      atomicMax(hmax_g + (size_t)ci * d.Hq + kv * d.grp + i, __float_as_int(hmax[i]));
}

// ---------------------------------------------------------------------------
// Backward preprocess, pass 2 (tensor-core kernels only), grid
// (nchunks * kPreOpsSplit, Hkv): the row-scaled upstream gradients in the two
// references of the forward split, as 16-bit MMA operands:
//   dOt_t = do_t exp(L_t)          (key blocks before the query chunk): fp16
//                                  when dsafe, else bf16
//   dOm_t = do_t exp(L_t - rho)    (the diagonal block; 0 for channels outside
//                                  the split's range): bf16 hi + lo
// with dsafe[ci * Hq + h] = (the chunk is fp16-safe and max |do| <= FIX_F16_VMAX).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kPreWarps * 32) bwd_pre_ops_kernel(
    Dims d, const Chunk* __restrict__ chunks, const float* __restrict__ L,
    const float* __restrict__ rho, const float* __restrict__ hr, const int* __restrict__ safe,
    const float* __restrict__ do_ws, const int* __restrict__ hmax_g, uint16_t* __restrict__ dot,
    __nv_bfloat16* __restrict__ domh, __nv_bfloat16* __restrict__ doml, int* __restrict__ dsafe) {
  const int Dv = d.Dv, kv = blockIdx.y;
  const int ci = blockIdx.x / kPreOpsSplit, sub = blockIdx.x % kPreOpsSplit;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Chunk ch = chunks[ci];
  const bool chunk_safe = safe[(size_t)ci * d.Hkv + kv] != 0;
  if (sub == 0)
    for (int i = threadIdx.x; i < d.grp; i += blockDim.x)
      dsafe[(size_t)ci * d.Hq + kv * d.grp + i] =
          (chunk_safe && __int_as_float(hmax_g[(size_t)ci * d.Hq + kv * d.grp + i]) <= FIX_F16_VMAX) ? 1 : 0;
  const size_t ors = (size_t)d.Hq * Dv, vrs = (size_t)d.Hkv * Dv;
  // lane = 4 consecutive channels
  const int c0 = 4 * lane;
  const bool cv = c0 < Dv;
  const size_t tb = ((size_t)ci * d.Hkv + kv) * Dv + c0;
  float rh[4], hq[4], good[4];
  ld4f(cv ? rho + tb : nullptr, rh);
  ld4f(cv ? hr + tb : nullptr, hq);
#pragma unroll
  for (int u = 0; u < 4; ++u) good[u] = (cv && hq[u] <= FIX_HR_MAX) ? 1.f : 0.f;
  constexpr int kRows = FIX_CHUNK / kPreOpsSplit;
  const int rend = min(ch.len, (sub + 1) * kRows);
  const int r0 = sub * kRows + warp;
  const int nrows = rend > r0 ? (rend - r0 + kPreWarps - 1) / kPreWarps : 0;
  const int grp = d.grp, nitems = nrows * grp;
  // the warp's (row, q head) items, loads issued two items ahead
  struct In {
    float d[4], l[4];
  };
  auto load = [&](int it, In& in) {
    const int i = it / grp, hh = it % grp;
    const size_t t = (size_t)ch.tok0 + r0 + i * kPreWarps;
    ld4f(cv ? do_ws + t * ors + (size_t)(kv * grp + hh) * Dv + c0 : nullptr, in.d);
    if (hh == 0) ld4f(cv ? L + t * vrs + (size_t)kv * Dv + c0 : nullptr, in.l);
  };
  float lr[4] = {0.f, 0.f, 0.f, 0.f};
  auto process = [&](int it, const In& cur) {
    const int i = it / grp, hh = it % grp;
    const size_t t = (size_t)ch.tok0 + r0 + i * kPreWarps;
    const int h = kv * grp + hh;
    if (hh == 0) {
#pragma unroll
      for (int u = 0; u < 4; ++u) lr[u] = cur.l[u];
    }
    const bool f16 = chunk_safe && __int_as_float(hmax_g[(size_t)ci * d.Hq + h]) <= FIX_F16_VMAX;
    if (cv) {
      float xt[4], hi[4], lo[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        xt[u] = cur.d[u] * exp_op(lr[u]);
        const float xm = good[u] != 0.f ? cur.d[u] * exp_op(lr[u] - rh[u]) : 0.f;
        hi[u] = bf2f(f2bf(xm));
        lo[u] = xm - hi[u];
      }
      const size_t a = t * ors + (size_t)h * Dv + c0;
      if (f16) {
        const __half2 x01 = __floats2half2_rn(xt[0], xt[1]), x23 = __floats2half2_rn(xt[2], xt[3]);
        *reinterpret_cast<uint2*>(dot + a) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&x01), *reinterpret_cast<const uint32_t*>(&x23));
      } else {
        st4b(reinterpret_cast<__nv_bfloat16*>(dot + a), xt);
      }
      st4b(domh + a, hi);   // hi is already bf16-exact
      st4b(doml + a, lo);
    }
  };
  // three item buffers used in place (a copy between them would wait for
  // the loads in flight)
  In b0, b1, b2;
  if (nitems > 0) load(0, b0);
  if (nitems > 1) load(1, b1);
  for (int it = 0; it < nitems; it += 3) {
    if (it + 2 < nitems) load(it + 2, b2);
    process(it, b0);
    if (it + 1 >= nitems) break;
    if (it + 3 < nitems) load(it + 3, b0);
    process(it + 1, b1);
    if (it + 2 >= nitems) break;
    if (it + 4 < nitems) load(it + 4, b1);
    process(it + 2, b2);
  }

}

// dw = sum of the partials in a fixed order (deterministic).  grid
// ceil(Dv / 32), block 1024: a CTA takes 32 channels (all of them for Dv <
// 32), its threads interleaved groups of partial rows, then the groups in
// order.
__global__ void __launch_bounds__(1024) dw_reduce_kernel(const float* __restrict__ parts,
                                                         int nparts, int Dv,
                                                         __nv_bfloat16* __restrict__ dw) {
  __shared__ float red[1024];
  const int cw = Dv < 32 ? Dv : 32;
  const int groups = 1024 / cw;
  const int c = blockIdx.x * cw + (int)threadIdx.x % cw, grp = (int)threadIdx.x / cw;
  float s = 0.f;
  if (grp < groups && c < Dv) {
    int i = grp;
    for (; i + 3 * groups < nparts; i += 4 * groups) {
      const float a = parts[(size_t)i * Dv + c], b = parts[(size_t)(i + groups) * Dv + c];
      const float e = parts[(size_t)(i + 2 * groups) * Dv + c];
      const float f = parts[(size_t)(i + 3 * groups) * Dv + c];
      s += a;
      s += b;
      s += e;
      s += f;
    }
    for (; i < nparts; i += groups) s += parts[(size_t)i * Dv + c];
  }
  red[threadIdx.x] = s;
  __syncthreads();
  if ((int)threadIdx.x < cw && c < Dv) {
    float t = 0.f;
    for (int g = 0; g < groups; ++g) t += red[g * cw + threadIdx.x];
    dw[c] = f2bf(t);
  }
}

// ---------------------------------------------------------------------------
// dq.  grid (nchunks * 4, Hq), block 256: 32 query rows per CTA.
//   dP_ts = sum_c do_t[c] exp(G_t[c] - G_s[c]) v_s[c],  dS = P dP,
//   dq_t  = scale sum_s dS_ts k_s
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dq_simt_kernel(
    Dims d, const Chunk* __restrict__ chunks, const __nv_bfloat16* __restrict__ q,
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const float* __restrict__ L, const float* __restrict__ tot,
    const float* __restrict__ m_s, const float* __restrict__ do_ws,
    const float* __restrict__ delta_in, __nv_bfloat16* __restrict__ dq,
    const int* __restrict__ gate) {
  if (gate && *gate == 0) return;  // the tensor-core kernel handles this problem
  extern __shared__ float sm[];
  const int Dk = d.Dk, Dv = d.Dv;
  float* sQ = sm;                        // [ST][Dk]
  float* sDo = sQ + ST * Dk;             // [ST][Dv]
  float* sLq = sDo + ST * Dv;            // [ST][Dv]
  float* sM = sLq + ST * Dv;             // [ST]
  float* sDelta = sM + ST;               // [Dv]
  float* sK = sDelta + Dv;               // [ST][Dk+1]
  float* sV = sK + ST * (Dk + 1);        // [ST][Dv+1]
  float* sLk = sV + ST * (Dv + 1);       // [ST][Dv+1]

  const int ci = blockIdx.x >> 2, r0 = (blockIdx.x & 3) * ST;
  const int h = blockIdx.y, kv = h / d.grp;
  const Chunk ch = chunks[ci];
  if (r0 >= ch.len) return;
  const int nrows = min(ST, ch.len - r0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t qrs = (size_t)d.Hq * Dk, krs = (size_t)d.Hkv * Dk;
  const size_t vrs = (size_t)d.Hkv * Dv, ors = (size_t)d.Hq * Dv;
  const int seq0 = ch.tok0 - ch.j * FIX_CHUNK;
  const int first = ci - ch.j;

  for (int e = threadIdx.x; e < ST * Dk; e += blockDim.x) {
    const int r = e / Dk, dd = e % Dk;
    sQ[e] = r < nrows ? bf2f(q[(size_t)(ch.tok0 + r0 + r) * qrs + (size_t)h * Dk + dd]) : 0.f;
  }
  for (int e = threadIdx.x; e < ST * Dv; e += blockDim.x) {
    const int r = e / Dv, c = e % Dv;
    const size_t tok = (size_t)(ch.tok0 + r0 + r);
    sDo[e] = r < nrows ? do_ws[tok * ors + (size_t)h * Dv + c] : 0.f;
    sLq[e] = r < nrows ? L[tok * vrs + (size_t)kv * Dv + c] : 0.f;
  }
  for (int r = threadIdx.x; r < ST; r += blockDim.x)
    sM[r] = r < nrows ? m_s[(size_t)(ch.tok0 + r0 + r) * d.Hq + h] : 0.f;
  for (int c = threadIdx.x; c < Dv; c += blockDim.x) sDelta[c] = 0.f;

  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[a][u] = 0.f;

  for (int jj = ch.j; jj >= 0; --jj) {
    const int klen = (jj == ch.j) ? (r0 + nrows) : FIX_CHUNK;
    for (int kt = 0; kt < klen; kt += ST) {
      const int nk = min(ST, klen - kt);
      const int ktok = seq0 + jj * FIX_CHUNK + kt;
      __syncthreads();
      if (kt == 0 && jj < ch.j)
        for (int c = threadIdx.x; c < Dv; c += blockDim.x)
          sDelta[c] += tot[((size_t)(first + jj) * d.Hkv + kv) * Dv + c];
      for (int e = threadIdx.x; e < ST * Dk; e += blockDim.x) {
        const int s = e / Dk, dd = e % Dk;
        sK[s * (Dk + 1) + dd] = s < nk ? bf2f(k[(size_t)(ktok + s) * krs + (size_t)kv * Dk + dd]) : 0.f;
      }
      for (int e = threadIdx.x; e < ST * Dv; e += blockDim.x) {
        const int s = e / Dv, c = e % Dv;
        const size_t a = (size_t)(ktok + s) * vrs + (size_t)kv * Dv + c;
        sV[s * (Dv + 1) + c] = s < nk ? bf2f(v[a]) : 0.f;
        sLk[s * (Dv + 1) + c] = s < nk ? L[a] : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const int r = warp * 4 + rr;
        if (r >= nrows) break;
        const int tpos = ch.j * FIX_CHUNK + r0 + r;
        const int spos = jj * FIX_CHUNK + kt + lane;
        const bool valid = lane < nk && spos <= tpos;
        float ds = 0.f;
        if (valid) {
          float sacc = 0.f;
          for (int dd = 0; dd < Dk; ++dd) sacc += sQ[r * Dk + dd] * sK[lane * (Dk + 1) + dd];
          const float p = expf(sacc * d.scale - sM[r]);
          if (p != 0.f) {
            float dp = 0.f;
            for (int c = 0; c < Dv; ++c)
              dp += sDo[r * Dv + c] *
                    expf(sLq[r * Dv + c] + sDelta[c] - sLk[lane * (Dv + 1) + c]) *
                    sV[lane * (Dv + 1) + c];
            // without the norm, dS carries the softmax-denominator term
            if (delta_in) dp -= delta_in[(size_t)(ch.tok0 + r0 + r) * d.Hq + h];
            ds = p * dp;
          }
        }
        for (int s = 0; s < nk; ++s) {
          const float dss = __shfl_sync(FULL, ds, s);
          if (dss == 0.f) continue;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int dd = lane + 32 * u;
            if (dd < Dk) acc[rr][u] += dss * sK[s * (Dk + 1) + dd];
          }
        }
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int r = warp * 4 + rr;
    if (r >= nrows) break;
    const size_t tok = (size_t)(ch.tok0 + r0 + r);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int dd = lane + 32 * u;
      if (dd < Dk) dq[tok * qrs + (size_t)h * Dk + dd] = f2bf(acc[rr][u] * d.scale);
    }
  }
}

// ---------------------------------------------------------------------------
// dk, dv and dG.  grid (nchunks * 4, Hkv), block 256: 32 key rows per CTA,
// 4 per warp, looping over the kv group's q heads and every later query row.
//   dv_s += P_ts D_ts do_t ;  dk_s += scale dS_ts q_t ;
//   dG_s  = A_s - v_s dv_strict_s   (A from bwd_pre_kernel, both without the
//   s = t pair; dv_strict = dv minus that pair's P_ss do_s)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dkv_simt_kernel(
    Dims d, const Chunk* __restrict__ chunks, const __nv_bfloat16* __restrict__ q,
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const float* __restrict__ L, const float* __restrict__ tot,
    const float* __restrict__ m_s, const float* __restrict__ do_ws,
    const float* __restrict__ delta_in, const float* __restrict__ A,
    __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv, float* __restrict__ dG,
    const int* __restrict__ gate) {
  if (gate && *gate == 0) return;  // the tensor-core kernel handles this problem
  extern __shared__ float sm[];
  const int Dk = d.Dk, Dv = d.Dv;
  float* sQ = sm;                        // [ST][Dk]
  float* sDo = sQ + ST * Dk;             // [ST][Dv]
  float* sLq = sDo + ST * Dv;            // [ST][Dv]
  float* sM = sLq + ST * Dv;             // [ST]

  const int ci = blockIdx.x >> 2, r0 = (blockIdx.x & 3) * ST;
  const int kv = blockIdx.y;
  const Chunk ch = chunks[ci];
  if (r0 >= ch.len) return;
  const int nkeys = min(ST, ch.len - r0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t qrs = (size_t)d.Hq * Dk, krs = (size_t)d.Hkv * Dk;
  const size_t vrs = (size_t)d.Hkv * Dv, ors = (size_t)d.Hq * Dv;
  const int first = ci - ch.j;

  float kr[4][4], vr[4][4], lk[4][4], gk[4][4], gv[4][4], gd[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int key = warp * 4 + a;
    const size_t tok = (size_t)(ch.tok0 + r0 + min(key, nkeys - 1));
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int dd = lane + 32 * u;
      kr[a][u] = dd < Dk ? bf2f(k[tok * krs + (size_t)kv * Dk + dd]) : 0.f;
      vr[a][u] = dd < Dv ? bf2f(v[tok * vrs + (size_t)kv * Dv + dd]) : 0.f;
      lk[a][u] = dd < Dv ? L[tok * vrs + (size_t)kv * Dv + dd] : 0.f;
      gk[a][u] = 0.f;
      gv[a][u] = 0.f;
      gd[a][u] = 0.f;
    }
  }

  for (int hh = 0; hh < d.grp; ++hh) {
    const int h = kv * d.grp + hh;
    float delta[4] = {0.f, 0.f, 0.f, 0.f};
    for (int ii = ch.j; ii < ch.nch; ++ii) {
      if (ii > ch.j) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = lane + 32 * u;
          if (c < Dv) delta[u] += tot[((size_t)(first + ii - 1) * d.Hkv + kv) * Dv + c];
        }
      }
      const Chunk qc = chunks[first + ii];
      const int qstart = (ii == ch.j) ? r0 : 0;
      for (int qt = qstart; qt < qc.len; qt += ST) {
        const int nq = min(ST, qc.len - qt);
        __syncthreads();
        for (int e = threadIdx.x; e < ST * Dk; e += blockDim.x) {
          const int r = e / Dk, dd = e % Dk;
          sQ[e] = r < nq ? bf2f(q[(size_t)(qc.tok0 + qt + r) * qrs + (size_t)h * Dk + dd]) : 0.f;
        }
        for (int e = threadIdx.x; e < ST * Dv; e += blockDim.x) {
          const int r = e / Dv, c = e % Dv;
          const size_t tok = (size_t)(qc.tok0 + qt + r);
          sDo[e] = r < nq ? do_ws[tok * ors + (size_t)h * Dv + c] : 0.f;
          sLq[e] = r < nq ? L[tok * vrs + (size_t)kv * Dv + c] : 0.f;
        }
        for (int r = threadIdx.x; r < ST; r += blockDim.x)
          sM[r] = r < nq ? m_s[(size_t)(qc.tok0 + qt + r) * d.Hq + h] : 0.f;
        __syncthreads();
        for (int r = 0; r < nq; ++r) {
          const int tpos = ii * FIX_CHUNK + qt + r;
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            const int key = warp * 4 + a;
            const int spos = ch.j * FIX_CHUNK + r0 + key;
            if (key >= nkeys || spos > tpos) continue;  // warp-uniform
            float sacc = 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int dd = lane + 32 * u;
              if (dd < Dk) sacc += sQ[r * Dk + dd] * kr[a][u];
            }
            sacc = warp_sum(sacc);
            const float p = expf(sacc * d.scale - sM[r]);
            if (p == 0.f) continue;
            float dc[4], dp = 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int c = lane + 32 * u;
              dc[u] = c < Dv ? expf(sLq[r * Dv + c] + delta[u] - lk[a][u]) : 0.f;
              if (c < Dv) dp += sDo[r * Dv + c] * dc[u] * vr[a][u];
            }
            dp = warp_sum(dp);
            // without the norm, dS carries the softmax-denominator term
            if (delta_in) dp -= delta_in[(size_t)(qc.tok0 + qt + r) * d.Hq + h];
            const float ds = p * dp;
            const bool same = spos == tpos;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int dd = lane + 32 * u;
              if (dd < Dk) gk[a][u] += ds * sQ[r * Dk + dd];
              if (dd < Dv) {
                const float x = p * dc[u] * sDo[r * Dv + dd];
                if (same) gd[a][u] += x;
                else gv[a][u] += x;
              }
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int key = warp * 4 + a;
    if (key >= nkeys) break;
    const size_t tok = (size_t)(ch.tok0 + r0 + key);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int dd = lane + 32 * u;
      if (dd < Dk) dk[tok * krs + (size_t)kv * Dk + dd] = f2bf(gk[a][u] * d.scale);
      if (dd < Dv) {
        const size_t av = tok * vrs + (size_t)kv * Dv + dd;
        dv[av] = f2bf(gv[a][u] + gd[a][u]);
        dG[av] = A[av] - vr[a][u] * gv[a][u];
      }
    }
  }
}

}  // namespace fix
