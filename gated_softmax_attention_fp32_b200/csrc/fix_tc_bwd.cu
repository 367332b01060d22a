// FiX attention backward on the tcgen05 tensor cores (sm_100a).
//
// With the row shift m_t held constant (it cancels under the RMSNorm), the
// gradients of o_t[c] = sum_{s<=t} P_ts D_ts[c] v_s[c] are
//   dP_ts = sum_c do_t[c] D_ts[c] v_s[c],   dS_ts = P_ts dP_ts,
//   dq_t  = scale sum_s dS_ts k_s,          dk_s = scale sum_t dS_ts q_t,
//   dv_s  = sum_t P_ts D_ts do_t,           dG_t = A_t - v_t dv_strict_t,
// where A (row part, from the preprocess) and dv_strict both leave out the
// s = t pair.  The FiX README lists the reference's backward as intra-chunk,
// inter-chunk dKV and inter-chunk dQ passes with inter-chunk scaling of dO;
// here two kernels cover every block pair, with the decay split exactly as in
// the forward:
//   * diagonal block (same chunk): reference rho, operands Vm (prefix pass)
//     and dOm = do exp(L_t - rho) (preprocess);
//   * earlier key blocks: reference = the query chunk's start, operands
//     Vt (prefix pass, pre-decayed to the key chunk's end), dOt = do exp(L_t)
//     and the per-pair channel factor f_ij = exp(sum_{j<j'<i} tot_j').
//
// dq kernel (one CTA per 128-row query chunk and q head, key blocks i..0):
//   S = Q K^T and dP = dO V'^T into TMEM, dS = P dP (fp32, then bf16, written
//   over S), dQ += dS K.  V' = Vt f_ij is formed in shared memory per block.
// dk/dv kernel (one CTA per kv head and part of a 128-row key chunk's work:
// either its diagonal query tiles or a run of the 64-row query tiles of later
// chunks, over the group's q heads):
//   S^T = K Q^T, dP^T = V X^T (X = dOt f_ij, or dOm on the diagonal),
//   dV += P^T X, dK += dS^T Q.  On the diagonal, whose terms dominate dv and
//   whose rounding would dominate dG, P and dOm are split into bf16 hi + lo
//   parts (three MMAs, accumulated as dV_d); elsewhere one MMA in fp16 when
//   every gate <= 0 and |v|, |do| <= 3e4, else bf16 (accumulated as dV_o).
//   Each part writes its fp32 dK and dV to a slot; the combine kernel adds a
//   key chunk's slots in order and finishes
//   dv_strict = exp(rho - L_s) dV_d + exp(tot_j - L_s) dV_o,
//   dv = dv_strict + sum_h P_ss do_s, dG = A - v dv_strict, dk = scale dK.
// Channels outside the split's float range (flagged by the prefix pass) have
// no diagonal operands; their diagonal terms are added exactly in fp32: by
// the dq kernel's dS warps into dP, and by dkv_diag_exact_kernel into the
// dk/dv slots.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "fix_internal.h"
#include "fix_sm100.cuh"

namespace fix {
namespace tcb {

using namespace sm100;

constexpr int BN = FIX_CHUNK;   // keys per block / rows per chunk
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;

struct Params {
  Dims d;
  const Chunk* chunks;
  const int* order;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* L;
  const float* tot;
  const float* rho;
  const float* hr;
  const float* lvt;
  const int* safe;
  const int* dsafe;
  const float* m_s;
  const float* do_ws;
  const uint16_t* dot;      // do exp(L_t), fp16 where dsafe else bf16
  const __nv_bfloat16* domh;  // do exp(L_t - rho), hi and lo bf16 parts
  const __nv_bfloat16* doml;
  const float* A;
  const float* ptt;         // P_tt per (token, q head), from the preprocess
  const float* delta;       // without the norm: sum_c do o per (token, q head); else NULL
  const int* badflag;
  const Part* parts;        // dk/dv work split (schedule kernel)
  const int2* cpart;
  int tiles_per_part;
  long long nslots;         // rows of `partial` per kv head, in units of 128-row slots
  float* partial;           // [slot][kv][128 rows][dK | dV] fp32 sums of the dk/dv parts
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dG;
  int* status;
};

// Byte offset of element (row, col) in a 128-byte-swizzled K-major tile of
// `rows` rows whose columns come in 64-wide halves.
__device__ __forceinline__ uint32_t sw_off(int rows, int row, int col) {
  return (uint32_t)((col >> 6) * (rows * 128) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4));
}

// Converts 8 floats to 8 16-bit values (fp16 or bf16) packed in a uint4.
__device__ __forceinline__ uint4 pack8(const float* x, bool f16) {
  uint4 r;
  if (f16) {
    r.x = pack_f16(x[0], x[1]); r.y = pack_f16(x[2], x[3]);
    r.z = pack_f16(x[4], x[5]); r.w = pack_f16(x[6], x[7]);
  } else {
    r.x = pack_bf16(x[0], x[1]); r.y = pack_bf16(x[2], x[3]);
    r.z = pack_bf16(x[4], x[5]); r.w = pack_bf16(x[6], x[7]);
  }
  return r;
}
// Whether 8 scale factors are no larger than 2, so that a packed fp16
// multiply by them cannot overflow.  A factor below fp16's normal range
// (2^-14) loses relative precision or becomes 0, but every value it scales is
// then already below 2^-14 of its undecayed size (absolute error under
// 2^-24 of it).
__device__ __forceinline__ bool f16_factors(const float* f) {
  bool ok = true;
#pragma unroll
  for (int e = 0; e < 8; ++e) ok = ok && f[e] <= 2.f;
  return ok;
}

// Rewrites in place this thread's 16-byte column chunk `col` of rows r0,
// r0 + step, ... (< rows) of a 128-byte-swizzled operand tile, fn(value, row)
// giving the new value: the loads of a batch of rows come before its stores
// (the compiler cannot move a load above a store to the same array).
template <typename Fn>
__device__ __forceinline__ void rewrite_rows(uint8_t* tile, int rows, int r0, int step, int col, Fn fn);

__device__ __forceinline__ void unpack8(uint4 u, bool f16, float* x) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (f16) {
      const float2 ab = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      x[2 * i] = ab.x;
      x[2 * i + 1] = ab.y;
    } else {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

template <typename Fn>
__device__ __forceinline__ void rewrite_rows(uint8_t* tile, int rows, int r0, int step, int col, Fn fn) {
  constexpr int kB = 4;   // rows per batch
#pragma unroll 1
  for (int s0 = r0; s0 < rows; s0 += kB * step) {
    uint4 x[kB];
#pragma unroll
    for (int i = 0; i < kB; ++i) {
      const int r = s0 + i * step;
      if (r < rows) x[i] = *reinterpret_cast<const uint4*>(tile + sw_off(rows, r, col));
    }
#pragma unroll
    for (int i = 0; i < kB; ++i) {
      const int r = s0 + i * step;
      if (r < rows) *reinterpret_cast<uint4*>(tile + sw_off(rows, r, col)) = fn(x[i], r);
    }
  }
}

__device__ __forceinline__ uint4 hmul8(uint4 v, const __half2 (&fh)[4]) {
  uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    __half2 h = __hmul2(*reinterpret_cast<const __half2*>(&w4[u]), fh[u]);
    w4[u] = *reinterpret_cast<uint32_t*>(&h);
  }
  return make_uint4(w4[0], w4[1], w4[2], w4[3]);
}

// =========================================================================== dq

// Named barrier (ids from 1; 0 is __syncthreads).
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Exact diagonal dP terms of out-of-range channels c, which the MMA's dP
// lacks: dP_ts += sum_c do_t[c] exp(L_t[c] - L_s[c]) v_s[c] for keys s <= t,
// in fp32, added in place to the dP columns in TMEM (dp_base: this warp's
// lanes).  As in the forward, the decay goes through the middle rho of each
// 8-key sub-block's range of L: the key factors w_s[c] = exp(rho - L_s[c])
// v_s[c] are formed once per key (a thread per key, into shared memory), the
// row factors do_t[c] exp(L_t[c] - rho) once per row and sub-block.  A
// sub-block whose L spreads more than 88, or a row whose L lies more than 44
// above rho, takes the direct exponential per pair; otherwise no factor and
// no partial product leaves the fp32 range unless the pair's own
// exp(L_t - L_s) does, and an underflowed row factor only drops terms below
// e^-43 of their own size.
// A sub-block whose every L_s exceeds L_t by more than 104 is skipped: each
// of its exponentials is below 2^-150 and flushes to zero (as the direct
// form's would).  Pairs above the diagonal inside a sub-block get finite
// values that the caller's causal selection discards.  Channels go in batches of
// kDqFixBatch.  Called by the 128 dS threads (named barrier 1), thread
// r = row t = key s.  Not inlined: it runs only for chunks holding such
// channels.
constexpr int kDqFixBatch = 16;
struct DqFixSmem {
  float w[kDqFixBatch][BN];        // key factors
  float lb[kDqFixBatch][BN / 8];   // the middle of each sub-block's L
  float sp[kDqFixBatch][BN / 8];   // the sub-block's spread of L
  float lm[kDqFixBatch][BN / 8];   // the sub-block's largest L
  int idx[128];                    // the bad channels, in order
};
template <int DV>
__device__ __noinline__ void dq_bad_terms(uint32_t dp_base, int r, int len, bool row_ok,
                                          const float* Lk, const __nv_bfloat16* vk, size_t vrs,
                                          const float* Lrow, const float* dorow,
                                          const uint32_t* badmask, DqFixSmem* fx) {
  const int lane = r & 31;
  int nb = 0, before = 0;
#pragma unroll
  for (int w = 0; w < DV / 32; ++w) {
    const int n = __popc(badmask[w]);
    if (w < r / 32) before += n;
    nb += n;
  }
  if (r < DV && ((badmask[r / 32] >> lane) & 1u))
    fx->idx[before + __popc(badmask[r / 32] & ((1u << lane) - 1u))] = r;
  const bool kin = r < len;
#pragma unroll 1
  for (int b0 = 0; b0 < nb; b0 += kDqFixBatch) {
    const int nbb = min(kDqFixBatch, nb - b0);
    named_sync(1, 128);   // the list, or the previous batch's readers
    // key side: thread r = key s
#pragma unroll 1
    for (int j = 0; j < nbb; ++j) {
      const int c = fx->idx[b0 + j];
      const float ls = kin ? Lk[(size_t)r * vrs + c] : 0.f;
      const float vs = kin ? bf2f(vk[(size_t)r * vrs + c]) : 0.f;
      float lmax = kin ? ls : -INFINITY, lmin = kin ? ls : INFINITY;
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
        lmin = fminf(lmin, __shfl_xor_sync(0xffffffffu, lmin, o));
      }
      const bool any = lmax >= lmin;   // the sub-block holds a key
      const float lb = any ? 0.5f * (lmax + lmin) : 0.f, spread = any ? lmax - lmin : 0.f;
      fx->w[j][r] = kin && spread <= 88.f ? ex2((lb - ls) * LOG2E) * vs : 0.f;
      if ((lane & 7) == 0) {
        fx->lb[j][r / 8] = lb;
        fx->sp[j][r / 8] = spread;
        fx->lm[j][r / 8] = lmax;
      }
    }
    // row side: thread r = row t
    float dt[kDqFixBatch], lt[kDqFixBatch];
#pragma unroll
    for (int j = 0; j < kDqFixBatch; ++j) {
      const int c = j < nbb ? fx->idx[b0 + j] : 0;
      dt[j] = j < nbb && row_ok ? dorow[c] : 0.f;
      lt[j] = j < nbb ? Lrow[c] : 0.f;
    }
    named_sync(1, 128);
#pragma unroll 1
    for (int c4 = 0; c4 < BN / 32; ++c4) {
      uint32_t xp[32];
      tmem_ld32(dp_base + c4 * 32, xp);
      tmem_wait_ld(xp);
#pragma unroll
      for (int j = 0; j < kDqFixBatch; ++j) {
        if (j >= nbb || !row_ok) continue;
#pragma unroll
        for (int sb = 0; sb < 4; ++sb) {
          const int blk = c4 * 4 + sb, b = blk * 8;
          if (b > r) continue;   // every key of the sub-block lies above the diagonal
          if (lt[j] - fx->lm[j][blk] < -104.f) continue;   // every term flushes to zero
          const float lbv = fx->lb[j][blk];
          if (fx->sp[j][blk] <= 88.f && lt[j] - lbv <= 44.f) {
            const float a = dt[j] * ex2((lt[j] - lbv) * LOG2E);
            const float4 w0 = *reinterpret_cast<const float4*>(&fx->w[j][b]);
            const float4 w1 = *reinterpret_cast<const float4*>(&fx->w[j][b + 4]);
            const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e)
              xp[sb * 8 + e] = __float_as_uint(fmaf(a, wv[e], __uint_as_float(xp[sb * 8 + e])));
          } else {
            const int c = fx->idx[b0 + j];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int key = b + e;
              if (key <= r && key < len) {
                const float f = ex2((lt[j] - Lk[(size_t)key * vrs + c]) * LOG2E);
                xp[sb * 8 + e] = __float_as_uint(__uint_as_float(xp[sb * 8 + e]) +
                                                 dt[j] * f * bf2f(vk[(size_t)key * vrs + c]));
              }
            }
          }
        }
      }
      tmem_st32(dp_base + c4 * 32, xp);
    }
    tmem_wait_st();
  }
}


struct DqBars {
  uint64_t q_full, o_full, o_ready;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2], v_ready[2];
  uint64_t s_full, ds_ready, dp0_done, done, drain;
};

template <int DK, int DV>
struct DqLayout {
  static constexpr int kQ = 0;                       // [128][DK] bf16
  static constexpr int kO = kQ + BN * DK * 2;        // [128][DV] dO operand
  static constexpr int kK = kO + BN * DV * 2;        // 2 x [128][DK]
  static constexpr int kV = kK + 2 * BN * DK * 2;    // 2 x [128][DV]
  static constexpr int kBars = kV + 2 * BN * DV * 2;
  static constexpr int kTmem = kBars + (int)sizeof(DqBars);
  static constexpr int kAbort = kTmem + 4;
  static constexpr int kFix = (kAbort + 4 + 15) / 16 * 16;   // DqFixSmem
  static constexpr int kAlloc = kFix + (int)sizeof(DqFixSmem) + 1024;
  static_assert(kAlloc <= 232448, "shared memory");
};

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
    dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_vt, const __grid_constant__ CUtensorMap tm_vm,
                 const __grid_constant__ CUtensorMap tm_domh, const __grid_constant__ CUtensorMap tm_dot,
                 const Params P) {
  using Lay = DqLayout<DK, DV>;
  // channels of this chunk outside the split's range (bit c of word c / 32):
  // their diagonal terms are missing from the MMA's dP and are added exactly
  __shared__ uint32_t sBadMask[4];
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const Dims& d = P.d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ci = P.order[blockIdx.x / d.Hq];
  const int h = blockIdx.x % d.Hq, kv = h / d.grp;
  const Chunk ch = P.chunks[ci];
  if (ch.len <= 0) return;
  const int nblk = ch.j + 1, first = ci - ch.j, seq0 = ch.tok0 - ch.j * FIX_CHUNK;

  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem + Lay::kQ);
  uint8_t* sO = smem + Lay::kO;
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem + Lay::kK);
  __nv_bfloat16* sV = reinterpret_cast<__nv_bfloat16*>(smem + Lay::kV);
  DqBars* bar = reinterpret_cast<DqBars*>(smem + Lay::kBars);
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + Lay::kTmem);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + Lay::kAbort);
  const Ctl ctl{P.status, sAbort};

  if (tid == 0) {
    *sAbort = 0;
    mbar_init(&bar->q_full, 1);
    mbar_init(&bar->o_full, 1);
    mbar_init(&bar->o_ready, 128);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
      mbar_init(&bar->v_ready[s], 128);
    }
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->ds_ready, 128);
    mbar_init(&bar->dp0_done, 1);
    mbar_init(&bar->done, 1);
    mbar_init(&bar->drain, 1);
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(sTmem, kTmemCols);
  if (warp < 4) {
    const int c = tid;
    const bool bad = c < DV && *P.badflag != 0 &&
                     P.hr[((size_t)ci * d.Hkv + kv) * DV + c] > FIX_HR_MAX;
    const uint32_t m = __ballot_sync(0xffffffffu, bad);
    if (lane == 0) sBadMask[warp] = m;
  }
  bool my_safe = true;
  for (int jj = tid; jj < nblk; jj += blockDim.x)
    my_safe = my_safe && P.safe[(size_t)(first + jj) * d.Hkv + kv];
  if (tid == 0) my_safe = my_safe && P.dsafe[(size_t)ci * d.Hq + h];
  tc_fence_before();
  const int cta_f16 = __syncthreads_and(my_safe);
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  // TMEM: S (then dS over its first half) double-buffered at 0 and 384, so
  // that the next block's QK^T runs while the dS warps work on this one;
  // dP at 128, the dQ accumulator at 256
  constexpr uint32_t kColP = 128, kColQ = 256;
  auto col_sb = [](int it) -> uint32_t { return (it & 1) ? 384u : 0u; };
  static_assert(256 + DK <= 384, "TMEM columns");

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_expect_tx(&bar->q_full, BN * DK * 2);
      for (int hh = 0; hh < DK / 64; ++hh)
        tma_load_3d(sQ + hh * BN * 64, &tm_q, &bar->q_full, hh * 64, h, ch.tok0);
      // dO operand: dOm (diagonal block) first, dOt once the first dP is done
      mbar_expect_tx(&bar->o_full, BN * DV * 2);
      for (int hh = 0; hh < DV / 64; ++hh)
        tma_load_3d(sO + hh * BN * 128, &tm_domh, &bar->o_full, hh * 64, h, ch.tok0);
      int nk = 0, nv = 0, no = 1;
      for (int it = 0; it < nblk; ++it) {
        const int st = it & 1;
        const uint32_t ph = (it >> 1) & 1;
        const int ktok = seq0 + (ch.j - it) * FIX_CHUNK;
        if (it >= 2 && !mbar_wait(&bar->k_empty[st], ph ^ 1, ctl)) break;
        mbar_expect_tx(&bar->k_full[st], BN * DK * 2);
        for (int hh = 0; hh < DK / 64; ++hh)
          tma_load_3d(sK + st * BN * DK + hh * BN * 64, &tm_k, &bar->k_full[st], hh * 64, kv, ktok);
        ++nk;
        if (it >= 2 && !mbar_wait(&bar->v_empty[st], ph ^ 1, ctl)) break;
        mbar_expect_tx(&bar->v_full[st], BN * DV * 2);
        const CUtensorMap* vmap = it == 0 ? &tm_vm : &tm_vt;
        for (int hh = 0; hh < DV / 64; ++hh)
          tma_load_3d(sV + st * BN * DV + hh * BN * 64, vmap, &bar->v_full[st], hh * 64, kv, ktok);
        ++nv;
        if (it == 1) {
          if (!mbar_wait(&bar->dp0_done, 0, ctl)) break;
          mbar_expect_tx(&bar->o_full, BN * DV * 2);
          for (int hh = 0; hh < DV / 64; ++hh)
            tma_load_3d(sO + hh * BN * 128, &tm_dot, &bar->o_full, hh * 64, h, ch.tok0);
          ++no;
        }
      }
      const Ctl drain{P.status, nullptr};
      for (int it = nk - 1; it >= 0 && it >= nk - 2; --it)
        mbar_wait(&bar->k_full[it & 1], (it >> 1) & 1, drain);
      for (int it = nv - 1; it >= 0 && it >= nv - 2; --it)
        mbar_wait(&bar->v_full[it & 1], (it >> 1) & 1, drain);
      mbar_wait(&bar->q_full, 0, drain);
      mbar_wait(&bar->o_full, (no - 1) & 1, drain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, BN, false, false);
      const uint32_t idesc_dp0 = idesc_bf16(128, BN, false, false);
      const uint32_t idesc_dp = idesc_bf16(128, BN, false, false, cta_f16 != 0);
      constexpr uint32_t idesc_dq = idesc_bf16(128, DK, false, true);
      const uint32_t q_addr = smem_u32(sQ), o_addr = smem_u32(sO);
      // S of block it + 1 (QK^T, into the other S buffer) is issued right
      // after dP of block it, so that it runs while the dS warps work
      auto issue_s = [&](int it) {
        const uint32_t k_addr = smem_u32(sK + (it & 1) * BN * DK);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
          mma_ss(tmem + col_sb(it), desc_add(desc_sw128(q_addr, 16, 1024), off),
                 desc_add(desc_sw128(k_addr, 16, 1024), off), idesc_s, kk > 0);
        }
      };
      bool ok = mbar_wait(&bar->q_full, 0, ctl) && mbar_wait(&bar->o_ready, 0, ctl);
      if (ok && nblk > 0) {
        ok = mbar_wait(&bar->k_full[0], 0, ctl);
        if (ok) {
          tc_fence_after();
          issue_s(0);
        }
      }
      for (int it = 0; ok && it < nblk; ++it) {
        const int st = it & 1;
        const uint32_t ph = (it >> 1) & 1;
        if (!mbar_wait(&bar->v_ready[st], ph, ctl)) break;
        if (it == 1 && !mbar_wait(&bar->o_ready, 1, ctl)) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + st * BN * DK), v_addr = smem_u32(sV + st * BN * DV);
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
          mma_ss(tmem + kColP, desc_add(desc_sw128(o_addr, 16, 1024), off), desc_add(desc_sw128(v_addr, 16, 1024), off),
                 it == 0 ? idesc_dp0 : idesc_dp, kk > 0);
        }
        tc_commit(&bar->s_full);   // S (issued before) and dP of block it
        if (it == 0) tc_commit(&bar->dp0_done);
        if (it + 1 < nblk) {
          // its K stage was released by block it - 1's dQ MMAs, issued before
          if (!mbar_wait(&bar->k_full[(it + 1) & 1], ((it + 1) >> 1) & 1, ctl)) break;
          tc_fence_after();
          issue_s(it + 1);
        }
        if (!mbar_wait(&bar->ds_ready, it & 1, ctl)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t b = desc_add(desc_sw128(k_addr, BN * 128, 1024), kk * 2048);
          mma_ts(tmem + kColQ, tmem + col_sb(it) + kk * 8, b, idesc_dq, (it > 0 || kk > 0));
        }
        tc_commit(&bar->k_empty[st]);
        tc_commit(&bar->v_empty[st]);
      }
      tc_commit(&bar->done);
      tc_commit(&bar->drain);
      mbar_wait(&bar->drain, 0, Ctl{P.status, nullptr});
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ dS + epilogue
    const int r = (warp - 4) * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)((warp - 4) * 32) << 16);
    const bool row_ok = r < ch.len;
    const size_t tok = (size_t)ch.tok0 + (size_t)(row_ok ? r : 0);
    const float moff = P.m_s[tok * d.Hq + h] * LOG2E;
    const float c1 = d.scale * LOG2E;
    // without the norm: dS = P (dP - sum_c do o) (the softmax denominator)
    const float dl = P.delta ? P.delta[tok * d.Hq + h] : 0.f;
    const bool any_bad = (sBadMask[0] | sBadMask[1] | sBadMask[2] | sBadMask[3]) != 0;
    const size_t vrs = (size_t)d.Hkv * DV;
    bool ok = true;
    for (int it = 0; it < nblk; ++it) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bar->s_full, it & 1, ctl))) { ok = false; break; }
      tc_fence_after();
      if (it == 0 && any_bad)
        dq_bad_terms<DV>(lane_base + kColP, r, ch.len, row_ok,
                         P.L + (size_t)ch.tok0 * vrs + (size_t)kv * DV,
                         P.v + (size_t)ch.tok0 * vrs + (size_t)kv * DV, vrs,
                         P.L + tok * vrs + (size_t)kv * DV,
                         P.do_ws + tok * (size_t)d.Hq * DV + (size_t)h * DV, sBadMask,
                         reinterpret_cast<DqFixSmem*>(smem + Lay::kFix));
#pragma unroll
      for (int c4 = 0; c4 < BN / 32; ++c4) {
        uint32_t xs[32], xp[32], pk[16];
        tmem_ld32(lane_base + col_sb(it) + c4 * 32, xs);
        tmem_ld32(lane_base + kColP + c4 * 32, xp);
        tmem_wait_ld();
        // rows past the chunk's end only feed dQ rows that are never stored;
        // only the diagonal block needs the causal mask (keys s <= t)
        if (it > 0) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float p0 = ex2(__uint_as_float(xs[e]) * c1 - moff);
            const float p1 = ex2(__uint_as_float(xs[e + 1]) * c1 - moff);
            pk[e >> 1] = pack_bf16(p0 * (__uint_as_float(xp[e]) - dl), p1 * (__uint_as_float(xp[e + 1]) - dl));
          }
        } else {
          // masked by selection: above the diagonal dOm Vm pairs
          // exp(L_t - rho) with exp(rho - L_s) for s > t and may overflow
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int key = c4 * 32 + e;
            const float d0 = key <= r ? ex2(__uint_as_float(xs[e]) * c1 - moff) * (__uint_as_float(xp[e]) - dl) : 0.f;
            const float d1 = key + 1 <= r ? ex2(__uint_as_float(xs[e + 1]) * c1 - moff) * (__uint_as_float(xp[e + 1]) - dl) : 0.f;
            pk[e >> 1] = pack_bf16(d0, d1);
          }
        }
        tmem_st16(lane_base + col_sb(it) + c4 * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar->ds_ready);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar->done, 0, ctl));
    tc_fence_after();
    float acc[DK];
#pragma unroll
    for (int cc = 0; cc < DK / 32; ++cc) {
      uint32_t x[32];
      tmem_ld32(lane_base + kColQ + cc * 32, x);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) acc[cc * 32 + e] = __uint_as_float(x[e]) * d.scale;
    }
    if (ok && row_ok) {
      __nv_bfloat16* dqp = P.dq + tok * (size_t)d.Hq * DK + (size_t)h * DK;
#pragma unroll
      for (int c = 0; c < DK; c += 8) {
        uint4 pkd;
        pkd.x = pack_bf16(acc[c], acc[c + 1]);
        pkd.y = pack_bf16(acc[c + 2], acc[c + 3]);
        pkd.z = pack_bf16(acc[c + 4], acc[c + 5]);
        pkd.w = pack_bf16(acc[c + 6], acc[c + 7]);
        *reinterpret_cast<uint4*>(dqp + c) = pkd;
      }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ operands in smem
    const int dt = tid - 256;
    constexpr int kChunks = DV / 8;
    constexpr int kRowsPerPass = 128 / kChunks;
    const int lc = dt % kChunks, r0 = dt / kChunks;
    // dO operand (loaded by TMA): dOm (bf16) for the diagonal block, then dOt,
    // converted in place when its storage type differs from the CTA's
    for (int phase = 0; phase < (nblk > 1 ? 2 : 1); ++phase) {
      if (!mbar_wait(&bar->o_full, phase, ctl)) break;
      if (phase == 1) {
        const bool stored_f16 = P.dsafe[(size_t)ci * d.Hq + h] != 0;
        if (stored_f16 != (cta_f16 != 0)) {
          rewrite_rows(sO, BN, r0, kRowsPerPass, lc * 8, [&](uint4 v, int) {
            float x[8];
            unpack8(v, stored_f16, x);
            return pack8(x, cta_f16 != 0);
          });
          fence_proxy_async_smem();
        }
      }
      mbar_arrive(&bar->o_ready);
      if (phase == 0) {
        // the diagonal block's V (Vm) goes to the MMA as loaded
        if (!mbar_wait(&bar->v_full[0], 0, ctl)) break;
        mbar_arrive(&bar->v_ready[0]);
      }
    }
    // V' = Vt f_ij for the earlier key blocks
    float delta[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) delta[e] = 0.f;
    for (int it = 1; it < nblk; ++it) {
      const int st = it & 1, j = ch.j - it;
      if (it >= 2) {
        const float* tp = P.tot + ((size_t)(first + j + 1) * d.Hkv + kv) * DV + lc * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) delta[e] += tp[e];
      }
      // Vt is stored as fp16 times 2^-e per channel (prefix pass)
      const float* lv = P.lvt + ((size_t)(first + j) * d.Hkv + kv) * DV + lc * 8;
      float f8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) f8[e] = ex2(delta[e] * LOG2E + vt_exponent(lv[e]));
      if (!mbar_wait(&bar->v_full[st], (it >> 1) & 1, ctl)) break;
      uint8_t* vb = reinterpret_cast<uint8_t*>(sV + st * BN * DV);
      if (cta_f16 && f16_factors(f8)) {
        // fp16 in and out: packed multiplies, no conversions
        __half2 fh[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) fh[u] = __floats2half2_rn(f8[2 * u], f8[2 * u + 1]);
        rewrite_rows(vb, BN, r0, kRowsPerPass, lc * 8, [&](uint4 v, int) { return hmul8(v, fh); });
      } else {
        rewrite_rows(vb, BN, r0, kRowsPerPass, lc * 8, [&](uint4 v, int) {
          float x[8];
          unpack8(v, true, x);
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] *= f8[e];
          return pack8(x, cta_f16);
        });
      }
      fence_proxy_async_smem();
      mbar_arrive(&bar->v_ready[st]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ========================================================================= dk/dv

constexpr int BQ = 64;         // query rows per streamed tile
constexpr int kQStages = 4;    // Q / X tiles in flight (later-block parts; diagonal parts: 2)

struct KvBars {
  uint64_t kv_full;
  uint64_t q_full[kQStages], q_empty[kQStages], x_ready[kQStages];
  uint64_t s_full[2], p_ready[2], done, drain;
};

// The stage region holds kQStages stages of [Q | X] for later-block parts, or
// two stages of [Q | X | X_lo] for diagonal parts (the smaller of the two).
template <int DK, int DV>
struct KvLayout {
  static constexpr int kK = 0;                              // [128][DK]
  static constexpr int kV = kK + BN * DK * 2;               // [128][DV] Vm (diagonal) or Vt
  static constexpr int kQ = kV + BN * DV * 2;               // stage region
  static constexpr int kStageOff = BQ * (DK + DV) * 2;      // bytes per later-block stage
  static constexpr int kStageDiag = BQ * (DK + 2 * DV) * 2; // bytes per diagonal stage
  static constexpr int kM = kQ + kQStages * kStageOff;      // stages x [64] f32 row max x log2(e)
  static_assert(2 * kStageDiag <= kQStages * kStageOff, "diagonal stages must fit the region");
  static constexpr int kDl = kM + kQStages * BQ * 4;        // stages x [64] f32 sum do o
  static constexpr int kBars = kDl + kQStages * BQ * 4;
  static constexpr int kTmem = kBars + (int)sizeof(KvBars);
  static constexpr int kAbort = kTmem + 4;
  static constexpr int kAlloc = kAbort + 4 + 1024;
};

// A dk/dv CTA streams the tiles of one kind: the diagonal ones (query chunk
// i = j) or the later ones (i > j); in order, for each q head of the group,
// for each query chunk, the 64-row halves that hold rows.
struct TileIter {
  int hh, i, half;
};

// One CTA per (part, kv head).  TMEM: S^T and dP^T double-buffered (128
// columns per buffer: S [0, 64), dP [64, 128)), the dV accumulator at 256 and
// dK at 256 + DV.  The MMA warp issues S / dP of tile n + 2 right after dV /
// dK of tile n, so the softmax of one buffer overlaps the MMAs of the other.
template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
    dkv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_vt, const __grid_constant__ CUtensorMap tm_vm,
                  const __grid_constant__ CUtensorMap tm_domh, const __grid_constant__ CUtensorMap tm_doml,
                  const __grid_constant__ CUtensorMap tm_dot, const Params P) {
  using Lay = KvLayout<DK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const Dims& d = P.d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Part pt = P.parts[blockIdx.x / d.Hkv];
  const int kv = blockIdx.x % d.Hkv;
  const int cj = pt.ci;
  const Chunk ch = P.chunks[cj];
  const bool dmode = pt.diag != 0;
  const int first = cj - ch.j;
  auto chunk_len = [&](int i) { return P.chunks[first + i].len; };
  const int i0 = dmode ? ch.j : ch.j + 1, i1 = dmode ? ch.j + 1 : ch.nch;   // query chunks
  int tiles_per_head = 0;
  for (int i = i0; i < i1; ++i) tiles_per_head += (chunk_len(i) + BQ - 1) / BQ;
  const int t_begin = pt.p * P.tiles_per_part;
  const int ntiles = ch.len > 0 ? min(P.tiles_per_part, tiles_per_head * d.grp - t_begin) : 0;
  constexpr int kCols = DK + DV;
  if (ntiles <= 0) {
    // nothing to stream (only for a chunk table that disagrees with the
    // host's plan): the slot still has to read as zero
    if (pt.slot >= 0 && pt.slot < P.nslots) {
      float* dst = P.partial + ((size_t)pt.slot * d.Hkv + kv) * BN * kCols;
      for (int i = tid; i < BN * kCols; i += blockDim.x) dst[i] = 0.f;
    }
    return;
  }

  uint8_t* sK = smem + Lay::kK;
  uint8_t* sV = smem + Lay::kV;
  // stage st: Q at sQ(st), X right after it, X_lo (diagonal) after X
  const int nst = dmode ? 2 : kQStages, lgst = dmode ? 1 : 2;
  const int stage_bytes = dmode ? Lay::kStageDiag : Lay::kStageOff;
  auto sQ = [&](int st) { return smem + Lay::kQ + st * stage_bytes; };
  auto sX = [&](int st) { return sQ(st) + BQ * DK * 2; };
  auto sXl = [&](int st) { return sX(st) + BQ * DV * 2; };
  float* sM = reinterpret_cast<float*>(smem + Lay::kM);
  float* sDl = reinterpret_cast<float*>(smem + Lay::kDl);
  KvBars* bar = reinterpret_cast<KvBars*>(smem + Lay::kBars);
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + Lay::kTmem);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + Lay::kAbort);
  const Ctl ctl{P.status, sAbort};

  if (tid == 0) {
    *sAbort = 0;
    mbar_init(&bar->kv_full, 1);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&bar->q_full[s], 1);
      mbar_init(&bar->q_empty[s], 1);
      mbar_init(&bar->x_ready[s], 128);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar->s_full[b], 1);
      mbar_init(&bar->p_ready[b], 128);
    }
    mbar_init(&bar->done, 1);
    mbar_init(&bar->drain, 1);
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(sTmem, kTmemCols);
  // operand type of the later-block MMAs: fp16 when every chunk they span is
  // fp16-safe for this kv head and its q heads (the diagonal ones are bf16)
  bool my_safe = !dmode;
  if (!dmode)
    for (int i = tid; i < ch.nch - ch.j; i += blockDim.x) {
      my_safe = my_safe && P.safe[(size_t)(first + ch.j + i) * d.Hkv + kv];
      for (int hh = 0; hh < d.grp; ++hh)
        my_safe = my_safe && P.dsafe[(size_t)(first + ch.j + i) * d.Hq + kv * d.grp + hh];
    }
  tc_fence_before();
  const int cta_f16 = __syncthreads_and(my_safe);
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  constexpr uint32_t kColV = 256, kColK = 256 + DV;
  static_assert(256 + DV + DK <= (int)kTmemCols, "TMEM columns");
  auto col_s = [](int b) { return (uint32_t)(b * 128); };
  auto col_p = [](int b) { return (uint32_t)(b * 128 + 64); };

  // walk the tile sequence (identical in every role)
  auto next_tile = [&](TileIter& t) {
    ++t.half;
    if (t.half * BQ >= chunk_len(t.i)) {
      t.half = 0;
      if (++t.i >= i1) {
        t.i = i0;
        ++t.hh;
      }
    }
  };
  auto tile_at = [&](int n) {
    TileIter t{0, i0, 0};
    for (int q = 0; q < n; ++q) next_tile(t);
    return t;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_expect_tx(&bar->kv_full, BN * DK * 2 + BN * DV * 2);
      for (int hh = 0; hh < DK / 64; ++hh)
        tma_load_3d(sK + hh * BN * 128, &tm_k, &bar->kv_full, hh * 64, kv, ch.tok0);
      for (int hh = 0; hh < DV / 64; ++hh)
        tma_load_3d(sV + hh * BN * 128, dmode ? &tm_vm : &tm_vt, &bar->kv_full, hh * 64, kv, ch.tok0);
      TileIter t = tile_at(t_begin);
      int nq = 0;
      for (int n = 0; n < ntiles; ++n, next_tile(t)) {
        const int st = n & (nst - 1);
        if (n >= nst && !mbar_wait(&bar->q_empty[st], ((n >> lgst) & 1) ^ 1, ctl)) break;
        // Q tile and the X operand (dOm hi + lo on the diagonal, dOt elsewhere)
        mbar_expect_tx(&bar->q_full[st], BQ * DK * 2 + (dmode ? 2 : 1) * BQ * DV * 2);
        const int h = kv * d.grp + t.hh;
        const int qtok = P.chunks[first + t.i].tok0 + t.half * BQ;
        for (int hh = 0; hh < DK / 64; ++hh)
          tma_load_3d(sQ(st) + hh * BQ * 128, &tm_q, &bar->q_full[st], hh * 64, h, qtok);
        for (int hh = 0; hh < DV / 64; ++hh) {
          tma_load_3d(sX(st) + hh * BQ * 128, dmode ? &tm_domh : &tm_dot, &bar->q_full[st], hh * 64,
                      h, qtok);
          if (dmode)
            tma_load_3d(sXl(st) + hh * BQ * 128, &tm_doml, &bar->q_full[st], hh * 64, h, qtok);
        }
        ++nq;
      }
      const Ctl drain{P.status, nullptr};
      for (int n = nq - 1; n >= 0 && n >= nq - nst; --n)
        mbar_wait(&bar->q_full[n & (nst - 1)], (n >> lgst) & 1, drain);
      mbar_wait(&bar->kv_full, 0, drain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, BQ, false, false);
      const uint32_t idesc_dp = idesc_bf16(128, BQ, false, false, cta_f16 != 0);
      const uint32_t idesc_dv = idesc_bf16(128, DV, false, true, cta_f16 != 0);
      constexpr uint32_t idesc_dk = idesc_bf16(128, DK, false, true);
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      bool ok = mbar_wait(&bar->kv_full, 0, ctl);
      // the operand warps may convert V in place after kv_full; every
      // x_ready covers their writes
      auto issue_sdp = [&](int n) -> bool {
        const int st = n & (nst - 1), b = n & 1;
        const uint32_t ph = (n >> lgst) & 1;
        // the operand warps arrive on x_ready only after they saw q_full, so
        // x_ready covers the TMA copies of the stage as well
        if (!mbar_wait(&bar->x_ready[st], ph, ctl)) return false;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sQ(st));
        const uint32_t x_addr = smem_u32(sX(st));
        // S^T = K Q^T   (M = 128 keys, N = 64 queries, K = DK)
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint32_t ka = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
          const uint32_t qa = (kk >> 2) * (BQ * 128) + (kk & 3) * 32;
          mma_ss(tmem + col_s(b), desc_add(desc_sw128(k_addr, 16, 1024), ka), desc_add(desc_sw128(q_addr, 16, 1024), qa),
                 idesc_s, kk > 0);
        }
        // dP^T = V X^T
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk) {
          const uint32_t vo = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
          const uint32_t xo = (kk >> 2) * (BQ * 128) + (kk & 3) * 32;
          mma_ss(tmem + col_p(b), desc_add(desc_sw128(v_addr, 16, 1024), vo), desc_add(desc_sw128(x_addr, 16, 1024), xo),
                 idesc_dp, kk > 0);
        }
        tc_commit(&bar->s_full[b]);
        return true;
      };
      if (ok) ok = issue_sdp(0);
      if (ok && ntiles > 1) ok = issue_sdp(1);
      for (int n = 0; ok && n < ntiles; ++n) {
        const int st = n & (nst - 1), b = n & 1;
        if (!mbar_wait(&bar->p_ready[b], (n >> 1) & 1, ctl)) break;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sQ(st));
        const uint32_t x_addr = smem_u32(sX(st));
        const uint32_t xl_addr = smem_u32(sXl(st));
        // dV += P^T X  (K = 64 queries; X read MN-major); on the diagonal
        // P_hi X_hi + P_lo X_hi + P_hi X_lo
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk) {
          const uint64_t bx = desc_add(desc_sw128(x_addr, BQ * 128, 1024), kk * 2048);
          mma_ts(tmem + kColV, tmem + col_s(b) + kk * 8, bx, idesc_dv, !(n == 0 && kk == 0));
          if (dmode) {
            const uint64_t bxl = desc_add(desc_sw128(xl_addr, BQ * 128, 1024), kk * 2048);
            mma_ts(tmem + kColV, tmem + col_s(b) + 32 + kk * 8, bx, idesc_dv, 1);
            mma_ts(tmem + kColV, tmem + col_s(b) + kk * 8, bxl, idesc_dv, 1);
          }
        }
        // dK += dS^T Q
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk) {
          const uint64_t bq = desc_add(desc_sw128(q_addr, BQ * 128, 1024), kk * 2048);
          mma_ts(tmem + kColK, tmem + col_p(b) + kk * 8, bq, idesc_dk, !(n == 0 && kk == 0));
        }
        tc_commit(&bar->q_empty[st]);
        // tile n + 2 reuses buffer b: its MMAs run after the ones above
        if (n + 2 < ntiles) ok = issue_sdp(n + 2);
      }
      tc_commit(&bar->done);
      tc_commit(&bar->drain);
      mbar_wait(&bar->drain, 0, Ctl{P.status, nullptr});
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ P, dS + epilogue
    const int s = (warp - 4) * 32 + lane;            // key row in the chunk
    const uint32_t lane_base = tmem + ((uint32_t)((warp - 4) * 32) << 16);
    const float c1 = d.scale * LOG2E;
    bool ok = true;
    TileIter t = tile_at(t_begin);
    for (int n = 0; n < ntiles; ++n, next_tile(t)) {
      const int st = n & (nst - 1), b = n & 1;
      const int qlen = min(BQ, chunk_len(t.i) - t.half * BQ);
      // x_ready covers the row maxima of this tile in sM
      if (!__all_sync(0xffffffffu, mbar_wait(&bar->s_full[b], (n >> 1) & 1, ctl) &&
                                       mbar_wait(&bar->x_ready[st], (n >> lgst) & 1, ctl))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* mrow = sM + st * BQ;       // row maxima times log2(e)
      const float* dlrow = sDl + st * BQ;     // zeros with the norm
      const bool full = !dmode && qlen == BQ;
      const int lo = dmode ? s - t.half * BQ : 0;   // first valid query column
      // two halves of 32 query columns; a half's packed P and dS go over
      // columns of S and dP that the half has already read
      uint32_t pl[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t xs[32], xp[32], ph[16], pd[16];
        tmem_ld32(lane_base + col_s(b) + 32 * h, xs);
        tmem_ld32(lane_base + col_p(b) + 32 * h, xp);
        tmem_wait_ld();
        if (full) {
          // full later tile: no masking
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float p0 = ex2(fmaf(__uint_as_float(xs[e]), c1, -mrow[32 * h + e]));
            const float p1 = ex2(fmaf(__uint_as_float(xs[e + 1]), c1, -mrow[32 * h + e + 1]));
            ph[e >> 1] = cta_f16 ? pack_f16(p0, p1) : pack_bf16(p0, p1);
            pd[e >> 1] = pack_bf16(p0 * (__uint_as_float(xp[e]) - dlrow[32 * h + e]),
                                   p1 * (__uint_as_float(xp[e + 1]) - dlrow[32 * h + e + 1]));
          }
        } else {
          // diagonal tile (queries t >= s; the s = t pair stays out of dv) or
          // a partial tile (columns past the chunk's end)
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float p[2], pv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int qi = 32 * h + e + u;
              const bool valid = qi >= lo && qi < qlen;
              p[u] = valid ? ex2(fmaf(__uint_as_float(xs[e + u]), c1, -mrow[qi])) : 0.f;
              pv[u] = (dmode && qi == lo) ? 0.f : p[u];
            }
            if (dmode) {
              ph[e >> 1] = pack_bf16(pv[0], pv[1]);
              const float h0 = __uint_as_float(ph[e >> 1] << 16);
              const float h1 = __uint_as_float(ph[e >> 1] & 0xFFFF0000u);
              pl[16 * h + (e >> 1)] = pack_bf16(pv[0] - h0, pv[1] - h1);
            } else {
              ph[e >> 1] = cta_f16 ? pack_f16(pv[0], pv[1]) : pack_bf16(pv[0], pv[1]);
            }
            // masked by selection (dP^T above the diagonal may overflow)
            const float d0 = 32 * h + e >= lo && 32 * h + e < qlen
                                 ? p[0] * (__uint_as_float(xp[e]) - dlrow[32 * h + e]) : 0.f;
            const float d1 = 32 * h + e + 1 >= lo && 32 * h + e + 1 < qlen
                                 ? p[1] * (__uint_as_float(xp[e + 1]) - dlrow[32 * h + e + 1]) : 0.f;
            pd[e >> 1] = pack_bf16(d0, d1);
          }
        }
        tmem_st16(lane_base + col_s(b) + 16 * h, ph);
        tmem_st16(lane_base + col_p(b) + 16 * h, pd);
      }
      // the low parts go over S columns [32, 64), read by the second half
      if (dmode) tmem_st32(lane_base + col_s(b) + 32, pl);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar->p_ready[b]);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar->done, 0, ctl));
    tc_fence_after();
    // ---------------------------------------------------------- epilogue
    // The CTA's raw sums (dK | dV, fp32, a row per key) go to its slot of the
    // partial buffer; the combine kernel adds the slots of a key chunk in
    // order and finishes dk, dv and dG.  Each thread stages its row, one
    // segment at a time, in the operand buffers (free once every MMA has
    // completed) and sends it with its own bulk copy.  Staged rows are padded
    // by 16 bytes so that eight consecutive rows start on distinct banks.
    constexpr int kPad0 = DK + 4, kPad1 = DV + 4;     // staged row strides, floats
    static_assert(BN * (kPad0 + kPad1) * 4 <= Lay::kM, "staging buffers must fit");
    if (ok && pt.slot >= 0 && pt.slot < P.nslots) {
      float* grow = P.partial + (((size_t)pt.slot * d.Hkv + kv) * BN + s) * kCols;
      float* b0 = reinterpret_cast<float*>(smem) + (size_t)s * kPad0;
      float* b1 = reinterpret_cast<float*>(smem) + (size_t)BN * kPad0 + (size_t)s * kPad1;
      auto stage32 = [&](float* dst, const uint32_t (&x)[32]) {
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + e) =
              make_float4(__uint_as_float(x[e]), __uint_as_float(x[e + 1]),
                          __uint_as_float(x[e + 2]), __uint_as_float(x[e + 3]));
      };
#pragma unroll
      for (int cc = 0; cc < DK / 32; ++cc) {
        uint32_t x[32];
        tmem_ld32(lane_base + kColK + cc * 32, x);
        tmem_wait_ld();
        stage32(b0 + cc * 32, x);
      }
      fence_proxy_async_smem();
      bulk_store(grow, b0, DK * 4);
      bulk_commit();
#pragma unroll
      for (int cc = 0; cc < DV / 32; ++cc) {
        uint32_t x[32];
        tmem_ld32(lane_base + kColV + cc * 32, x);
        tmem_wait_ld();
        stage32(b1 + cc * 32, x);
      }
      fence_proxy_async_smem();
      bulk_store(grow + DK, b1, DV * 4);
      bulk_commit();
      bulk_wait_read<0>();
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ X operand tiles
    const int dt = tid - 256;
    constexpr int kChunks = DV / 8;
    constexpr int kRowsPerPass = 128 / kChunks;
    const int lc = dt % kChunks, r0 = dt / kChunks;
    if (!mbar_wait(&bar->kv_full, 0, ctl)) {
      // aborted: fall through to the teardown
    } else {
      if (!dmode) {
        // Vt arrives as fp16 times 2^-e per channel; the later-block MMAs read
        // it unscaled in the CTA's operand type, so this thread rewrites its
        // channels once if either differs
        const float* lv = P.lvt + ((size_t)cj * d.Hkv + kv) * DV + lc * 8;
        float sc[8];
        bool unit = true;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float ve = vt_exponent(lv[e]);
          sc[e] = exp2f(ve);
          unit = unit && ve == 0.f;
        }
        if (!unit || !cta_f16) {
          rewrite_rows(sV, BN, r0, kRowsPerPass, lc * 8, [&](uint4 v, int) {
            float x[8];
            unpack8(v, true, x);
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] *= sc[e];
            return pack8(x, cta_f16 != 0);
          });
        }
        fence_proxy_async_smem();
      }
      // Per tile: the row maxima into sM and, for later blocks, X = dOt f_ij
      // with f_ij = exp(sum_{j<j'<i} tot_j').  The global values a tile needs
      // (its row maxima and the totals that extend the running sum) are
      // loaded one tile ahead, so that x_ready follows q_full closely.
      TileIter t = tile_at(t_begin);
      // what a tile needs from global memory besides its totals
      struct Pre {
        float m;     // row maximum of query row dt (dt < 64)
        float dl;    // its sum_c do o (without the norm; else 0)
        int qlen;    // rows of the tile
        int in_f16;  // storage type of its dOt
      };
      auto fetch = [&](const TileIter& u) {
        const Chunk qc = P.chunks[first + u.i];
        Pre r;
        r.qlen = min(BQ, qc.len - u.half * BQ);
        const size_t ri = ((size_t)qc.tok0 + u.half * BQ + dt) * d.Hq + kv * d.grp + u.hh;
        r.m = dt < r.qlen ? P.m_s[ri] : 0.f;
        r.dl = (dt < r.qlen && P.delta) ? P.delta[ri] : 0.f;
        r.in_f16 = dmode ? 0 : P.dsafe[(size_t)(first + u.i) * d.Hq + kv * d.grp + u.hh];
        return r;
      };
      // sum of tot over query chunks [a, b) for this thread's 8 channels
      auto tot_sum = [&](int a, int b, float* acc) {
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        for (int i = a; i < b; ++i) {
          const float* tp = P.tot + ((size_t)(first + i) * d.Hkv + kv) * DV + lc * 8;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] += tp[e];
        }
      };
      float delta[8];
      if (!dmode) tot_sum(ch.j + 1, t.i, delta);
      Pre cur = fetch(t);
      for (int n = 0; n < ntiles; ++n) {
        const int st = n & (nst - 1);
        float f8[8];
        if (!dmode) {
#pragma unroll
          for (int e = 0; e < 8; ++e) f8[e] = ex2(delta[e] * LOG2E);
        }
        // prefetch for tile n + 1
        TileIter u = t;
        next_tile(u);
        const bool more = n + 1 < ntiles;
        const Pre nxt = more ? fetch(u) : cur;
        float add[8];
        const bool new_head = u.hh != t.hh;
        if (!dmode) tot_sum(t.i, (more && !new_head) ? u.i : t.i, add);
        if (!mbar_wait(&bar->q_full[st], (n >> lgst) & 1, ctl)) break;
        const int qlen = cur.qlen;
        if (!dmode) {
          // X = dOt f_ij, in the CTA's operand type; rows past the chunk's end
          // are zeroed
          const bool in_f16 = cur.in_f16 != 0;
          uint8_t* xb = sX(st);
          if (in_f16 && cta_f16 && f16_factors(f8)) {
            // fp16 in and out: packed multiplies, no conversions
            __half2 fh[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) fh[u] = __floats2half2_rn(f8[2 * u], f8[2 * u + 1]);
            rewrite_rows(xb, BQ, r0, kRowsPerPass, lc * 8, [&](uint4 v, int rr) {
              return rr < qlen ? hmul8(v, fh) : make_uint4(0u, 0u, 0u, 0u);
            });
          } else {
            rewrite_rows(xb, BQ, r0, kRowsPerPass, lc * 8, [&](uint4 v, int rr) {
              float x[8];
              unpack8(v, in_f16, x);
#pragma unroll
              for (int e = 0; e < 8; ++e) x[e] = rr < qlen ? x[e] * f8[e] : 0.f;
              return pack8(x, cta_f16 != 0);
            });
          }
          fence_proxy_async_smem();
        }
        if (dt < BQ) {
          sM[st * BQ + dt] = cur.m * LOG2E;   // in log2 units, as the exponentials take it
          sDl[st * BQ + dt] = cur.dl;
        }
        mbar_arrive(&bar->x_ready[st]);
        // advance to tile n + 1
        if (!dmode) {
#pragma unroll
          for (int e = 0; e < 8; ++e) delta[e] = new_head ? 0.f : delta[e] + add[e];
        }
        cur = nxt;
        t = u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// V consecutive floats (V = 2 or 4) from a 4V-byte aligned address.
template <int V>
__device__ __forceinline__ void ldf(const float* p, float* x) {
  if constexpr (V == 4) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  } else {
    const float2 a = *reinterpret_cast<const float2*>(p);
    x[0] = a.x; x[1] = a.y;
  }
}
template <int V>
__device__ __forceinline__ void stf(float* p, const float* x) {
  if constexpr (V == 4) *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  else *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
}
template <int V>
__device__ __forceinline__ void ldb(const __nv_bfloat16* p, float* x) {
  if constexpr (V == 4) {
    const uint2 a = *reinterpret_cast<const uint2*>(p);
    x[0] = __uint_as_float(a.x << 16); x[1] = __uint_as_float(a.x & 0xFFFF0000u);
    x[2] = __uint_as_float(a.y << 16); x[3] = __uint_as_float(a.y & 0xFFFF0000u);
  } else {
    const uint32_t a = *reinterpret_cast<const uint32_t*>(p);
    x[0] = __uint_as_float(a << 16); x[1] = __uint_as_float(a & 0xFFFF0000u);
  }
}
template <int V>
__device__ __forceinline__ void stb(__nv_bfloat16* p, const float* x) {
  if constexpr (V == 4) *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]));
  else *reinterpret_cast<uint32_t*>(p) = pack_bf16(x[0], x[1]);
}

// Sums the partial rows of key chunks split over several CTAs (in slot
// order, so the result does not depend on scheduling) and finishes dv, dG,
// dk.  grid (nchunks * BN / 8, Hkv), block 256: a warp per key row, lanes
// over channels, so that every row of every array is read and written in
// one coalesced stretch.
template <int DK, int DV>
__global__ void __launch_bounds__(256) dkv_combine_kernel(const Params P) {
  const Dims& d = P.d;
  constexpr int kRowBlocks = BN / 8;
  const int ci = blockIdx.x / kRowBlocks, kv = blockIdx.y, lane = threadIdx.x & 31;
  const int s = (blockIdx.x % kRowBlocks) * 8 + (threadIdx.x >> 5);
  const int2 cp = P.cpart[ci];
  if (cp.x < 1 || cp.y < 0 || cp.y + cp.x > P.nslots) return;
  const Chunk ch = P.chunks[ci];
  if (s >= ch.len) return;
  const size_t tok = (size_t)ch.tok0 + s;
  constexpr int kCols = DK + DV;
  constexpr int VK = DK / 32, VV = DV / 32;            // channels per lane
  const int ck = lane * VK, cv = lane * VV;
  // the chunk's first nd slots hold its diagonal parts (dV_d), the rest its
  // later-block parts (dV_o)
  const int halves = (ch.len + BQ - 1) / BQ;
  const int nd = (d.grp * halves + P.tiles_per_part - 1) / P.tiles_per_part;
  float fk[VK] = {}, fd[VV] = {}, fo[VV] = {};
  // slots four at a time: a batch's loads in flight together, the sums in
  // slot order
  constexpr int kSB = 4;
  for (int q0 = 0; q0 < cp.x; q0 += kSB) {
    float a[kSB][VK], b[kSB][VV];
#pragma unroll
    for (int i = 0; i < kSB; ++i) {
      if (q0 + i < cp.x) {
        const float* prow = P.partial + (((size_t)(cp.y + q0 + i) * d.Hkv + kv) * BN + s) * kCols;
        ldf<VK>(prow + ck, a[i]);
        ldf<VV>(prow + DK + cv, b[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < kSB; ++i) {
      const int q = q0 + i;
      if (q >= cp.x) break;
#pragma unroll
      for (int e = 0; e < VK; ++e) fk[e] += a[i][e];
      if (q < nd) {
#pragma unroll
        for (int e = 0; e < VV; ++e) fd[e] += b[i][e];
      } else {
#pragma unroll
        for (int e = 0; e < VV; ++e) fo[e] += b[i][e];
      }
    }
  }
  // dk = scale * sum dS^T Q
  const size_t krs = (size_t)d.Hkv * DK;
#pragma unroll
  for (int e = 0; e < VK; ++e) fk[e] *= d.scale;
  stb<VK>(P.dk + tok * krs + (size_t)kv * DK + ck, fk);
  // the s = t terms: P_ss (one per q head of the group, as the preprocess
  // used it in A) times do_s
  const size_t vrs = (size_t)d.Hkv * DV, ors = (size_t)d.Hq * DV;
  float diag[VV] = {};
  for (int hh = 0; hh < d.grp; ++hh) {
    const int h = kv * d.grp + hh;
    const float pss = P.ptt[tok * d.Hq + h];
    float dw[VV];
    ldf<VV>(P.do_ws + tok * ors + (size_t)h * DV + cv, dw);
#pragma unroll
    for (int e = 0; e < VV; ++e) diag[e] += pss * dw[e];
  }
  // dv_strict = exp(rho - L_s) dV_d + exp(tot - L_s) dV_o (dV_d of a channel
  // outside the split's range is already exact: factor 1);
  // dv = dv_strict + the s = t terms, dG = A - v dv_strict
  const size_t cb = ((size_t)ci * d.Hkv + kv) * DV + cv, rb = tok * vrs + (size_t)kv * DV + cv;
  const bool has_off = ch.nch - ch.j > 1;
  float ls[VV], rh[VV], hr[VV], tt[VV], av[VV], vv[VV];
  ldf<VV>(P.L + rb, ls);
  ldf<VV>(P.rho + cb, rh);
  ldf<VV>(P.hr + cb, hr);
  ldf<VV>(P.tot + cb, tt);
  ldf<VV>(P.A + rb, av);
  ldb<VV>(P.v + rb, vv);
  float dvv[VV], dgv[VV];
#pragma unroll
  for (int e = 0; e < VV; ++e) {
    float strict = hr[e] > FIX_HR_MAX ? fd[e] : fd[e] * ex2((rh[e] - ls[e]) * LOG2E);
    if (has_off) strict += fo[e] * ex2((tt[e] - ls[e]) * LOG2E);
    dvv[e] = strict + diag[e];
    dgv[e] = av[e] - vv[e] * strict;
  }
  stb<VV>(P.dv + rb, dvv);
  stf<VV>(P.dG + rb, dgv);
}

// ======================================================= out-of-range channels
// A channel whose in-chunk range exceeds the split's float range (hr > 80 or
// |rho| > 80) has Vm = 0 and dOm = 0 on the diagonal block, so the dk/dv
// kernel's diagonal parts leave out its terms:
//   dP_ts  gains  sum_{c bad} do_t[c] exp(L_t[c] - L_s[c]) v_s[c]   (s <= t),
//   so dK_s gains sum_t P_ts dP^bad_ts q_t,  and
//   dv_s[c] (c bad) gets its diagonal part sum_{t > s} P_ts exp(L_t[c] - L_s[c]) do_t[c].
// This kernel adds them, in fp32 on the CUDA cores, to the first diagonal
// slot of the key chunk (its dV columns of bad channels hold exact zeros,
// and the combine takes them unscaled).  One CTA per (chunk, kv head); CTAs
// of chunks without such a channel return at once.  P is recomputed from q,
// k and the saved row maxima as in the tensor-core kernels.
// The decay goes through the middle f of each aligned group of 8 rows' (or
// keys') range of L: exp(L_t - L_s) = u'_t exp(f(t) - f(s)) w'_s with
// u'_t = exp(L_t - f(t)) and w'_s = exp(f(s) - L_s), one exponential per
// index and channel, staged with do and v folded in, and one per pair of
// groups.  Where either group's L spreads more than kFixSpread, or the
// middle rises by more than kFixRise from the key group to the row group,
// the pairs take the direct exponential.  Within those bounds no
// factor and no partial product leaves the fp32 range unless the pair's own
// exp(L_t - L_s) does, and an underflowed group factor only drops terms
// below e^-27 of their own size.  A pair of groups whose every L_t lies more
// than 104 below every L_s is skipped: each of its exponentials is below
// 2^-150 and flushes to zero (as the direct form's would).
constexpr int kFixThreads = 256;
constexpr int kFixBatch = 8;      // bad channels staged per pass
constexpr float kFixSpread = 60.f;
constexpr float kFixRise = 28.f;

template <int DK, int DV>
struct FixLayout {
  static constexpr int kPs = BN + 4;                          // sP row stride (floats)
  static constexpr int kQt = 0;                               // [DK][BN] f32, q transposed
  static constexpr int kKt = kQt + DK * BN * 4;               // [DK][BN] f32, k transposed
  static constexpr int kP = kKt + DK * BN * 4;                // [BN][kPs] f32: P, then dS^bad
  static constexpr int kL = kP + BN * kPs * 4;                // [kFixBatch][BN] L of the batch
  static constexpr int kV = kL + kFixBatch * BN * 4;          // [kFixBatch][BN] v
  static constexpr int kDo = kV + kFixBatch * BN * 4;         // [kFixBatch][BN] do (one head)
  static constexpr int kU = kDo + kFixBatch * BN * 4;         // [kFixBatch][BN] u' do
  static constexpr int kWp = kU + kFixBatch * BN * 4;         // [kFixBatch][BN] w'
  static constexpr int kLg = kWp + kFixBatch * BN * 4;        // [kFixBatch][BN / 8] the middle of each group's L
  static constexpr int kSp = kLg + kFixBatch * (BN / 8) * 4;  // [kFixBatch][BN / 8] the group's spread of L
  static constexpr int kLx = kSp + kFixBatch * (BN / 8) * 4;  // [kFixBatch][BN / 8] the group's largest L
  static constexpr int kLn = kLx + kFixBatch * (BN / 8) * 4;  // [kFixBatch][BN / 8] its smallest L
  static constexpr int kM = kLn + kFixBatch * (BN / 8) * 4;   // [BN] row maxima (one head)
  static constexpr int kIdx = kM + BN * 4;                    // [DV] bad channel list
  static constexpr int kBytes = kIdx + DV * 4 + 16;
  static_assert(kBytes <= 232448, "shared memory");
};

template <int DK, int DV>
__global__ void __launch_bounds__(kFixThreads, 1) dkv_diag_exact_kernel(const Params P) {
  using Lay = FixLayout<DK, DV>;
  if (*P.badflag == 0) return;
  extern __shared__ __align__(16) uint8_t fsm[];
  const Dims& d = P.d;
  const int ci = blockIdx.x, kv = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Chunk ch = P.chunks[ci];
  const int n = ch.len;
  const int2 cp = P.cpart[ci];
  if (n <= 0 || cp.x < 1 || cp.y < 0 || cp.y >= P.nslots) return;
  float* sQt = reinterpret_cast<float*>(fsm + Lay::kQt);
  float* sKt = reinterpret_cast<float*>(fsm + Lay::kKt);
  float* sP = reinterpret_cast<float*>(fsm + Lay::kP);
  float* sL = reinterpret_cast<float*>(fsm + Lay::kL);
  float* sV = reinterpret_cast<float*>(fsm + Lay::kV);
  float* sDo = reinterpret_cast<float*>(fsm + Lay::kDo);
  float* sU = reinterpret_cast<float*>(fsm + Lay::kU);
  float* sWp = reinterpret_cast<float*>(fsm + Lay::kWp);
  float* sLg = reinterpret_cast<float*>(fsm + Lay::kLg);
  float* sSp = reinterpret_cast<float*>(fsm + Lay::kSp);
  float* sLx = reinterpret_cast<float*>(fsm + Lay::kLx);
  float* sLn = reinterpret_cast<float*>(fsm + Lay::kLn);
  float* sM = reinterpret_cast<float*>(fsm + Lay::kM);
  int* sIdx = reinterpret_cast<int*>(fsm + Lay::kIdx);
  int* sNb = sIdx + DV;
  uint32_t* sMask = reinterpret_cast<uint32_t*>(sNb + 1);
  // the chunk's bad channels, in channel order
  if (warp < 4) {
    const int c = tid;
    const bool bad = c < DV && P.hr[((size_t)ci * d.Hkv + kv) * DV + c] > FIX_HR_MAX;
    const uint32_t m = __ballot_sync(0xffffffffu, bad);
    if (lane == 0) sMask[warp] = m;
  }
  __syncthreads();
  if (tid == 0) {
    int nb = 0;
    for (int w = 0; w < DV / 32; ++w)
      for (uint32_t m = sMask[w]; m; m &= m - 1) sIdx[nb++] = w * 32 + __ffs(m) - 1;
    *sNb = nb;
  }
  __syncthreads();
  const int nbad = *sNb;
  if (nbad == 0) return;

  const size_t qrs = (size_t)d.Hq * DK, krs = (size_t)d.Hkv * DK;
  const size_t vrs = (size_t)d.Hkv * DV, ors = (size_t)d.Hq * DV;
  const size_t tok0 = (size_t)ch.tok0;
  // k of the chunk, transposed (rows past its end are zero)
  for (int i = tid; i < BN * DK; i += kFixThreads) {
    const int r = i / DK, c = i % DK;
    sKt[c * BN + r] = r < n ? bf2f(P.k[(tok0 + r) * krs + (size_t)kv * DK + c]) : 0.f;
  }
  // dK accumulator: keys 4 sq .. 4 sq + 3, columns cb * CK .. + CK
  constexpr int CK = DK / 8;
  const int sq = tid % 32, cb = tid / 32;
  float dk[4][CK];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int e = 0; e < CK; ++e) dk[a][e] = 0.f;
  // P / dS block of this thread: rows 8 tb .. + 7, keys 8 sb .. + 7
  const int tb = tid / 16, sb = tid % 16;
  // dv of a batch: key s_dv, batch channels 4 cg .. 4 cg + 3
  const int s_dv = tid % BN, cg = tid / BN;
  const int t_dv = s_dv & ~31;               // first query row of the warp's keys
  const float c1 = d.scale * LOG2E;
  float* slot = P.partial + ((size_t)cp.y * d.Hkv + kv) * BN * (DK + DV);

  for (int hh = 0; hh < d.grp; ++hh) {
    const int h = kv * d.grp + hh;
    __syncthreads();
    for (int i = tid; i < BN * DK; i += kFixThreads) {
      const int r = i / DK, c = i % DK;
      sQt[c * BN + r] = r < n ? bf2f(P.q[(tok0 + r) * qrs + (size_t)h * DK + c]) : 0.f;
    }
    for (int r = tid; r < BN; r += kFixThreads) sM[r] = r < n ? P.m_s[(tok0 + r) * d.Hq + h] : 0.f;
    __syncthreads();
    // P_ts for s <= t < n, else 0
    {
      float acc[8][8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
      if (sb <= tb) {
#pragma unroll 2
        for (int c = 0; c < DK; ++c) {
          const float4 q0 = *reinterpret_cast<const float4*>(sQt + c * BN + 8 * tb);
          const float4 q1 = *reinterpret_cast<const float4*>(sQt + c * BN + 8 * tb + 4);
          const float4 k0 = *reinterpret_cast<const float4*>(sKt + c * BN + 8 * sb);
          const float4 k1 = *reinterpret_cast<const float4*>(sKt + c * BN + 8 * sb + 4);
          const float qa[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
          const float ka[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
          for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(qa[i], ka[j], acc[i][j]);
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int t = 8 * tb + i;
        const float mo = sM[t] * LOG2E;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int sk = 8 * sb + j;
          sP[t * Lay::kPs + sk] = (sk <= t && t < n) ? ex2(acc[i][j] * c1 - mo) : 0.f;
        }
      }
    }
    // dP^bad over all bad channels, batch by batch
    float dp[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) dp[i][j] = 0.f;
    for (int b0 = 0; b0 < nbad; b0 += kFixBatch) {
      const int nb = min(kFixBatch, nbad - b0);
      __syncthreads();   // P written; the previous batch's readers are done
      static_assert(kFixBatch * BN % kFixThreads == 0, "every lane takes part in the shuffles");
      for (int i = tid; i < kFixBatch * BN; i += kFixThreads) {
        const int b = i / BN, r = i % BN;
        const bool ok = b < nb && r < n;
        const int c = ok ? sIdx[b0 + b] : 0;
        const size_t a = (tok0 + (ok ? r : 0)) * vrs + (size_t)kv * DV + c;
        const float l = ok ? P.L[a] : 0.f;
        const float dd = ok ? P.do_ws[(tok0 + r) * ors + (size_t)h * DV + c] : 0.f;
        sL[i] = l;
        sV[i] = ok ? bf2f(P.v[a]) : 0.f;
        sDo[i] = dd;
        // the group of 8 indices (8 lanes): the middle of its L and its spread
        float lx = ok ? l : -INFINITY, ln = ok ? l : INFINITY;
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
          lx = fmaxf(lx, __shfl_xor_sync(0xffffffffu, lx, o));
          ln = fminf(ln, __shfl_xor_sync(0xffffffffu, ln, o));
        }
        const bool any = lx >= ln;   // the group holds an index
        const float lf = any ? 0.5f * (lx + ln) : 0.f, sp = any ? lx - ln : 0.f;
        const bool fac = ok && sp <= kFixSpread;
        sU[i] = fac ? ex2((l - lf) * LOG2E) * dd : 0.f;
        sWp[i] = fac ? ex2((lf - l) * LOG2E) : 0.f;
        if ((lane & 7) == 0) {
          sLg[i / 8] = lf;
          sSp[i / 8] = sp;
          sLx[i / 8] = lx;
          sLn[i / 8] = ln;
        }
      }
      __syncthreads();
      // dv_s[c] += sum_{t > s} P_ts exp(L_t[c] - L_s[c]) do_t[c], into the slot
      if (4 * cg < nb && s_dv < n) {
        float ls[4], wps[4], lfs[4], dvb[4] = {0.f, 0.f, 0.f, 0.f};
        bool fs[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int b = 4 * cg + u;
          ls[u] = sL[b * BN + s_dv];
          wps[u] = sWp[b * BN + s_dv];
          lfs[u] = sLg[b * (BN / 8) + s_dv / 8];
          fs[u] = sSp[b * (BN / 8) + s_dv / 8] <= kFixSpread;
        }
        for (int g = t_dv / 8; g * 8 < n; ++g) {   // warp-uniform group: broadcast reads
          float pts[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            // selected, not multiplied by zero: exp(L_t - L_s) overflows for t < s
            const int t = 8 * g + e;
            pts[e] = t > s_dv && t < n ? sP[t * Lay::kPs + s_dv] : 0.f;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int b = 4 * cg + u;
            if (sLx[b * (BN / 8) + g] - ls[u] < -104.f) continue;   // every term flushes to zero
            float acc = 0.f;
            if (fs[u] && sSp[b * (BN / 8) + g] <= kFixSpread && sLg[b * (BN / 8) + g] - lfs[u] <= kFixRise) {
#pragma unroll
              for (int e = 0; e < 8; ++e) acc = fmaf(pts[e], sU[b * BN + 8 * g + e], acc);
              dvb[u] += wps[u] * ex2((sLg[b * (BN / 8) + g] - lfs[u]) * LOG2E) * acc;
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int t = 8 * g + e;
                if (t > s_dv && t < n) acc += pts[e] * ex2((sL[b * BN + t] - ls[u]) * LOG2E) * sDo[b * BN + t];
              }
              dvb[u] += acc;
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (4 * cg + u < nb) slot[(size_t)s_dv * (DK + DV) + DK + sIdx[b0 + 4 * cg + u]] += dvb[u];
      }
      // dP^bad_ts += sum_{c in batch} do_t[c] exp(L_t[c] - L_s[c]) v_s[c]
      // (pairs above the diagonal get finite values there, which P = 0 then
      // removes; the direct form selects them away instead)
      if (sb <= tb) {
        for (int b = 0; b < nb; ++b) {
          if (sLx[b * (BN / 8) + tb] - sLn[b * (BN / 8) + sb] < -104.f) continue;   // every term flushes to zero
          if (sSp[b * (BN / 8) + tb] <= kFixSpread && sSp[b * (BN / 8) + sb] <= kFixSpread &&
              sLg[b * (BN / 8) + tb] - sLg[b * (BN / 8) + sb] <= kFixRise) {
            const float gf = ex2((sLg[b * (BN / 8) + tb] - sLg[b * (BN / 8) + sb]) * LOG2E);
            float ut[8], ws[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              ut[i] = sU[b * BN + 8 * tb + i] * gf;
              ws[i] = sWp[b * BN + 8 * sb + i] * sV[b * BN + 8 * sb + i];
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
              for (int j = 0; j < 8; ++j) dp[i][j] = fmaf(ut[i], ws[j], dp[i][j]);
          } else {
            float lt[8], dt[8], ls[8], vs[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              lt[i] = sL[b * BN + 8 * tb + i];
              dt[i] = sDo[b * BN + 8 * tb + i];
              ls[i] = sL[b * BN + 8 * sb + i];
              vs[i] = sV[b * BN + 8 * sb + i];
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
              for (int j = 0; j < 8; ++j)
                if (8 * sb + j <= 8 * tb + i)
                  dp[i][j] += dt[i] * ex2((lt[i] - ls[j]) * LOG2E) * vs[j];
          }
        }
      }
    }
    __syncthreads();   // every dv reader of P is done
    // dS^bad = P dP^bad, over P
    if (sb <= tb) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float* e = sP + (8 * tb + i) * Lay::kPs + 8 * sb + j;
          *e = *e * dp[i][j];
        }
    }
    __syncthreads();
    // dK_s += sum_t dS^bad_ts q_t (unscaled, like the slots)
    for (int t = 0; t < n; ++t) {   // dS^bad is zero for t < s
      const float4 ds = *reinterpret_cast<const float4*>(sP + t * Lay::kPs + 4 * sq);
      const float dsa[4] = {ds.x, ds.y, ds.z, ds.w};
#pragma unroll
      for (int e = 0; e < CK; ++e) {
        const float qv = sQt[(cb * CK + e) * BN + t];
#pragma unroll
        for (int a = 0; a < 4; ++a) dk[a][e] = fmaf(dsa[a], qv, dk[a][e]);
      }
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int sk = 4 * sq + a;
    if (sk < n) {
#pragma unroll
      for (int e = 0; e < CK; ++e) slot[(size_t)sk * (DK + DV) + cb * CK + e] += dk[a][e];
    }
  }
}

// ---------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;  // cached driver entry point
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

static bool make_map(CUtensorMap* m, const void* base, int D, int H, int N, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)N};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK, int DV>
static fix_status launch(const Params& prm, const void* vt, const void* vm, int which,
                         long long nparts, long long nslots, cudaStream_t st) {
  const Dims& d = prm.d;
  const int rows = which == 0 ? 128 : BQ;
  CUtensorMap mq, mk, mvt, mvm, mdomh, mdoml, mdot;
  if (!make_map(&mq, prm.q, DK, d.Hq, d.N, rows) ||
      !make_map(&mk, prm.k, DK, d.Hkv, d.N, 128) || !make_map(&mvt, vt, DV, d.Hkv, d.N, 128) ||
      !make_map(&mvm, vm, DV, d.Hkv, d.N, 128) || !make_map(&mdomh, prm.domh, DV, d.Hq, d.N, rows) ||
      !make_map(&mdoml, prm.doml, DV, d.Hq, d.N, rows) || !make_map(&mdot, prm.dot, DV, d.Hq, d.N, rows))
    return FIX_ERR_CUDA;
  if (which == 0) {
    const int smem = DqLayout<DK, DV>::kAlloc;
    auto kern = dq_tc_kernel<DK, DV>;
    if (!set_smem_limit(reinterpret_cast<const void*>(kern), smem))
      return FIX_ERR_CUDA;
    kern<<<(unsigned)((long long)d.nchunks * d.Hq), kThreads, smem, st>>>(mq, mk, mvt, mvm, mdomh,
                                                                         mdot, prm);
  } else {
    const int smem = KvLayout<DK, DV>::kAlloc;
    auto kern = dkv_tc_kernel<DK, DV>;
    if (!set_smem_limit(reinterpret_cast<const void*>(kern), smem))
      return FIX_ERR_CUDA;
    kern<<<(unsigned)(nparts * d.Hkv), kThreads, smem, st>>>(mq, mk, mvt, mvm, mdomh, mdoml, mdot,
                                                            prm);
  }
  return launch_status();
}

// The exact terms of out-of-range channels, then the combine of the dk/dv
// partial slots (which = 2).
template <int DK, int DV>
static fix_status launch_combine(const Params& prm, long long nslots, cudaStream_t st) {
  const Dims& d = prm.d;
  if (nslots <= 0) return FIX_OK;
  const int smem = FixLayout<DK, DV>::kBytes;
  auto fix = dkv_diag_exact_kernel<DK, DV>;
  if (!set_smem_limit(reinterpret_cast<const void*>(fix), smem)) return FIX_ERR_CUDA;
  fix<<<dim3(d.nchunks, d.Hkv), kFixThreads, smem, st>>>(prm);
  dkv_combine_kernel<DK, DV><<<dim3(d.nchunks * (BN / 8), d.Hkv), 256, 0, st>>>(prm);
  return launch_status();
}

}  // namespace tcb

bool tc_bwd_supported(const Dims& d) {
  const bool dims_ok = (d.Dk == 64 || d.Dk == 128) && (d.Dv == 64 || d.Dv == 128);
  return dims_ok && d.N >= FIX_CHUNK && d.grp <= 16;
}

int tc_bwd_kernel_count(const Dims&, long long nslots) { return nslots > 0 ? 4 : 2; }

fix_status tc_bwd(const fix_attn_problem*, const Dims& d, const TcBwdArgs& a, int which,
                  cudaStream_t st) {
  tcb::Params prm{};
  prm.d = d;
  prm.chunks = a.chunks;
  prm.order = a.order;
  prm.q = static_cast<const __nv_bfloat16*>(a.q);
  prm.k = static_cast<const __nv_bfloat16*>(a.k);
  prm.v = static_cast<const __nv_bfloat16*>(a.v);
  prm.L = a.L;
  prm.tot = a.tot;
  prm.rho = a.rho;
  prm.hr = a.hr;
  prm.lvt = a.lvt;
  prm.safe = a.safe;
  prm.dsafe = a.dsafe;
  prm.m_s = a.m_s;
  prm.do_ws = a.do_ws;
  prm.dot = a.dot;
  prm.domh = a.domh;
  prm.doml = a.doml;
  prm.A = a.A;
  prm.ptt = a.ptt;
  prm.delta = a.delta;
  prm.badflag = a.badflag;
  prm.parts = a.parts;
  prm.cpart = a.cpart;
  prm.tiles_per_part = a.tiles_per_part;
  prm.nslots = a.nslots;
  prm.partial = a.partial;
  prm.dq = static_cast<__nv_bfloat16*>(a.dq);
  prm.dk = static_cast<__nv_bfloat16*>(a.dk);
  prm.dv = static_cast<__nv_bfloat16*>(a.dv);
  prm.dG = a.dG;
  prm.status = a.status;
  if (which == 2) {
    if (d.Dk == 128 && d.Dv == 128) return tcb::launch_combine<128, 128>(prm, a.nslots, st);
    if (d.Dk == 64 && d.Dv == 64) return tcb::launch_combine<64, 64>(prm, a.nslots, st);
    if (d.Dk == 128 && d.Dv == 64) return tcb::launch_combine<128, 64>(prm, a.nslots, st);
    if (d.Dk == 64 && d.Dv == 128) return tcb::launch_combine<64, 128>(prm, a.nslots, st);
    return FIX_ERR_HEAD_DIM;
  }
  if (d.Dk == 128 && d.Dv == 128) return tcb::launch<128, 128>(prm, a.vt, a.vm, which, a.nparts, a.nslots, st);
  if (d.Dk == 64 && d.Dv == 64) return tcb::launch<64, 64>(prm, a.vt, a.vm, which, a.nparts, a.nslots, st);
  if (d.Dk == 128 && d.Dv == 64) return tcb::launch<128, 64>(prm, a.vt, a.vm, which, a.nparts, a.nslots, st);
  if (d.Dk == 64 && d.Dv == 128) return tcb::launch<64, 128>(prm, a.vt, a.vm, which, a.nparts, a.nslots, st);
  return FIX_ERR_HEAD_DIM;
}

}  // namespace fix
