// FiX attention forward on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// FiX (poster abstract): causal softmax attention whose forget gate scales the
// value channels element-wise; the softmax denominator is dropped because an
// RMSNorm follows.  The README's "Code Structure" splits the reference into
// intra-chunk preprocessing, inter-chunk scaling of V and a parallel forward;
// here the preprocessing is the prefix pass (fix_prefix.cu) and the rest is
// this one kernel.
//
// One CTA computes one query chunk (128 rows) of one q head against the key
// blocks j = i, i-1, ..., 0 of its sequence (diagonal block first).  Every
// decay factor is split at a per-channel reference so that the row part is
// applied once in the epilogue and the key part scales the value tiles:
//   * diagonal block (j = i), reference rho (the middle of the chunk's range
//     of prefix sums):  exp(G_t - G_s) = exp(L_t - rho) * exp(rho - L_s),
//     both factors in [e^-80, e^80]; Vm_s = v_s exp(rho - L_s) comes from the
//     prefix pass.  Accumulator O_d.
//   * earlier blocks (j < i), reference = the chunk start:
//     exp(G_t - G_s) = exp(L_t) * Vt_s f_ij / v_s, with Vt_s = v_s exp(tot_j -
//     L_s) (prefix pass) and f_ij[c] = exp(sum_{j<j'<i} tot_j'[c]); for g <= 0
//     every factor is <= 1.  Accumulator O_o.
// Epilogue: o_t = exp(L_t - rho) O_d + exp(L_t) O_o + P_tt v_t (the s = t term,
// in fp32), then the RMSNorm.
// The diagonal block carries most of the attention weight whenever the gate
// decays within a chunk, so its bf16 rounding would dominate the error: there
// both P and Vm are split into bf16 hi + lo parts and the block costs three
// MMAs (P_hi Vm_hi + P_lo Vm_hi + P_hi Vm_lo, near-exact).  The other blocks
// use one MMA in fp16 (11-bit significand) when every gate of the sequence up
// to this chunk is <= 0 and |v| <= 3e4, since then P <= e^8 and |V'| <= |v|
// fit fp16; otherwise (rising gates, huge values) in bf16.  Channels whose
// chunk range exceeds the split's float range (Vm = 0, rho = 0 there) get
// their diagonal block exactly in fp32 in the epilogue.
//
// Warp roles (384 threads): warp 0 issues TMA loads (Q once; K and V tiles
// through a 2-stage ring), warp 1 issues the MMAs (one thread) and owns TMEM,
// warps 4-7 turn S into P (one TMEM lane = one query row per thread) and move
// the accumulators to a shared fp32 tile (epilogue phase A), warps 8-11 scale
// the V tiles in shared memory by f_ij.  Once every MMA has completed (the
// MMA warp's single-use `drain` barrier), all twelve warps run epilogue phase
// B: row factor, the s = t term, RMSNorm and coalesced stores, a row per warp
// at a time.  TMEM: two S buffers (P is written over the S it came from, as
// 16-bit pairs) and the two O accumulators.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "fix_internal.h"
#include "fix_sm100.cuh"

namespace fix {
namespace tcf {

using namespace sm100;

constexpr int BM = 128;          // query rows per CTA
constexpr int BN = FIX_CHUNK;    // keys per block
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
__host__ __device__ constexpr uint32_t col_s(int st) { return st ? 128u : 0u; }
constexpr uint32_t kColOd = 256;           // diagonal-block accumulator [256, 256 + DV)
// off-diagonal accumulator O_o at [256 + DV, 256 + 2 DV).  P_lo of the
// diagonal block (64 columns at 384) may share O_o's columns: it is consumed
// by the diagonal PV MMAs, which complete before the first off-diagonal PV
// MMA overwrites O_o (MMAs run in issue order).
constexpr uint32_t kColPlo = 384;
constexpr float kRescaleThreshold = 8.0f;  // lazy row-max update (natural log units)

struct Bars {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2];
  uint64_t v_full[2], v_empty[2], v_ready[2];
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done;
  uint64_t drain;        // final commit: every MMA issued has completed
};

template <int DK, int DV>
struct Layout {
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + BM * DK * 2;
  static constexpr int kV = kK + 2 * BN * DK * 2;
  static constexpr int kVl = kV + 2 * BN * DV * 2;       // Vm_lo of the diagonal block
  static constexpr int kRho = kVl + BN * DV * 2;
  static constexpr int kHr = kRho + DV * 4;
  static constexpr int kW = kHr + DV * 4;
  static constexpr int kRow = kW + DV * 4;              // per-row alpha, P_tt, m (3 x 128 f32)
  static constexpr int kBars = kRow + 3 * BM * 4;
  static constexpr int kTmem = kBars + (int)sizeof(Bars);
  static constexpr int kAbort = kTmem + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr int kAlloc = kBytes + 1024;   // slack for 1024-byte alignment
  // after the last MMA: the exact path's P rows, then the accumulators of
  // every row (fp32, 2 DV per row), reuse the K/V ring and Vm_lo
  static constexpr int kScratch = kK;
  static_assert(2 * BN * DK * 2 + 2 * BN * DV * 2 >= BM * BN * 4, "scratch does not fit");
  static_assert(kRho - kK >= BM * 2 * DV * 4, "accumulator tile does not fit");
};

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
  const int* safe;
  const __nv_bfloat16* w;
  void* y;
  int y_f32;
  float* o_s;
  float* m_s;
  float* rstd_s;
  int* status;
};

// Exact diagonal-block sum of one channel whose chunk range is too wide for
// the split: sum_{s<t} P_ts exp(L_t - L_s) v_s in fp32 (P rows in scratch).
__device__ __noinline__ float exact_diag_channel(const float* __restrict__ prow, int nkeys,
                                                 float lt, const float* __restrict__ Lcol,
                                                 const __nv_bfloat16* __restrict__ vcol,
                                                 size_t rs) {
  float acc = 0.f;
  for (int s = 0; s < nkeys; ++s) {
    const float p = prow[s];
    if (p == 0.f) continue;
    acc += p * ex2((lt - Lcol[(size_t)s * rs]) * LOG2E) * bf2f(vcol[(size_t)s * rs]);
  }
  return acc;
}

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_vt, const __grid_constant__ CUtensorMap tm_vm,
                  const __grid_constant__ CUtensorMap tm_vml, const Params P) {
  using Lay = Layout<DK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const Dims& d = P.d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ci = P.order[blockIdx.x / d.Hq];
  const int h = blockIdx.x % d.Hq, kv = h / d.grp;
  const Chunk ch = P.chunks[ci];
  if (ch.len <= 0) return;
  const int nblk = ch.j + 1;
  const int first = ci - ch.j;
  const int seq0 = ch.tok0 - ch.j * FIX_CHUNK;
  const size_t vrs = (size_t)d.Hkv * DV;

  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem + Lay::kQ);
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem + Lay::kK);
  __nv_bfloat16* sV = reinterpret_cast<__nv_bfloat16*>(smem + Lay::kV);
  __nv_bfloat16* sVl = reinterpret_cast<__nv_bfloat16*>(smem + Lay::kVl);
  float* sRho = reinterpret_cast<float*>(smem + Lay::kRho);
  float* sHr = reinterpret_cast<float*>(smem + Lay::kHr);
  float* sW = reinterpret_cast<float*>(smem + Lay::kW);
  Bars* bar = reinterpret_cast<Bars*>(smem + Lay::kBars);
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + Lay::kTmem);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + Lay::kAbort);
  const Ctl ctl{P.status, sAbort};

  // ---------------------------------------------------------------- setup
  bool my_bad = false;
  if (tid < DV) {
    const size_t ti = ((size_t)ci * d.Hkv + kv) * DV + tid;
    const float hrv = P.hr[ti];
    my_bad = hrv > FIX_HR_MAX;
    sHr[tid] = hrv;
    sRho[tid] = P.rho[ti];
    sW[tid] = bf2f(P.w[tid]);
  }
  if (tid == 0) {
    *sAbort = 0;
    mbar_init(&bar->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
      mbar_init(&bar->v_ready[s], 128);
      mbar_init(&bar->s_full[s], 1);
      mbar_init(&bar->p_full[s], 128);
    }
    mbar_init(&bar->pv_done, 1);
    mbar_init(&bar->drain, 1);
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(sTmem, kTmemCols);
  bool my_safe = true;
  for (int jj = tid; jj < nblk; jj += blockDim.x) my_safe = my_safe && P.safe[(size_t)(first + jj) * d.Hkv + kv];
  const int cta_f16 = __syncthreads_and(my_safe);
  tc_fence_before();
  const int any_bad = __syncthreads_or(my_bad);
  tc_fence_after();
  const uint32_t tmem = *sTmem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_expect_tx(&bar->q_full, BM * DK * 2);
      for (int hh = 0; hh < DK / 64; ++hh)
        tma_load_3d(sQ + hh * BM * 64, &tm_q, &bar->q_full, hh * 64, h, ch.tok0);
      int nk = 0, nv = 0;  // K / V tiles issued
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
        mbar_expect_tx(&bar->v_full[st], (it == 0 ? 2 : 1) * BN * DV * 2);
        const CUtensorMap* vmap = it == 0 ? &tm_vm : &tm_vt;
        for (int hh = 0; hh < DV / 64; ++hh)
          tma_load_3d(sV + st * BN * DV + hh * BN * 64, vmap, &bar->v_full[st], hh * 64, kv, ktok);
        if (it == 0)
          for (int hh = 0; hh < DV / 64; ++hh)
            tma_load_3d(sVl + hh * BN * 64, &tm_vml, &bar->v_full[0], hh * 64, kv, ktok);
        ++nv;
      }
      // every issued copy must land before the CTA may exit (also after an
      // abort): wait for the last one or two issued per ring, timeout only
      const Ctl drain{P.status, nullptr};
      for (int it = nk - 1; it >= 0 && it >= nk - 2; --it)
        mbar_wait(&bar->k_full[it & 1], (it >> 1) & 1, drain);
      for (int it = nv - 1; it >= 0 && it >= nv - 2; --it)
        mbar_wait(&bar->v_full[it & 1], (it >> 1) & 1, drain);
      mbar_wait(&bar->q_full, 0, drain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(BM, BN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(BM, DV, false, true);
      const uint32_t idesc_pv_off = idesc_bf16(BM, DV, false, true, cta_f16 != 0);
      const uint32_t q_addr = smem_u32(sQ);
      bool ok = mbar_wait(&bar->q_full, 0, ctl);
      auto issue_qk = [&](int it) -> bool {
        const int st = it & 1;
        if (!mbar_wait(&bar->k_full[st], (it >> 1) & 1, ctl)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + st * BN * DK);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          const uint64_t a = desc_add(desc_sw128(q_addr, 16, 1024), off);
          const uint64_t b = desc_add(desc_sw128(k_addr, 16, 1024), (kk >> 2) * (BN * 128) + (kk & 3) * 32);
          mma_ss(tmem + col_s(st), a, b, idesc_qk, kk > 0);
        }
        tc_commit(&bar->s_full[st]);
        tc_commit(&bar->k_empty[st]);
        return true;
      };
      if (ok) ok = issue_qk(0);
      if (ok && nblk > 1) ok = issue_qk(1);
      for (int it = 0; ok && it < nblk; ++it) {
        const int st = it & 1;
        const uint32_t ph = (it >> 1) & 1;
        if (!mbar_wait(&bar->p_full[st], ph, ctl) || !mbar_wait(&bar->v_ready[st], ph, ctl)) break;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sV + st * BN * DV);
        if (it == 0) {
          const uint32_t vl_addr = smem_u32(sVl);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t bh = desc_add(desc_sw128(v_addr, BN * 128, 1024), kk * 2048);
            const uint64_t bl = desc_add(desc_sw128(vl_addr, BN * 128, 1024), kk * 2048);
            mma_ts(tmem + kColOd, tmem + col_s(0) + kk * 8, bh, idesc_pv, kk > 0);
            mma_ts(tmem + kColOd, tmem + kColPlo + kk * 8, bh, idesc_pv, 1);
            mma_ts(tmem + kColOd, tmem + col_s(0) + kk * 8, bl, idesc_pv, 1);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t b = desc_add(desc_sw128(v_addr, BN * 128, 1024), kk * 2048);
            mma_ts(tmem + kColOd + DV, tmem + col_s(st) + kk * 8, b, idesc_pv_off,
                   (it > 1 || kk > 0));
          }
        }
        tc_commit(&bar->v_empty[st]);
        tc_commit(&bar->pv_done);
        if (it + 2 < nblk) ok = issue_qk(it + 2);
      }
      // TMEM must not be released while an issued MMA may still write it
      tc_commit(&bar->drain);
      mbar_wait(&bar->drain, 0, Ctl{P.status, nullptr});
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ softmax + epilogue
    const int r = (warp - 4) * 32 + lane;              // query row in the chunk
    const uint32_t lane_base = tmem + ((uint32_t)((warp - 4) * 32) << 16);
    const float c1 = d.scale * LOG2E;
    float m_used = -INFINITY, m_true = -INFINITY, s_diag = 0.f;
    bool ok = true;
    for (int it = 0; it < nblk; ++it) {
      const int st = it & 1;
      // waits vote warp-wide: the TMEM accesses below are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&bar->s_full[st], (it >> 1) & 1, ctl))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sbase = lane_base + col_s(st);
      // the whole S row in registers: four TMEM loads, one wait
      uint32_t xs[BN];
#pragma unroll
      for (int c4 = 0; c4 < BN / 32; ++c4)
        tmem_ld32(sbase + c4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&xs[c4 * 32]));
      tmem_wait_ld();
      float mx = -INFINITY;
      if (it > 0) {
#pragma unroll
        for (int e = 0; e < BN; e += 2)
          mx = fmaxf(mx, fmaxf(__uint_as_float(xs[e]), __uint_as_float(xs[e + 1])));
      } else {
        // diagonal block: keys s <= t; S_tt kept for the exact s = t term
#pragma unroll
        for (int e = 0; e < BN; ++e) {
          const float sv = __uint_as_float(xs[e]);
          mx = e <= r ? fmaxf(mx, sv) : mx;
          s_diag = e == r ? sv : s_diag;
        }
      }
      const float mrow = mx * d.scale;
      m_true = fmaxf(m_true, mrow);
      if (it == 0) {
        m_used = m_true;
      } else if (__any_sync(0xffffffffu, m_true > m_used + kRescaleThreshold)) {
        // rare: some row's max grew past the threshold; the whole warp (the
        // TMEM accesses are warp-collective) rescales its rows of O to their
        // new max before P_it is formed against it
        if (!__all_sync(0xffffffffu, mbar_wait(&bar->pv_done, (it - 1) & 1, ctl))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float alpha = ex2((m_used - m_true) * LOG2E);
        // both accumulators (before the first off-diagonal PV the O_o columns
        // hold stale data that PV_1 overwrites, so scaling them is harmless)
#pragma unroll
        for (int cc = 0; cc < 2 * DV / 32; ++cc) {
          uint32_t x[32];
          tmem_ld32(lane_base + kColOd + cc * 32, x);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] = __float_as_uint(__uint_as_float(x[e]) * alpha);
          tmem_st32(lane_base + kColOd + cc * 32, x);
        }
        tmem_wait_st();
        m_used = m_true;
      }
      const float moff = m_used * LOG2E;
      if (it == 0) {
        // diagonal block: strictly causal P as bf16 hi + lo
#pragma unroll
        for (int c4 = 0; c4 < BN / 32; ++c4) {
          uint32_t pk[16], pl[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int key = c4 * 32 + e;
            const float p0 = key < r ? ex2(__uint_as_float(xs[key]) * c1 - moff) : 0.f;
            const float p1 = key + 1 < r ? ex2(__uint_as_float(xs[key + 1]) * c1 - moff) : 0.f;
            pk[e >> 1] = pack_bf16(p0, p1);
            const float h0 = __uint_as_float(pk[e >> 1] << 16);
            const float h1 = __uint_as_float(pk[e >> 1] & 0xFFFF0000u);
            pl[e >> 1] = pack_bf16(p0 - h0, p1 - h1);
          }
          tmem_st16(sbase + c4 * 16, pk);
          tmem_st16(lane_base + kColPlo + c4 * 16, pl);
        }
      } else if (cta_f16) {
#pragma unroll
        for (int c4 = 0; c4 < BN / 32; ++c4) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int key = c4 * 32 + e;
            pk[e >> 1] = pack_f16(ex2(__uint_as_float(xs[key]) * c1 - moff),
                                  ex2(__uint_as_float(xs[key + 1]) * c1 - moff));
          }
          tmem_st16(sbase + c4 * 16, pk);
        }
      } else {
#pragma unroll
        for (int c4 = 0; c4 < BN / 32; ++c4) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int key = c4 * 32 + e;
            pk[e >> 1] = pack_bf16(ex2(__uint_as_float(xs[key]) * c1 - moff),
                                   ex2(__uint_as_float(xs[key + 1]) * c1 - moff));
          }
          tmem_st16(sbase + c4 * 16, pk);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar->p_full[st]);
    }

    // ---------------------------------------------------------- epilogue
    // Every MMA of the CTA has completed once `drain` has: the MMA warp
    // commits it once, after its last PV.  (pv_done completes once per PV, so
    // a warp that reaches this point late could find it two phases on and
    // wait for a phase that never comes.)
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar->drain, 0, ctl));
    tc_fence_after();
    const bool row_ok = ok && r < ch.len;
    const size_t tok = (size_t)ch.tok0 + (size_t)(r < ch.len ? r : 0);
    if (any_bad) {
      // exact fp32 diagonal block for channels outside the split's range:
      // P rows into the (now idle) K/V ring, then one pass per such channel;
      // the result replaces that channel's (zero) diagonal accumulator column
      float* prow = reinterpret_cast<float*>(smem + Lay::kScratch) + (size_t)r * BN;
      const size_t krs = (size_t)d.Hkv * DK;
      const __nv_bfloat16* kbase = P.k + (size_t)ch.tok0 * krs + (size_t)kv * DK;
      const __nv_bfloat16* qrow = P.q + tok * (size_t)d.Hq * DK + (size_t)h * DK;
      const int nk = row_ok ? r : 0;
      for (int s = 0; s < nk; ++s) {
        const __nv_bfloat16* krow = kbase + (size_t)s * krs;
        float acc = 0.f;
        for (int dd = 0; dd < DK; dd += 8) {
          const uint4 qa = *reinterpret_cast<const uint4*>(qrow + dd);
          const uint4 ka = *reinterpret_cast<const uint4*>(krow + dd);
          const uint32_t qw[4] = {qa.x, qa.y, qa.z, qa.w}, kw[4] = {ka.x, ka.y, ka.z, ka.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            acc += __uint_as_float(qw[u] << 16) * __uint_as_float(kw[u] << 16);
            acc += __uint_as_float(qw[u] & 0xFFFF0000u) * __uint_as_float(kw[u] & 0xFFFF0000u);
          }
        }
        prow[s] = ex2((acc * d.scale - m_true) * LOG2E);
      }
      const float* Lrow = P.L + tok * vrs + (size_t)kv * DV;
      const float* Lcol0 = P.L + (size_t)ch.tok0 * vrs + (size_t)kv * DV;
      const __nv_bfloat16* vcol0 = P.v + (size_t)ch.tok0 * vrs + (size_t)kv * DV;
      for (int c = 0; c < DV; ++c) {
        if (sHr[c] <= FIX_HR_MAX) continue;   // CTA-uniform
        const float e = exact_diag_channel(prow, nk, Lrow[c], Lcol0 + c, vcol0 + c, vrs);
        tmem_st1(lane_base + kColOd + c, __float_as_uint(e));
      }
      tmem_wait_st();
      asm volatile("bar.sync 1, 128;" ::: "memory");   // P rows done before the tile overwrites them
    }
    // phase A: this row's two accumulators into a shared fp32 tile, its 16-byte
    // groups XOR-swizzled by row so that neighbouring rows hit other banks
    float* tile = reinterpret_cast<float*>(smem + Lay::kScratch);
    float* trow = tile + (size_t)r * (2 * DV);
#pragma unroll
    for (int cc = 0; cc < 2 * DV / 32; ++cc) {
      uint32_t x[32];
      tmem_ld32(lane_base + kColOd + cc * 32, x);
      tmem_wait_ld();
#pragma unroll
      for (int g4 = 0; g4 < 8; ++g4) {
        const int grp = cc * 8 + g4;
        *reinterpret_cast<float4*>(trow + ((grp ^ (r & 7)) << 2)) =
            make_float4(__uint_as_float(x[4 * g4]), __uint_as_float(x[4 * g4 + 1]),
                        __uint_as_float(x[4 * g4 + 2]), __uint_as_float(x[4 * g4 + 3]));
      }
    }
    float* sRow = reinterpret_cast<float*>(smem + Lay::kRow);
    sRow[r] = ok ? ex2((m_used - m_true) * LOG2E) : 0.f;                 // alpha
    sRow[BM + r] = ex2((s_diag * d.scale - m_true) * LOG2E);              // P_tt
    sRow[2 * BM + r] = m_true;
  } else if (warp >= 8) {
    // ------------------------------------------------------------ V decay (j < i)
    const int dt = tid - 256;                        // 0..127
    constexpr int kChunks = DV / 8;                  // 16-byte chunks per row
    constexpr int kRowsPerPass = 128 / kChunks;
    const int lc = dt % kChunks;                     // logical chunk: channels lc*8 .. +7
    const int r0 = dt / kChunks;
    const int half = lc >> 3, lcc = lc & 7;
    float delta[8], f8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) delta[e] = 0.f;
    for (int it = 0; it < nblk; ++it) {
      const int st = it & 1;
      const int j = ch.j - it;
      if (it >= 2) {
        const float* tp = P.tot + ((size_t)(first + j + 1) * d.Hkv + kv) * DV + lc * 8;
        const float4 t0 = *reinterpret_cast<const float4*>(tp);
        const float4 t1 = *reinterpret_cast<const float4*>(tp + 4);
        delta[0] += t0.x; delta[1] += t0.y; delta[2] += t0.z; delta[3] += t0.w;
        delta[4] += t1.x; delta[5] += t1.y; delta[6] += t1.z; delta[7] += t1.w;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) f8[e] = ex2(delta[e] * LOG2E);
      if (!mbar_wait(&bar->v_full[st], (it >> 1) & 1, ctl)) break;
      if (it > 0) {
        // Vt arrives as fp16 or bf16 (per chunk, see the prefix pass); V' is
        // written in the operand type of this CTA's off-diagonal MMAs
        const bool in_f16 = P.safe[(size_t)(first + j) * d.Hkv + kv] != 0;
        uint8_t* vb = reinterpret_cast<uint8_t*>(sV + st * BN * DV) + half * (BN * 128);
#pragma unroll 4
        for (int s = r0; s < BN; s += kRowsPerPass) {
          uint4* p = reinterpret_cast<uint4*>(vb + s * 128 + ((lcc ^ (s & 7)) << 4));
          uint4 x = *p;
          uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float a, b;
            if (in_f16) {
              const float2 ab = __half22float2(*reinterpret_cast<const __half2*>(&w4[u]));
              a = ab.x;
              b = ab.y;
            } else {
              a = __uint_as_float(w4[u] << 16);
              b = __uint_as_float(w4[u] & 0xFFFF0000u);
            }
            a *= f8[2 * u];
            b *= f8[2 * u + 1];
            w4[u] = cta_f16 ? pack_f16(a, b) : pack_bf16(a, b);
          }
          *p = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async_smem();
      }
      mbar_arrive(&bar->v_ready[st]);
    }
  }

  // ------------------------------------------------------------ phase B
  // every warp once the roles are done, rows in batches, lanes over
  // channels: coalesced L / v loads, the RMSNorm reduction and coalesced
  // y / o stores
  __syncthreads();
  {
    if (!*sAbort) {
      const float* __restrict__ tile = reinterpret_cast<const float*>(smem + Lay::kScratch);
      const float* __restrict__ sRow = reinterpret_cast<const float*>(smem + Lay::kRow);
      const float* __restrict__ Lg = P.L + (size_t)kv * DV;
      const __nv_bfloat16* __restrict__ vg = P.v + (size_t)kv * DV;
      float* __restrict__ yf = P.y_f32 ? reinterpret_cast<float*>(P.y) : nullptr;
      __nv_bfloat16* __restrict__ yb = P.y_f32 ? nullptr : reinterpret_cast<__nv_bfloat16*>(P.y);
      float* __restrict__ osv = P.o_s;
      const bool has_off = nblk > 1;
      const size_t ors = (size_t)d.Hq * DV;
      constexpr int kU = DV / 32;
      constexpr int kRows = 4;                         // rows in flight per warp
      float rho_l[kU], w_l[kU];
      bool bad_l[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = lane + 32 * u;
        rho_l[u] = sRho[c];
        w_l[u] = sW[c];
        bad_l[u] = sHr[c] > FIX_HR_MAX;           // od holds the exact diagonal sum
      }
      for (int r0 = warp * kRows; r0 < ch.len; r0 += (kThreads / 32) * kRows) {
        float lt[kRows][kU], vt[kRows][kU];
#pragma unroll
        for (int q = 0; q < kRows; ++q) {
          const int rr = min(r0 + q, ch.len - 1);
          const size_t tk = (size_t)ch.tok0 + rr;
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int c = lane + 32 * u;
            lt[q][u] = Lg[tk * vrs + c];
            vt[q][u] = bf2f(vg[tk * vrs + c]);
          }
        }
#pragma unroll
        for (int q = 0; q < kRows; ++q) {
          const int rr = r0 + q;
          if (rr >= ch.len) break;
          const size_t tk = (size_t)ch.tok0 + rr;
          const float* trow = tile + (size_t)rr * (2 * DV);
          const float alpha = sRow[rr], ptt = sRow[BM + rr];
          float o[kU];
          float ss = 0.f;
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int c = lane + 32 * u;
            const float od = trow[(((c >> 2) ^ (rr & 7)) << 2) + (c & 3)];
            const int co = DV + c;
            const float oo = trow[(((co >> 2) ^ (rr & 7)) << 2) + (co & 3)];
            float x = bad_l[u] ? od : alpha * od * ex2((lt[q][u] - rho_l[u]) * LOG2E);
            if (has_off) x += alpha * oo * ex2(lt[q][u] * LOG2E);
            x += ptt * vt[q][u];
            o[u] = x;
            ss += x * x;
          }
          ss = warp_sum(ss);
          const float rstd = 1.0f / sqrtf(ss / (float)DV + d.eps);
          const size_t a0 = tk * ors + (size_t)h * DV;
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int c = lane + 32 * u;
            const float yv = o[u] * rstd * w_l[u];
            if (yf) yf[a0 + c] = yv;
            else yb[a0 + c] = f2bf(yv);
            if (osv) osv[a0 + c] = o[u];
          }
          if (osv && lane == 0) {
            P.m_s[tk * d.Hq + h] = sRow[2 * BM + rr];
            P.rstd_s[tk * d.Hq + h] = rstd;
          }
        }
      }
    }
  }
  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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

// [N, H, D] bf16 viewed as a 3-D tensor (D, H, N); box = 64 x 1 x 128 rows,
// 128-byte swizzle (the canonical K-major / MN-major operand layout).
static bool make_map(CUtensorMap* m, const void* base, int D, int H, int N) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)N};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK, int DV>
static fix_status launch(const Params& prm, const void* q, const void* k, const void* vt,
                         const void* vm, const void* vml, cudaStream_t st) {
  const Dims& d = prm.d;
  CUtensorMap mq, mk, mvt, mvm, mvml;
  if (!make_map(&mq, q, DK, d.Hq, d.N) || !make_map(&mk, k, DK, d.Hkv, d.N) ||
      !make_map(&mvt, vt, DV, d.Hkv, d.N) || !make_map(&mvm, vm, DV, d.Hkv, d.N) ||
      !make_map(&mvml, vml, DV, d.Hkv, d.N))
    return FIX_ERR_CUDA;
  const int smem = Layout<DK, DV>::kAlloc;
  auto kern = fwd_tc_kernel<DK, DV>;
  if (!set_smem_limit(reinterpret_cast<const void*>(kern), smem))
    return FIX_ERR_CUDA;
  const long long grid = (long long)d.nchunks * d.Hq;
  if (grid <= 0) return FIX_OK;
  kern<<<(unsigned)grid, kThreads, smem, st>>>(mq, mk, mvt, mvm, mvml, prm);
  return cudaGetLastError() == cudaSuccess ? FIX_OK : FIX_ERR_CUDA;
}

}  // namespace tcf

bool tc_fwd_supported(const Dims& d) {
  const bool dims_ok = (d.Dk == 64 || d.Dk == 128) && (d.Dv == 64 || d.Dv == 128);
  return dims_ok && d.N >= FIX_CHUNK;
}

int tc_fwd_kernel_count(const Dims&) { return 1; }

fix_status tc_fwd(const Dims& d, const Chunk* chunks, const int* order, const void* q,
                  const void* k, const uint16_t* vt, const __nv_bfloat16* vm,
                  const __nv_bfloat16* vml, const void* v,
                  const float* L, const float* tot, const float* rho, const float* hr,
                  const int* safe,
                  const void* w, void* y, bool y_f32, float* o_s, float* m_s, float* rstd_s,
                  int* status, cudaStream_t st) {
  tcf::Params prm{};
  prm.d = d;
  prm.chunks = chunks;
  prm.order = order;
  prm.q = static_cast<const __nv_bfloat16*>(q);
  prm.k = static_cast<const __nv_bfloat16*>(k);
  prm.v = static_cast<const __nv_bfloat16*>(v);
  prm.L = L;
  prm.tot = tot;
  prm.rho = rho;
  prm.hr = hr;
  prm.safe = safe;
  prm.w = static_cast<const __nv_bfloat16*>(w);
  prm.y = y;
  prm.y_f32 = y_f32 ? 1 : 0;
  prm.o_s = o_s;
  prm.m_s = m_s;
  prm.rstd_s = rstd_s;
  prm.status = status;
  if (d.Dk == 128 && d.Dv == 128) return tcf::launch<128, 128>(prm, q, k, vt, vm, vml, st);
  if (d.Dk == 64 && d.Dv == 64) return tcf::launch<64, 64>(prm, q, k, vt, vm, vml, st);
  if (d.Dk == 128 && d.Dv == 64) return tcf::launch<128, 64>(prm, q, k, vt, vm, vml, st);
  if (d.Dk == 64 && d.Dv == 128) return tcf::launch<64, 128>(prm, q, k, vt, vm, vml, st);
  return FIX_ERR_HEAD_DIM;
}

}  // namespace fix
