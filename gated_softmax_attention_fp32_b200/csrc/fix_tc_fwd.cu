// FiX attention forward on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// FiX (poster abstract): causal softmax attention whose forget gate scales the
// value channels element-wise; the softmax denominator is dropped because an
// RMSNorm follows.  The README's "Code Structure" splits the reference into
// intra-chunk preprocessing, inter-chunk scaling of V and a parallel forward;
// here the preprocessing is the prefix pass (fix_prefix.cu) and the rest is
// this one persistent kernel.
//
// Work unit ("tile"): one query chunk i (128 rows) of one q head against the
// key blocks of its sequence: first the earlier blocks j = i-1, ..., 0, then
// the diagonal block j = i.  Tiles are sorted longest first (the host-side
// order of chunks) and dealt to the persistent CTAs in snake order, so that
// every CTA gets a mix of long and short tiles.
//
// Decay split, per channel c (L = chunk-local prefix sums of g, rho = the
// middle of the chunk's range of L, tot = chunk totals):
//   * earlier blocks: exp(G_t - G_s) = exp(L_t) * f_ij * exp(tot_j - L_s),
//     f_ij = exp(sum_{j<j'<i} tot_j').  The prefix pass stores Vt_s = v_s
//     exp(tot_j - L_s) (fp16, times 2^-e per channel); the V-scaling warps
//     form V'' = Vt f_ij 2^-k_c in shared memory, with one power of two k_c per
//     (tile, channel) chosen so that every V'' fits fp16 (k_c = 0 whenever
//     every gate is <= 0).  P V'' accumulates in fp16 MMAs into A.
//   * fold: once those MMAs are done, A is scaled per column by
//     F_c = exp(rho_c) 2^k_c, which moves the accumulator to the diagonal
//     block's reference: A = sum_{j<i} exp(rho - L_t) ... (see below).
//   * diagonal block: exp(G_t - G_s) = exp(L_t - rho) exp(rho - L_s), both
//     factors in [e^-80, e^80]; Vm_s = v_s exp(rho - L_s) comes from the
//     prefix pass as bf16 hi + lo, and P as bf16 hi + lo, so the block costs
//     three MMAs (P_hi Vm_hi + P_lo Vm_hi + P_hi Vm_lo) and is near-exact
//     (keys s <= t, the s = t pair included).
//   * epilogue: o_t = alpha_t exp(L_t - rho) A_t (alpha_t = exp(m_used - m_t)
//     undoes the lazily updated row shift), then the RMSNorm.  L comes from
//     a channel-major copy (prefix pass), so that the row factors of a warp's
//     32 rows are one coalesced load per channel.
// Channels outside the split's range (prefix pass: rho = 0, Vm = 0) get no
// fold beyond 2^k_c, and the softmax warps add their exact diagonal sum
// exp(L_t) A_t + sum_{s<=t} P_ts exp(L_t - L_s) v_s (fp32) in place; the
// epilogue then applies no row factor to them.
//
// Warp roles (352 threads):
//   warp 0       TMA producer: Q per tile, K through a 2-stage ring
//   warp 1       MMA issuer (one thread) and TMEM owner
//   warps 2-5    softmax, a thread per query row: S -> P in TMEM.  Earlier
//                blocks in one pass (lazy row-max reference, moved in place
//                when a 32-key chunk exceeds it), the diagonal in two (row
//                max first); the fold; the exact sums of out-of-range
//                channels; then half of the tile's epilogue (channels
//                [0, DV/2)) before the next tile
//   warps 6-9    V scaling: V'' in shared memory, the tile's fold factors;
//                then the other half of the tile's epilogue.  One warp of
//                each group per SM sub-partition.
//   warp 10      TMA producer: V (Vt / Vm hi) through a 2-stage ring, Vm lo
//                of the diagonal block (apart from K, whose loads then run
//                ahead of the V ring's waits)
// The epilogue (a thread per row: o = alpha exp(L - rho) A written back over
// A, the RMSNorm's sum of squares joined across the two halves, then y and
// the saved o) runs while the next tile's first QK^T MMAs and V loads do.
// TMEM (512 columns): S/P double buffer at 0 and 128 (P written over S as
// 16-bit pairs; the diagonal's P_lo in the buffer's upper half), and the
// accumulator A double-buffered by tile parity at 256 and 256 + DV.
//
// Every mbarrier wait is bounded (1 s); a wait that expires sets the status
// word to FIX_DEV_TIMEOUT and the CTA's abort flag, the roles stop, copies in
// flight are drained and TMEM is released.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "fix_internal.h"
#include "fix_sm100.cuh"

namespace fix {
namespace tcf {

using namespace sm100;

constexpr int BM = 128;          // query rows per tile
constexpr int BN = FIX_CHUNK;    // keys per block
constexpr int kThreads = 352;
constexpr int kVsThreads = 128;  // V-scaling threads (warps 6-9)
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // lazy row-max update, natural-log units
// One pair of softmax exponentials in this many by the FMA-pipe polynomial
// (0: none).  Off: with one softmax warp per scheduler the softmax is bound
// by issue and latency, not by the MUFU unit, and the polynomial's extra
// instructions cost more than the MUFU time they save (measured: 2.8K
// against 3.1-3.3K cycles per block with one pair in four).
constexpr int kPolyPairEvery = 0;
__host__ __device__ constexpr uint32_t col_s(int b) { return b ? 128u : 0u; }

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[2], k_empty[2];
  uint64_t v_full[2], v_empty[2], v_ready[2];
  uint64_t vlo_empty;
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done;
  uint64_t acc_full[2], acc_empty[2];
  uint64_t fold_ready[2];
  uint64_t rows_ready[2];
  uint64_t xs_sync;   // the softmax warps' meeting point in the exact sums
  uint64_t drain;
};

template <int DK, int DV>
struct Layout {
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + BM * DK * 2;
  static constexpr int kV = kK + 2 * BN * DK * 2;
  // Vm lo of the diagonal block; from a tile's last MMA to the next diagonal
  // load, the epilogue's staging tiles (8 warps x 32 rows x 32 fp32)
  static constexpr int kVl = kV + 2 * BN * DV * 2;
  static constexpr int kVlBytes = BN * DV * 2 > 8 * 4096 ? BN * DV * 2 : 8 * 4096;
  static constexpr int kF = kVl + kVlBytes;              // [2][DV] f32 fold factors
  static constexpr int kBad = kF + 2 * DV * 4;           // [2][DV] int out-of-range flags
  static constexpr int kAnyBad = kBad + 2 * DV * 4;      // [2] int
  static constexpr int kRows = kAnyBad + 16;             // [2][4][BM] f32: alpha, (unused), m, l
  static constexpr int kPlo = kRows + 2 * 4 * BM * 4;    // [BM][33] u32: diagonal P_lo, key chunks 0-1
  static constexpr int kEpiW = kPlo + BM * 33 * 4;       // [DV] f32 w
  static constexpr int kSS = kEpiW + DV * 4;             // [2][BM] f32: the epilogue halves' sums of squares
  static constexpr int kEC = kSS + 2 * BM * 4;           // [2][DV] f32: rho log2e, NaN out of range
  static constexpr int kBars = (kEC + 2 * DV * 4 + 7) / 8 * 8;
  static constexpr int kTmem = kBars + (int)sizeof(Bars);
  static constexpr int kAbort = kTmem + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr int kAlloc = kBytes + 1024;   // slack for 1024-byte alignment
  static_assert(kAlloc <= 232448, "shared memory");
};

struct Params {
  Dims d;
  const Chunk* chunks;
  const int* order;
  int ntiles;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* L;
  const float* Lt;            // L channel-major [Hkv][DV][N]
  const float* tot;
  const float* rho;
  const float* hr;
  const float* lvt;
  const int* safe;
  const __nv_bfloat16* w;     // NULL allowed without the norm
  const __nv_bfloat16* z;     // output gate or NULL
  void* y;
  int y_f32;
  float* o_s;
  float* m_s;
  float* rstd_s;
  int* status;
  int stall;       // test builds only: issue no loads, waits give up after 1 ms
};

// The tile a CTA takes in a given round: snake order over the longest-first
// tile list, so that the long tiles of round 0 pair with the short ones of
// round 1.
__device__ __forceinline__ int tile_of(int round, int G, int c) {
  return round * G + ((round & 1) ? (G - 1 - c) : c);
}

struct Tile {
  int ci, h, kv;
  int j, nblk, first, seq0, tok0, len;
};

__device__ __forceinline__ Tile tile_info(const Params& P, int t) {
  Tile x;
  const int ci = P.order[t / P.d.Hq];
  x.ci = ci;
  x.h = t % P.d.Hq;
  x.kv = x.h / P.d.grp;
  const Chunk ch = P.chunks[ci];
  x.j = ch.j;
  x.nblk = ch.j + 1;
  x.first = ci - ch.j;
  x.seq0 = ch.tok0 - ch.j * FIX_CHUNK;
  x.tok0 = ch.tok0;
  x.len = ch.len;
  return x;
}

// Named barriers (ids 1..2; 0 is __syncthreads): id 1 the epilogue's two
// groups (softmax and V-scaling warps, 256 threads), id 2 the V-scaling warps.
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ int wg_and(int id, int n, int pred) {
  int out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(pred), "r"(id), "r"(n)
      : "memory");
  return out;
}
__device__ __forceinline__ int wg_or(int id, int n, int pred) {
  int out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(pred), "r"(id), "r"(n)
      : "memory");
  return out;
}

// Exact diagonal sums of out-of-range channels, in fp32 from the fp32 logits
// of the diagonal block (TMEM columns sbase..sbase+BN of this warp's rows):
//   A_tc <- exp(L_t) A_tc + sum_{s<=t} P_ts exp(L_t - L_s) v_s.
// Called by the 128 softmax threads together (thread r = row t = key s),
// which meet on an mbarrier: sync_n meetings have taken place before, the
// count after the call is returned, or -1 after an abort (bounded waits).
// The decay goes through the middle rho of each 8-key sub-block's range of L:
// exp(L_t - L_s) = exp(L_t - rho) exp(rho - L_s).  Channels go in groups:
// the key factors w_s = exp(rho - L_s) v_s (a thread per key, all loads of
// the group in flight at once), rho, the sub-block's spread of L and its
// largest L go to shared memory (the P_lo staging area, free until pass 2);
// then each row takes one exponential per sub-block.  A sub-block whose L
// spreads more than 88 (|L_s - rho| > 44), or where the row's L lies more
// than 44 above rho, takes the direct exponential per pair; otherwise no
// factor and no partial product leaves the fp32 range unless the pair's own
// exp(L_t - L_s) does, and a row factor that underflows only drops terms
// below e^-43 of their own size.  A sub-block whose every L_s exceeds L_t by more than 104
// is skipped: each of its exponentials is below 2^-150 and flushes to zero
// (as the direct form's would).  Not inlined: it runs only for tiles holding
// such channels, and its registers stay out of the softmax loop.
constexpr int kExactGroup = 8;
template <int DK, int DV>
__device__ __noinline__ int diag_exact_sums(const float* Lrow, const float* LtK, int N,
                                            const __nv_bfloat16* vk, int vrs, uint8_t* smem,
                                            int tb, int nk, int r, uint32_t sbase, uint32_t acol,
                                            float c1, float moff, int sync_n, int* status) {
  using Lay = Layout<DK, DV>;
  const Ctl ctl{status, reinterpret_cast<volatile int*>(smem + Lay::kAbort)};
  constexpr int kG = kExactGroup, kSB = BN / 8;
  const int lane = r & 31;
  const int* bad = reinterpret_cast<const int*>(smem + Lay::kBad) + tb * DV;
  float* stg = reinterpret_cast<float*>(smem + Lay::kPlo);
  uint64_t* sync_bar = &reinterpret_cast<Bars*>(smem + Lay::kBars)->xs_sync;
  int* list = reinterpret_cast<int*>(stg);   // [DV] the bad channels, in order
  float* sw = stg + DV;                      // [kG][BN] key factors
  float* slb = sw + kG * BN;                 // [kG][kSB] the middle of the sub-block's L
  float* ssp = slb + kG * kSB;               // [kG][kSB] its spread of L
  float* slm = ssp + kG * kSB;               // [kG][kSB] its largest L
  float* slt = slm + kG * kSB;               // [kG][BM] L_t of each thread's row
  float* sacc = slt + kG * BM;               // [kG][BM] each thread's sums
  static_assert(DV + kG * BN + 3 * kG * kSB + 2 * kG * BM <= BM * 33, "staging area");
  auto sync = [&]() -> bool {
    mbar_arrive(sync_bar);
    const bool ok = mbar_wait(sync_bar, sync_n & 1, ctl);
    ++sync_n;
    return __all_sync(0xffffffffu, ok);
  };
  if (r == 0) {
    int n = 0;
    for (int c = 0; c < DV; ++c)
      if (bad[c]) list[n++] = c;
  }
  int nbad = 0;
  for (int c = 0; c < DV; ++c) nbad += bad[c];
  const bool kin = nk > 0;   // this thread's key (nk = 0 exactly for rows past the chunk)
#pragma unroll 1
  for (int g0 = 0; g0 < nbad; g0 += kG) {
    const int ng = min(kG, nbad - g0);
    if (!sync()) return -1;   // the list written; the previous group's readers done
    // key side: thread r = key s
    {
      float ls[kG], vs[kG];
#pragma unroll
      for (int j = 0; j < kG; ++j) {
        const int c = j < ng ? list[g0 + j] : 0;
        ls[j] = j < ng && kin ? LtK[(size_t)c * N + r] : 0.f;
        vs[j] = j < ng && kin ? bf2f(vk[(size_t)r * vrs + c]) : 0.f;
      }
#pragma unroll
      for (int j = 0; j < kG; ++j) {
        if (j < ng) {   // uniform
          float lm = kin ? ls[j] : -INFINITY, ln = kin ? ls[j] : INFINITY;
#pragma unroll
          for (int o = 1; o < 8; o <<= 1) {
            lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, o));
            ln = fminf(ln, __shfl_xor_sync(0xffffffffu, ln, o));
          }
          const bool any = lm >= ln;   // the sub-block holds a key
          const float rho = any ? 0.5f * (lm + ln) : 0.f, sp = any ? lm - ln : 0.f;
          sw[j * BN + r] = kin && sp <= 88.f ? ex2((rho - ls[j]) * LOG2E) * vs[j] : 0.f;
          if ((lane & 7) == 0) {
            slb[j * kSB + r / 8] = rho;
            ssp[j * kSB + r / 8] = sp;
            slm[j * kSB + r / 8] = lm;
          }
        }
      }
    }
    // row side: thread r = row t; its L_t and sums live in shared memory
    // ([j][row], conflict-free), so that the loops below stay rolled (one
    // short code copy)
    {
      float lt[kG];
#pragma unroll
      for (int j = 0; j < kG; ++j) lt[j] = j < ng ? Lrow[list[g0 + j]] : 0.f;
#pragma unroll
      for (int j = 0; j < kG; ++j) {
        slt[j * BM + r] = lt[j];
        sacc[j * BM + r] = 0.f;
      }
    }
    if (!sync()) return -1;
    // a sub-block of 8 keys at a time: its P_ts from the logits in TMEM
#pragma unroll 1
    for (int blk = 0; blk < kSB; ++blk) {
      const int b = blk * 8;
      if (!__any_sync(0xffffffffu, b < nk)) break;     // the warp's rows all lie above
      uint32_t x8[8];
      tmem_ld8_wait(sbase + b, x8);
      if (b >= nk) continue;                            // every key above the diagonal
      float pv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) pv[e] = b + e < nk ? ex2(__uint_as_float(x8[e]) * c1 - moff) : 0.f;
#pragma unroll 1
      for (int j = 0; j < ng; ++j) {
        const float lt = slt[j * BM + r];
        if (lt - slm[j * kSB + blk] < -104.f) continue;   // every term flushes to zero
        const float lbv = slb[j * kSB + blk];
        float add;
        if (ssp[j * kSB + blk] <= 88.f && lt - lbv <= 44.f) {
          const float4 w0 = *reinterpret_cast<const float4*>(sw + j * BN + b);
          const float4 w1 = *reinterpret_cast<const float4*>(sw + j * BN + b + 4);
          const float part = pv[0] * w0.x + pv[1] * w0.y + pv[2] * w0.z + pv[3] * w0.w +
                             pv[4] * w1.x + pv[5] * w1.y + pv[6] * w1.z + pv[7] * w1.w;
          add = ex2((lt - lbv) * LOG2E) * part;
        } else {
          const int c = list[g0 + j];
          add = 0.f;
#pragma unroll 1
          for (int e = 0; e < 8; ++e) {
            const int key = b + e;
            if (key < nk)
              add += pv[e] * ex2((lt - LtK[(size_t)c * N + key]) * LOG2E) * bf2f(vk[(size_t)key * vrs + c]);
          }
        }
        sacc[j * BM + r] += add;
      }
    }
    // into A, a column per channel
#pragma unroll 1
    for (int j = 0; j < ng; ++j) {
      const uint32_t col = acol + (uint32_t)list[g0 + j];
      const float a = __uint_as_float(tmem_ld1(col));
      tmem_wait_ld();
      tmem_st1(col, __float_as_uint(ex2(slt[j * BM + r] * LOG2E) * a + sacc[j * BM + r]));
    }
    tmem_wait_st();
  }
  // the staging area goes back to the P_lo staging of pass 2 once every
  // thread is done with the last group
  if (!sync()) return -1;
  return sync_n;
}

// 11 warps, one CTA per SM.  Each SM sub-partition holds 16,384 registers
// and takes every fourth warp, so three of them hold three warps: at most
// 168 registers a thread.
template <int DK, int DV>
__global__ void __maxnreg__(168)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_vt, const __grid_constant__ CUtensorMap tm_vm,
                  const __grid_constant__ CUtensorMap tm_vml, const Params P) {
  using Lay = Layout<DK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const Dims& d = P.d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int rounds = (P.ntiles + G - 1) / G;
  const size_t vrs = (size_t)d.Hkv * DV;

  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem + Lay::kQ);
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem + Lay::kK);
  __nv_bfloat16* sV = reinterpret_cast<__nv_bfloat16*>(smem + Lay::kV);
  __nv_bfloat16* sVl = reinterpret_cast<__nv_bfloat16*>(smem + Lay::kVl);
  float* sF = reinterpret_cast<float*>(smem + Lay::kF);
  int* sBad = reinterpret_cast<int*>(smem + Lay::kBad);
  int* sAnyBad = reinterpret_cast<int*>(smem + Lay::kAnyBad);
  float* sRows = reinterpret_cast<float*>(smem + Lay::kRows);
  float* sEC = reinterpret_cast<float*>(smem + Lay::kEC);
  Bars* bar = reinterpret_cast<Bars*>(smem + Lay::kBars);
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + Lay::kTmem);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + Lay::kAbort);
  const Ctl ctl{P.status, sAbort, P.stall ? 1000000ull : kWaitTimeoutNs};

  // ---------------------------------------------------------------- setup
  if (tid == 0) {
    *sAbort = 0;
    mbar_init(&bar->q_full, 1);
    mbar_init(&bar->q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
      mbar_init(&bar->v_ready[s], kVsThreads);
      mbar_init(&bar->s_full[s], 1);
      mbar_init(&bar->p_full[s], 128);
      mbar_init(&bar->acc_full[s], 1);
      mbar_init(&bar->acc_empty[s], 256);
      mbar_init(&bar->fold_ready[s], kVsThreads);
      mbar_init(&bar->rows_ready[s], 128);
    }
    mbar_init(&bar->vlo_empty, 1 + 256);   // the diagonal MMAs, then the epilogue
    mbar_init(&bar->pv_done, 1);
    mbar_init(&bar->drain, 1);
    mbar_init(&bar->xs_sync, 128);
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(sTmem, kTmemCols);
  if (tid >= 192 && tid - 192 < DV)
    reinterpret_cast<float*>(smem + Lay::kEpiW)[tid - 192] =
        (P.w && !d.no_norm) ? bf2f(P.w[tid - 192]) : 1.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;

  // ---------------------------------------------------------------- epilogue
  // The epilogue of a tile is shared by the softmax warps (group 0, channels
  // [0, DV/2)) and the V-scaling warps (group 1, [DV/2, DV)): a thread per
  // tile row (its TMEM lane), row r = 32 (warp % 4) + lane in both groups.
  // Pass 1 forms o = alpha exp(L - rho) A (A holds the s = t term too; no row
  // factor for out-of-range channels), writes it back over A and sums its
  // squares; the two halves' sums meet in shared memory; pass 2 writes y and
  // the saved o.  Its stores go through a per-warp staging tile in shared
  // memory (the diagonal's Vm lo buffer, free from the tile's last MMA until
  // the epilogue releases it): written a row per thread, read back a row per
  // 8 lanes, so that every global store covers whole 128-byte lines.  Both
  // groups call it for every tile they take, also after a failed wait (ok_in
  // false): its first named barrier (id 1, both groups) votes, so that both
  // groups leave together.
  float* sSS = reinterpret_cast<float*>(smem + Lay::kSS);
  const float* sW = reinterpret_cast<const float*>(smem + Lay::kEpiW);
  const size_t ors = (size_t)d.Hq * DV;
  constexpr int kU = DV / 32;          // 32-channel chunks
  constexpr int kUH = kU / 2;          // chunks per group
  auto epilogue = [&](const Tile& x, int tb, int grpid, bool ok_in, float alpha, float mt,
                      float lsum) -> bool {
    if (!wg_and(1, 256, ok_in)) return false;
    tc_fence_after();
    const int r = (warp & 3) * 32 + lane;
    const uint32_t acol = tmem + ((uint32_t)((warp & 3) * 32) << 16) + 256u + (uint32_t)(tb * DV);
    const bool valid = r < x.len;
    const size_t tk = (size_t)x.tok0 + (valid ? r : 0);
    // L of this row, channel-major: for a channel, the warp's 32 rows are 32
    // consecutive floats
    const float* Lr = P.Lt + (size_t)x.kv * DV * d.N + tk;
    const float* ec = sEC + tb * DV;
    const int u0 = grpid * kUH;
    float ss = 0.f;
    // all of this group's L loads in flight at once (the tile's L was pulled
    // into L2 when the tile began)
#pragma unroll 1
    for (int h = 0; h < kUH; ++h) {
      const int u = u0 + h;
      float le[1][32];
#pragma unroll
      for (int e = 0; e < 32; ++e) le[0][e] = Lr[(size_t)(u * 32 + e) * d.N];
      uint32_t xa[32];
      tmem_ld32(acol + u * 32, xa);
      tmem_wait_ld(xa);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        // exp2(L log2e - rho log2e), or 1 for an out-of-range channel (NaN
        // in its slot); the same shared-memory word across the warp
        const float b = ec[u * 32 + e];
        const float f = ex2(fmaf(le[0][e], LOG2E, -b));
        const float o = alpha * (b != b ? 1.f : f) * __uint_as_float(xa[e]);
        ss += o * o;
        xa[e] = __float_as_uint(o);
      }
      tmem_st32(acol + u * 32, xa);
    }
    tmem_wait_st();
    sSS[grpid * BM + r] = ss;
    named_sync(1, 256);
    ss = sSS[r] + sSS[BM + r];
    // the RMSNorm, or without it the softmax denominator: y = o / l; the
    // saved tensors are then o / l, the log-sum-exp and ones
    const float rstd = d.no_norm ? 1.0f / lsum : 1.0f / sqrtf(ss / (float)DV + d.eps);
    // staging tile of this warp: [32 rows][8 float4], float4 q of row i at
    // slot q ^ (i & 7), so that both the row writes and the column reads of
    // eight lanes hit eight different 16-byte bank groups
    float4* stg = reinterpret_cast<float4*>(smem + Lay::kVl) + (warp - 2) * 256;
    const int cq = lane & 7;               // float4 of the row this lane stores
    auto pass2 = [&](int u, const uint32_t (&xo)[32]) {
#pragma unroll
      for (int q = 0; q < 8; ++q)
        stg[lane * 8 + (q ^ (lane & 7))] =
            make_float4(__uint_as_float(xo[4 * q]), __uint_as_float(xo[4 * q + 1]),
                        __uint_as_float(xo[4 * q + 2]), __uint_as_float(xo[4 * q + 3]));
      __syncwarp();
      const int c0 = u * 32 + cq * 4;
      const float w0 = sW[c0], w1 = sW[c0 + 1], w2 = sW[c0 + 2], w3 = sW[c0 + 3];
#pragma unroll 4
      for (int i = 0; i < 8; ++i) {
        const int rr = i * 4 + (lane >> 3);  // row of the warp's 32
        const float rs = __shfl_sync(0xffffffffu, rstd, rr);
        const float4 o = stg[rr * 8 + (cq ^ (rr & 7))];
        const int row = (warp & 3) * 32 + rr;
        if (row < x.len) {
          const size_t at = ((size_t)x.tok0 + row) * ors + (size_t)x.h * DV + c0;
          if (P.o_s) {
            const float so = d.no_norm ? rs : 1.f;
            *reinterpret_cast<float4*>(P.o_s + at) = make_float4(o.x * so, o.y * so, o.z * so, o.w * so);
          }
          float y0 = o.x * rs * w0, y1 = o.y * rs * w1, y2 = o.z * rs * w2, y3 = o.w * rs * w3;
          if (P.z) {
            const uint2 z2 = *reinterpret_cast<const uint2*>(P.z + at);
            y0 *= swish(__uint_as_float(z2.x << 16));
            y1 *= swish(__uint_as_float(z2.x & 0xFFFF0000u));
            y2 *= swish(__uint_as_float(z2.y << 16));
            y3 *= swish(__uint_as_float(z2.y & 0xFFFF0000u));
          }
          if (P.y_f32)
            *reinterpret_cast<float4*>(reinterpret_cast<float*>(P.y) + at) = make_float4(y0, y1, y2, y3);
          else
            *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(P.y) + at) =
                make_uint2(pack_bf16(y0, y1), pack_bf16(y2, y3));
        }
      }
      __syncwarp();   // the tile is rewritten by the next chunk
    };
#pragma unroll 1
    for (int u = u0; u < u0 + kUH; ++u) {
      // pass 2 from o in TMEM
      uint32_t xa[32];
      tmem_ld32(acol + u * 32, xa);
      tmem_wait_ld(xa);
      pass2(u, xa);
    }
    if (grpid == 0 && P.o_s && valid) {
      P.m_s[tk * d.Hq + x.h] = d.no_norm ? mt + logf(lsum) : mt;
      P.rstd_s[tk * d.Hq + x.h] = d.no_norm ? 1.f : rstd;
    }
    tc_fence_before();
    mbar_arrive(&bar->acc_empty[tb]);
    // the staging tiles go back to the next diagonal's Vm lo (a TMA write)
    fence_proxy_async_smem();
    mbar_arrive(&bar->vlo_empty);
    return true;
  };

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer: Q, K
    if (lane == 0) {
      int kc = 0, nq = 0;
      bool ok = !P.stall;   // a stalled producer (test builds) issues nothing
      for (int round = 0; ok && round < rounds; ++round) {
        const int t = tile_of(round, G, cta);
        if (t >= P.ntiles) continue;
        const Tile x = tile_info(P, t);
        if (x.len <= 0) continue;
        // Q of this tile once the previous tile's last QK^T has completed
        if (nq > 0 && !mbar_wait(&bar->q_empty, (nq - 1) & 1, ctl)) { ok = false; break; }
        mbar_expect_tx(&bar->q_full, BM * DK * 2);
        for (int hh = 0; hh < DK / 64; ++hh)
          tma_load_3d(sQ + hh * BM * 64, &tm_q, &bar->q_full, hh * 64, x.h, x.tok0);
        ++nq;
        for (int it = 0; it < x.nblk; ++it) {
          const bool diag = it == x.nblk - 1;
          const int j = diag ? x.j : x.j - 1 - it;
          const int ktok = x.seq0 + j * BN;
          const int st = kc & 1;
          if (kc >= 2 && !mbar_wait(&bar->k_empty[st], ((kc >> 1) & 1) ^ 1, ctl)) { ok = false; break; }
          mbar_expect_tx(&bar->k_full[st], BN * DK * 2);
          for (int hh = 0; hh < DK / 64; ++hh)
            tma_load_3d(sK + st * BN * DK + hh * BN * 64, &tm_k, &bar->k_full[st], hh * 64, x.kv, ktok);
          ++kc;
        }
      }
      // every issued copy must land before the CTA may exit (also after an
      // abort): wait for the last one or two issued per ring, timeout only
      const Ctl drain{P.status, nullptr, ctl.limit_ns};
      for (int n = kc - 1; n >= 0 && n >= kc - 2; --n) mbar_wait(&bar->k_full[n & 1], (n >> 1) & 1, drain);
      if (nq > 0) mbar_wait(&bar->q_full, (nq - 1) & 1, drain);
    }
  } else if (warp == 10) {
    // ------------------------------------------- TMA producer: V (Vt or Vm hi), Vm lo
    // (its own warp, so that the K ring runs ahead of the V ring's waits)
    if (lane == 0) {
      int vc = 0, ndiag = 0;
      bool ok = !P.stall;
      for (int round = 0; ok && round < rounds; ++round) {
        const int t = tile_of(round, G, cta);
        if (t >= P.ntiles) continue;
        const Tile x = tile_info(P, t);
        if (x.len <= 0) continue;
        for (int it = 0; it < x.nblk; ++it) {
          const bool diag = it == x.nblk - 1;
          const int j = diag ? x.j : x.j - 1 - it;
          const int ktok = x.seq0 + j * BN;
          const int sv = vc & 1;
          if (vc >= 2 && !mbar_wait(&bar->v_empty[sv], ((vc >> 1) & 1) ^ 1, ctl)) { ok = false; break; }
          if (diag && ndiag > 0 && !mbar_wait(&bar->vlo_empty, (ndiag - 1) & 1, ctl)) { ok = false; break; }
          mbar_expect_tx(&bar->v_full[sv], (diag ? 2 : 1) * BN * DV * 2);
          const CUtensorMap* vmap = diag ? &tm_vm : &tm_vt;
          for (int hh = 0; hh < DV / 64; ++hh)
            tma_load_3d(sV + sv * BN * DV + hh * BN * 64, vmap, &bar->v_full[sv], hh * 64, x.kv, ktok);
          if (diag) {
            for (int hh = 0; hh < DV / 64; ++hh)
              tma_load_3d(sVl + hh * BN * 64, &tm_vml, &bar->v_full[sv], hh * 64, x.kv, ktok);
            ++ndiag;
          }
          ++vc;
        }
      }
      const Ctl drain{P.status, nullptr, ctl.limit_ns};
      for (int n = vc - 1; n >= 0 && n >= vc - 2; --n) mbar_wait(&bar->v_full[n & 1], (n >> 1) & 1, drain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(BM, BN, false, false);
      constexpr uint32_t idesc_off = idesc_bf16(BM, DV, false, true, true);   // fp16 P V''
      constexpr uint32_t idesc_diag = idesc_bf16(BM, DV, false, true);        // bf16 hi/lo
      const uint32_t q_addr = smem_u32(sQ);
      // the PV of block g - 1 is issued right after the QK^T of block g
      struct Pend {
        int g, it, vc, ab, use;
        bool diag, valid;
      } pend{0, 0, 0, 0, 0, false, false};
      int g = 0, kc = 0, vc = 0, nt = 0;
      bool ok = true;
      auto issue_pv = [&](const Pend& pb) -> bool {
        const int b = pb.g & 1, sv = pb.vc & 1;
        if (!mbar_wait(&bar->p_full[b], (pb.g >> 1) & 1, ctl)) return false;
        if (!mbar_wait(&bar->v_ready[sv], (pb.vc >> 1) & 1, ctl)) return false;
        // the tile's first PV overwrites A: the epilogue of the tile that
        // used this buffer before must have released it
        if (pb.it == 0 && pb.use >= 1 && !mbar_wait(&bar->acc_empty[pb.ab], (pb.use - 1) & 1, ctl))
          return false;
        tc_fence_after();
        const uint32_t acol = tmem + 256u + (uint32_t)(pb.ab * DV);
        const uint32_t scol = tmem + col_s(b);
        const uint32_t v_addr = smem_u32(sV + sv * BN * DV);
        if (!pb.diag) {
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t bd = desc_add(desc_sw128(v_addr, BN * 128, 1024), kk * 2048);
            mma_ts(acol, scol + kk * 8, bd, idesc_off, (pb.it > 0 || kk > 0));
          }
        } else {
          // A holds the folded earlier blocks, or (first block of a chunk-0
          // tile) what the softmax warps wrote: always accumulate
          const uint32_t vl_addr = smem_u32(sVl);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t bh = desc_add(desc_sw128(v_addr, BN * 128, 1024), kk * 2048);
            const uint64_t bl = desc_add(desc_sw128(vl_addr, BN * 128, 1024), kk * 2048);
            mma_ts(acol, scol + kk * 8, bh, idesc_diag, 1);
            mma_ts(acol, scol + 64 + kk * 8, bh, idesc_diag, 1);
            mma_ts(acol, scol + kk * 8, bl, idesc_diag, 1);
          }
        }
        tc_commit(&bar->v_empty[sv]);
        tc_commit(&bar->pv_done);
        if (pb.diag) {
          tc_commit(&bar->acc_full[pb.ab]);
          tc_commit(&bar->vlo_empty);
        }
        return true;
      };
      for (int round = 0; ok && round < rounds; ++round) {
        const int t = tile_of(round, G, cta);
        if (t >= P.ntiles) continue;
        const Tile x = tile_info(P, t);
        if (x.len <= 0) continue;
        const int ab = nt & 1, use = nt >> 1;
        if (!mbar_wait(&bar->q_full, nt & 1, ctl)) { ok = false; break; }
        for (int it = 0; it < x.nblk; ++it) {
          const bool diag = it == x.nblk - 1;
          const int b = g & 1, st = kc & 1;
          if (!mbar_wait(&bar->k_full[st], (kc >> 1) & 1, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sK + st * BN * DK);
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk) {
            const uint64_t a = desc_add(desc_sw128(q_addr, 16, 1024), (kk >> 2) * (BM * 128) + (kk & 3) * 32);
            const uint64_t bd = desc_add(desc_sw128(k_addr, 16, 1024), (kk >> 2) * (BN * 128) + (kk & 3) * 32);
            mma_ss(tmem + col_s(b), a, bd, idesc_qk, kk > 0);
          }
          tc_commit(&bar->s_full[b]);
          tc_commit(&bar->k_empty[st]);
          if (diag) tc_commit(&bar->q_empty);
          ++kc;
          if (pend.valid && !issue_pv(pend)) { ok = false; break; }
          pend = Pend{g, it, vc, ab, use, diag, true};
          ++g;
          ++vc;
        }
        ++nt;
      }
      if (ok && pend.valid) issue_pv(pend);
      // TMEM must not be released while an issued MMA may still write it
      tc_commit(&bar->drain);
      mbar_wait(&bar->drain, 0, Ctl{P.status, nullptr, ctl.limit_ns});
    }
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------ softmax
    const int r = (warp & 3) * 32 + lane;              // query row in the tile
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const float c1 = d.scale * LOG2E;
    int g = 0, nt = 0;
    int xs_n = 0;   // meetings on xs_sync so far
    bool ok = true;
    for (int round = 0; ok && round < rounds; ++round) {
      const int t = tile_of(round, G, cta);
      if (t >= P.ntiles) continue;
      const Tile x = tile_info(P, t);
      if (x.len <= 0) continue;
      const int tb = nt & 1, use = nt >> 1;
      const uint32_t acol = lane_base + 256u + (uint32_t)(tb * DV);
      float m_used = -INFINITY, m_true = -INFINITY;
      float l_used = 0.f;   // without the norm: sum of P relative to m_used
      for (int it = 0; it < x.nblk; ++it) {
        const bool diag = it == x.nblk - 1;
        const int b = g & 1;
        const uint32_t sbase = lane_base + col_s(b);
        // waits vote warp-wide: the TMEM accesses below are warp-collective
        if (!__all_sync(0xffffffffu, mbar_wait(&bar->s_full[b], (g >> 1) & 1, ctl))) { ok = false; break; }
        tc_fence_after();
        if (!diag) {
          // One pass: P = exp(S scale - m_used) chunk by chunk (fp16, over the
          // S columns already read), with the next chunk's TMEM load in
          // flight.  The exponentials of a chunk start at once with the
          // current reference, beside its maximum; a chunk whose maximum
          // exceeds m_used by more than the lazy threshold (rare) moves the
          // reference (warp-wide) and is redone: the P already written in
          // this block, the running sum and A (the earlier blocks, once their
          // last PV has completed) are scaled by exp(m_used - m_new).  The
          // tile's first chunk sets the reference from its own maximum.
          float ls = 0.f;
          auto chunk = [&](const uint32_t (&xs)[32], int c4) -> bool {
            // packed pairs: the scaling and the running sum as f32x2; the
            // exponentials on the MUFU unit, or one pair in kPolyPairEvery as a
            // polynomial on the FMA pipe (both well inside fp16's rounding)
            uint32_t pk[16];
            auto expo = [&]() -> float {
              const float moff = m_used * LOG2E;
              const uint64_t c1x2 = f2_pack(c1, c1), mo2 = f2_pack(-moff, -moff);
              uint64_t lsa = f2_pack(0.f, 0.f), lsb = lsa;
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const uint64_t a2 =
                    f2_fma(f2_pack(__uint_as_float(xs[e]), __uint_as_float(xs[e + 1])), c1x2, mo2);
                uint64_t p2;
                if (kPolyPairEvery > 0 && (e >> 1) % kPolyPairEvery == kPolyPairEvery - 1) {
                  p2 = exp2_poly3_x2(a2);
                } else {
                  float a0, a1;
                  f2_unpack(a2, a0, a1);
                  p2 = f2_pack(ex2(a0), ex2(a1));
                }
                if ((e >> 1) & 1) lsb = f2_add(lsb, p2);
                else lsa = f2_add(lsa, p2);
                float p0, p1;
                f2_unpack(p2, p0, p1);
                pk[e >> 1] = pack_f16(p0, p1);
              }
              float s0, s1;
              f2_unpack(f2_add(lsa, lsb), s0, s1);
              return s0 + s1;
            };
            // the chunk maximum, four independent chains
            float m4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) m4[k] = __uint_as_float(xs[k]);
#pragma unroll
            for (int e = 4; e < 32; e += 4)
#pragma unroll
              for (int k = 0; k < 4; ++k) m4[k] = fmaxf(m4[k], __uint_as_float(xs[e + k]));
            const float cm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * d.scale;
            m_true = fmaxf(m_true, cm);
            if (it == 0 && c4 == 0) m_used = m_true;   // the tile's first chunk
            // (one copy of the exponentials: a chunk that moves the reference
            // takes the loop twice, the second time within the threshold)
            float lsc;
            while (true) {
              lsc = expo();
              if (!__any_sync(0xffffffffu, cm > m_used + kRescaleThreshold)) break;
              const float m_new = fmaxf(m_used, m_true);
              const float rr = m_used == -INFINITY ? 0.f : ex2((m_used - m_new) * LOG2E);
              if (c4 > 0) {
                tmem_wait_st();
                const __half2 r2 = __float2half2_rn(rr);
                for (int cp = 0; cp < c4; ++cp) {
                  uint32_t pq[16];
                  tmem_ld16(sbase + cp * 16, pq);
                  tmem_wait_ld();
#pragma unroll
                  for (int e = 0; e < 16; ++e) {
                    __half2 h = *reinterpret_cast<__half2*>(&pq[e]);
                    h = __hmul2(h, r2);
                    pq[e] = *reinterpret_cast<uint32_t*>(&h);
                  }
                  tmem_st16(sbase + cp * 16, pq);
                }
              }
              if (it > 0) {
                // A is quiescent once the previous block's PV has completed
                if (!__all_sync(0xffffffffu, mbar_wait(&bar->pv_done, (g - 1) & 1, ctl))) return false;
                tc_fence_after();
#pragma unroll 1
                for (int cc = 0; cc < DV / 32; ++cc) {
                  uint32_t xa[32];
                  tmem_ld32(acol + cc * 32, xa);
                  tmem_wait_ld(xa);
#pragma unroll
                  for (int e = 0; e < 32; ++e) xa[e] = __float_as_uint(__uint_as_float(xa[e]) * rr);
                  tmem_st32(acol + cc * 32, xa);
                }
              }
              ls *= rr;
              l_used *= rr;
              m_used = m_new;   // this chunk again, with the new reference
            }
            ls += lsc;
            tmem_st16(sbase + c4 * 16, pk);
            return true;
          };
          // two chunks per pass (one code copy each), the next chunk's load
          // in flight while one is computed
          uint32_t xa[32], xb[32];
          tmem_ld32(sbase, xa);
          tmem_wait_ld(xa);
          bool good = true;
#pragma unroll 1
          for (int c4 = 0; c4 < BN / 32; c4 += 2) {
            tmem_ld32(sbase + (c4 + 1) * 32, xb);
            good = chunk(xa, c4);
            tmem_wait_ld(xb);
            if (!good) break;
            if (c4 + 2 < BN / 32) tmem_ld32(sbase + (c4 + 2) * 32, xa);
            good = chunk(xb, c4 + 1);
            if (c4 + 2 < BN / 32) tmem_wait_ld(xa);
            if (!good) break;
          }
          if (!good) {
            tmem_wait_ld();   // no TMEM load may stay in flight
            ok = false;
            break;
          }
          if (d.no_norm) l_used += ls;
        } else {
          // pass 1: the row maximum (diagonal block: keys s <= t)
          float mx = -INFINITY;
#pragma unroll
          for (int c4 = 0; c4 < BN / 32; ++c4) {
            uint32_t xs[32];
            tmem_ld32(sbase + c4 * 32, xs);
            tmem_wait_ld(xs);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int key = c4 * 32 + e;
              mx = key <= r ? fmaxf(mx, __uint_as_float(xs[e])) : mx;
            }
          }
          m_true = fmaxf(m_true, mx * d.scale);
          bool rescale = false;
          if (it == 0) m_used = m_true;
          else rescale = __any_sync(0xffffffffu, m_true > m_used + kRescaleThreshold);
          const bool fold = diag && x.nblk > 1;
          // the fold factors and out-of-range flags of this tile
          if (diag && !__all_sync(0xffffffffu, mbar_wait(&bar->fold_ready[tb], use & 1, ctl))) { ok = false; break; }
          if (rescale || fold) {
            // A must be quiescent: the previous block's PV has completed
            if (!__all_sync(0xffffffffu, mbar_wait(&bar->pv_done, (g - 1) & 1, ctl))) { ok = false; break; }
            tc_fence_after();
            const float a_r = rescale ? ex2((m_used - m_true) * LOG2E) : 1.f;
            const float* F = sF + tb * DV;
#pragma unroll 1
            for (int cc = 0; cc < DV / 32; ++cc) {
              uint32_t xa[32];
              tmem_ld32(acol + cc * 32, xa);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const float f = fold ? F[cc * 32 + e] * a_r : a_r;
                xa[e] = __float_as_uint(__uint_as_float(xa[e]) * f);
              }
              tmem_st32(acol + cc * 32, xa);
            }
            tmem_wait_st();
            if (rescale) {
              m_used = m_true;
              l_used *= a_r;
            }
          }
          if (diag && x.nblk == 1) {
            // chunk 0: the diagonal MMAs accumulate into A, which starts at
            // zero here; the epilogue of the tile that used it before must be
            // done with it
            if (use >= 1 && !__all_sync(0xffffffffu, mbar_wait(&bar->acc_empty[tb], (use - 1) & 1, ctl))) {
              ok = false;
              break;
            }
            tc_fence_after();
            uint32_t z[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) z[e] = 0u;
#pragma unroll
            for (int cc = 0; cc < DV / 32; ++cc) tmem_st32(acol + cc * 32, z);
            tmem_wait_st();
          }
          const float moff = m_used * LOG2E;
          if (diag && sAnyBad[tb]) {
            const size_t rowL = ((size_t)x.tok0 + (r < x.len ? r : 0)) * vrs + (size_t)x.kv * DV;
            xs_n = diag_exact_sums<DK, DV>(P.L + rowL, P.Lt + (size_t)x.kv * DV * d.N + x.tok0, d.N,
                                           P.v + (size_t)x.tok0 * vrs + (size_t)x.kv * DV, (int)vrs,
                                           smem, tb, r < x.len ? r + 1 : 0, r, sbase, acol, c1, moff,
                                           xs_n, P.status);
            if (xs_n < 0) {
              ok = false;
              break;
            }
          }
          // pass 2: P, written over the S columns already read
          {
            // strictly causal P as bf16 hi (columns [0, 64)) + lo ([64, 128));
            // lo parts are stored only over S columns already read: those of
            // key chunks 0 and 1 (staged in shared memory meanwhile) after
            // chunk 2 is read, those of 2 and 3 after chunk 3
            uint32_t* plo = reinterpret_cast<uint32_t*>(smem + Lay::kPlo) + r * 33;
            uint32_t plo2[16];
#pragma unroll 1
            for (int c4 = 0; c4 < BN / 32; ++c4) {
              uint32_t xs[32], ph[16], pl[16];
              tmem_ld32(sbase + c4 * 32, xs);
              tmem_wait_ld(xs);
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const int key = c4 * 32 + e;
                const float p0 = key <= r ? ex2(__uint_as_float(xs[e]) * c1 - moff) : 0.f;
                const float p1 = key + 1 <= r ? ex2(__uint_as_float(xs[e + 1]) * c1 - moff) : 0.f;
                if (d.no_norm) l_used += p0 + p1;
                ph[e >> 1] = pack_bf16(p0, p1);
                const float h0 = __uint_as_float(ph[e >> 1] << 16);
                const float h1 = __uint_as_float(ph[e >> 1] & 0xFFFF0000u);
                pl[e >> 1] = pack_bf16(p0 - h0, p1 - h1);
              }
              tmem_st16(sbase + c4 * 16, ph);
              if (c4 < 2) {
#pragma unroll
                for (int e = 0; e < 16; ++e) plo[c4 * 16 + e] = pl[e];
              } else if (c4 == 2) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  uint32_t t16[16];
#pragma unroll
                  for (int e = 0; e < 16; ++e) t16[e] = plo[h * 16 + e];
                  tmem_st16(sbase + 64 + h * 16, t16);
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) plo2[e] = pl[e];
              } else {
                tmem_st16(sbase + 96, plo2);
                tmem_st16(sbase + 112, pl);
              }
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar->p_full[b]);
        ++g;
      }
      // per-row results of the tile, for the V-scaling warps' half of its
      // epilogue, then this group's half once the diagonal PV has completed
      float* rows = sRows + tb * 4 * BM;
      const float alpha = ex2((m_used - m_true) * LOG2E);
      if (ok) {
        rows[r] = alpha;
        rows[2 * BM + r] = m_true;
        rows[3 * BM + r] = alpha * l_used;                         // l (no norm)
        mbar_arrive(&bar->rows_ready[tb]);
        ok = __all_sync(0xffffffffu, mbar_wait(&bar->acc_full[tb], use & 1, ctl));
      }
      ok = epilogue(x, tb, 0, ok, alpha, m_true, alpha * l_used);
      ++nt;
    }
  } else if (warp >= 6 && warp < 10) {
    // ------------------------------------------------------------ V scaling
    const int dt = tid - 192;                        // 0..127
    constexpr int kChunks = DV / 8;                  // 16-byte chunks per row
    constexpr int kRowsPerPass = kVsThreads / kChunks;
    const int lc = dt % kChunks;                     // logical chunk: channels lc*8 .. +7
    const int r0 = dt / kChunks;
    const int half = lc >> 3, lcc = lc & 7;
    int vc = 0, nt = 0;
    bool ok = true;
    for (int round = 0; ok && round < rounds; ++round) {
      const int t = tile_of(round, G, cta);
      if (t >= P.ntiles) continue;
      const Tile x = tile_info(P, t);
      if (x.len <= 0) continue;
      const int tb = nt & 1, use = nt >> 1;
      // (a failed wait ends the tile's work: break leaves this block, and
      // the epilogue below is still entered, to vote)
      do {
      // pull the tile's L (channel-major) into L2 for its epilogue
      if (dt < DV) {
        const char* lp = reinterpret_cast<const char*>(P.Lt + ((size_t)x.kv * DV + dt) * d.N + x.tok0);
        for (int b = 0; b < x.len * 4; b += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(lp + b));
      }
      // the fold factors of two tiles ago are consumed once its diagonal PV
      // has completed (it follows the fold)
      // (every wait of this warpgroup ends in a vote on a named barrier, so
      // that all its threads leave together after an abort)
      if (!wg_and(2, kVsThreads, use < 1 || mbar_wait(&bar->acc_full[tb], (use - 1) & 1, ctl))) { ok = false; break; }
      // tile-wide power-of-two scale k_c of the earlier blocks' operands:
      // not needed (0) when every earlier chunk is fp16-safe (g <= 0)
      int my_safe = 1;
      for (int jj = dt; jj < x.nblk - 1; jj += kVsThreads) my_safe &= P.safe[(size_t)(x.first + jj) * d.Hkv + x.kv];
      const int tile_safe = wg_and(2, kVsThreads, my_safe);
      float kexp[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) kexp[e] = 0.f;
      if (!tile_safe) {
        float delta[8], kmax[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          delta[e] = 0.f;
          kmax[e] = -1e30f;
        }
        for (int it = 0; it < x.nblk - 1; ++it) {
          const int j = x.j - 1 - it;
          if (it >= 1) {
            const float* tp = P.tot + ((size_t)(x.first + j + 1) * d.Hkv + x.kv) * DV + lc * 8;
#pragma unroll
            for (int e = 0; e < 8; ++e) delta[e] += tp[e];
          }
          const float* lv = P.lvt + ((size_t)(x.first + j) * d.Hkv + x.kv) * DV + lc * 8;
#pragma unroll
          for (int e = 0; e < 8; ++e) kmax[e] = fmaxf(kmax[e], lv[e] + delta[e] * LOG2E);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) kexp[e] = kmax[e] > 15.f ? ceilf(kmax[e] - 15.f) : 0.f;
      }
      if (r0 == 0) {
        const size_t ti = ((size_t)x.ci * d.Hkv + x.kv) * DV + lc * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const bool bad = P.hr[ti + e] > FIX_HR_MAX;
          const float rho = P.rho[ti + e];
          sF[tb * DV + lc * 8 + e] = ex2(rho * LOG2E + kexp[e]);
          sBad[tb * DV + lc * 8 + e] = bad ? 1 : 0;
          // the epilogue's row factor exp(L - rho), or none (out of range)
          sEC[tb * DV + lc * 8 + e] = bad ? __int_as_float(0x7fc00000) : rho * LOG2E;
        }
      }
      {
        int my_bad = 0;
        if (r0 == 0) {
          const size_t ti = ((size_t)x.ci * d.Hkv + x.kv) * DV + lc * 8;
#pragma unroll
          for (int e = 0; e < 8; ++e) my_bad |= P.hr[ti + e] > FIX_HR_MAX ? 1 : 0;
        }
        const int any = wg_or(2, kVsThreads, my_bad);
        if (dt == 0) sAnyBad[tb] = any;
      }
      mbar_arrive(&bar->fold_ready[tb]);
      float delta[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) delta[e] = 0.f;
      // the per-block values (the total of chunk j + 1 that extends the
      // running sum, the exponents of chunk j) are loaded one block ahead
      auto fetch = [&](int it, float4 (&t)[2], float4 (&l)[2]) {
        const int j = x.j - 1 - it;
        const bool off = it < x.nblk - 1;
        const size_t cb = (size_t)x.kv * DV + lc * 8;
        if (off && it >= 1) {
          const float4* tp = reinterpret_cast<const float4*>(P.tot + (size_t)(x.first + j + 1) * d.Hkv * DV + cb);
          t[0] = tp[0];
          t[1] = tp[1];
        } else {
          t[0] = t[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (off) {
          const float4* lp = reinterpret_cast<const float4*>(P.lvt + (size_t)(x.first + j) * d.Hkv * DV + cb);
          l[0] = lp[0];
          l[1] = lp[1];
        } else {
          l[0] = l[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      };
      float4 tcur[2], lcur[2];
      fetch(0, tcur, lcur);
      for (int it = 0; it < x.nblk; ++it) {
        const bool diag = it == x.nblk - 1;
        const int sv = vc & 1;
        float4 tnxt[2], lnxt[2];
        if (!diag) fetch(it + 1, tnxt, lnxt);
        float f8[8];
        if (!diag) {
          const float t8[8] = {tcur[0].x, tcur[0].y, tcur[0].z, tcur[0].w, tcur[1].x, tcur[1].y, tcur[1].z, tcur[1].w};
          const float l8[8] = {lcur[0].x, lcur[0].y, lcur[0].z, lcur[0].w, lcur[1].x, lcur[1].y, lcur[1].z, lcur[1].w};
          // Vt is stored as fp16 times 2^-e; V'' = Vt_true f_ij 2^-k
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            delta[e] += t8[e];
            f8[e] = ex2(delta[e] * LOG2E + vt_exponent(l8[e]) - kexp[e]);
          }
        }
        // Factors no larger than 2 (always with g <= 0) go to fp16: V'' = Vt f
        // is then one packed fp16 multiply per channel pair, with no
        // conversion.  A factor below fp16's normal range (2^-14) loses
        // relative precision or becomes 0, but then every value it scales is
        // already below 2^-14 of its undecayed size, an absolute error under
        // 2^-24 |v|.  Factors that are all exactly 1 leave Vt as it is;
        // larger ones take the fp32 path.
        bool h16 = true, unit = true;
        __half2 fh[4];
        if (!diag) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            h16 = h16 && f8[2 * u] <= 2.f && f8[2 * u + 1] <= 2.f;
            unit = unit && f8[2 * u] == 1.f && f8[2 * u + 1] == 1.f;
            fh[u] = __floats2half2_rn(f8[2 * u], f8[2 * u + 1]);
          }
        }
        if (!wg_and(2, kVsThreads, mbar_wait(&bar->v_full[sv], (vc >> 1) & 1, ctl))) { ok = false; break; }
        if (!diag && !unit) {
          uint8_t* vb = reinterpret_cast<uint8_t*>(sV + sv * BN * DV) + half * (BN * 128);
          // rows in batches of 8: all loads of a batch before its stores (the
          // compiler cannot move a load above a store to the same array)
          constexpr int kBatch = 8;
          static_assert((BN / kRowsPerPass) % kBatch == 0, "row batches");
#pragma unroll 1
          for (int s0 = r0; s0 < BN; s0 += kBatch * kRowsPerPass) {
            uint4 xv[kBatch];
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
              const int s = s0 + i * kRowsPerPass;
              xv[i] = *reinterpret_cast<const uint4*>(vb + s * 128 + ((lcc ^ (s & 7)) << 4));
            }
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
              uint32_t w4[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                if (h16) {
                  __half2 h = __hmul2(*reinterpret_cast<const __half2*>(&w4[u]), fh[u]);
                  w4[u] = *reinterpret_cast<uint32_t*>(&h);
                } else {
                  const float2 ab = __half22float2(*reinterpret_cast<const __half2*>(&w4[u]));
                  w4[u] = pack_f16(ab.x * f8[2 * u], ab.y * f8[2 * u + 1]);
                }
              }
              xv[i] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
              const int s = s0 + i * kRowsPerPass;
              *reinterpret_cast<uint4*>(vb + s * 128 + ((lcc ^ (s & 7)) << 4)) = xv[i];
            }
          }
          fence_proxy_async_smem();
        }
        mbar_arrive(&bar->v_ready[sv]);
        ++vc;
        if (!diag) {
          tcur[0] = tnxt[0]; tcur[1] = tnxt[1];
          lcur[0] = lnxt[0]; lcur[1] = lnxt[1];
        }
      }
      } while (false);
      // this group's half of the tile's epilogue: the softmax warps' per-row
      // results and the diagonal PV come first
      float alpha = 0.f, mt = 0.f, lsum = 1.f;
      if (ok) {
        ok = wg_and(2, kVsThreads, mbar_wait(&bar->rows_ready[tb], use & 1, ctl) &&
                                       mbar_wait(&bar->acc_full[tb], use & 1, ctl));
        const float* rows = sRows + tb * 4 * BM;
        const int rr = (warp & 3) * 32 + lane;
        alpha = rows[rr];
        mt = rows[2 * BM + rr];
        lsum = rows[3 * BM + rr];
      }
      ok = epilogue(x, tb, 1, ok, alpha, mt, lsum);
      ++nt;
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

// [N, H, D] 16-bit viewed as a 3-D tensor (D, H, N); box = 64 x 1 x 128 rows,
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

static int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
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
  if (prm.ntiles <= 0) return FIX_OK;
  static int sms = 0;   // one CTA per SM, persistent
  if (!sms) sms = num_sms();
  const int grid = prm.ntiles < sms ? prm.ntiles : sms;
  kern<<<(unsigned)grid, kThreads, smem, st>>>(mq, mk, mvt, mvm, mvml, prm);
  return launch_status();
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
                  const float* L, const float* Lt, const float* tot, const float* rho, const float* hr,
                  const float* lvt, const int* safe,
                  const void* w, const void* z, void* y, bool y_f32, float* o_s, float* m_s,
                  float* rstd_s, int* status, cudaStream_t st) {
  tcf::Params prm{};
  prm.d = d;
  prm.chunks = chunks;
  prm.order = order;
  const long long nt = (long long)d.nchunks * d.Hq;
  if (nt > (1LL << 30)) return FIX_ERR_SHAPE;
  prm.ntiles = (int)nt;
  prm.q = static_cast<const __nv_bfloat16*>(q);
  prm.k = static_cast<const __nv_bfloat16*>(k);
  prm.v = static_cast<const __nv_bfloat16*>(v);
  prm.L = L;
  prm.Lt = Lt;
  prm.tot = tot;
  prm.rho = rho;
  prm.hr = hr;
  prm.lvt = lvt;
  prm.safe = safe;
  prm.w = static_cast<const __nv_bfloat16*>(w);
  prm.z = static_cast<const __nv_bfloat16*>(z);
  prm.y = y;
  prm.y_f32 = y_f32 ? 1 : 0;
  prm.o_s = o_s;
  prm.m_s = m_s;
  prm.rstd_s = rstd_s;
  prm.status = status;
#ifdef FIX_TEST_HOOKS
  prm.stall = test_stall_forward();
#endif
  if (d.Dk == 128 && d.Dv == 128) return tcf::launch<128, 128>(prm, q, k, vt, vm, vml, st);
  if (d.Dk == 64 && d.Dv == 64) return tcf::launch<64, 64>(prm, q, k, vt, vm, vml, st);
  if (d.Dk == 128 && d.Dv == 64) return tcf::launch<128, 64>(prm, q, k, vt, vm, vml, st);
  if (d.Dk == 64 && d.Dv == 128) return tcf::launch<64, 128>(prm, q, k, vt, vm, vml, st);
  return FIX_ERR_HEAD_DIM;
}

}  // namespace fix
