// Host side of the FiX attention C ABI (include/fix_attn.h): argument
// validation, workspace layout, the packed-sequence chunk schedule (built
// here from the host mirror of cu_seqlens and uploaded through kernel
// parameters) and the kernel launches.  Nothing here allocates device memory
// or synchronises.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "fix_attn.h"
#include "fix_common.cuh"
#include "fix_internal.h"

namespace fix {

static inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static bool head_dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates the problem descriptor and fills the kernel-side dims.
static fix_status make_dims(const fix_attn_problem* p, Dims* d);
fix_status validate_problem(const fix_attn_problem* p, Dims* d) { return make_dims(p, d); }
static fix_status make_dims(const fix_attn_problem* p, Dims* d) {
  if (!p) return FIX_ERR_NULL;
  if (p->flags & ~(FIX_FLAG_REUSE_FWD_WORKSPACE | FIX_FLAG_NO_NORM | FIX_FLAG_SCALAR_GATE))
    return FIX_ERR_SHAPE;
  if (p->y_dtype != FIX_DTYPE_BF16 && p->y_dtype != FIX_DTYPE_F32) return FIX_ERR_DTYPE;
  if (p->algo < FIX_ALGO_AUTO || p->algo > FIX_ALGO_TC) return FIX_ERR_DTYPE;
  if (p->batch < 1 || p->seqlen < 0 || p->num_q_heads < 1 || p->num_kv_heads < 1)
    return FIX_ERR_SHAPE;
  if (!head_dim_ok(p->head_dim_k) || !head_dim_ok(p->head_dim_v)) return FIX_ERR_HEAD_DIM;
  if (p->num_q_heads % p->num_kv_heads) return FIX_ERR_GQA;
  if (!(p->eps >= 0.f) || !std::isfinite(p->eps)) return FIX_ERR_SHAPE;
  if (!std::isfinite(p->scale)) return FIX_ERR_SHAPE;
  const long long N = (long long)p->batch * p->seqlen;
  if (N > (1LL << 30)) return FIX_ERR_SHAPE;
  if ((long long)N * p->num_q_heads * (p->head_dim_k > p->head_dim_v ? p->head_dim_k : p->head_dim_v) >
      (1LL << 40))
    return FIX_ERR_SHAPE;
  d->N = (int)N;
  d->B = p->batch;
  d->T = p->seqlen;
  d->Hq = p->num_q_heads;
  d->Hkv = p->num_kv_heads;
  d->Dk = p->head_dim_k;
  d->Dv = p->head_dim_v;
  d->grp = p->num_q_heads / p->num_kv_heads;
  d->scale = p->scale > 0.f ? p->scale : 1.0f / std::sqrt((float)p->head_dim_k);
  d->eps = p->eps;
  d->no_norm = (p->flags & FIX_FLAG_NO_NORM) ? 1 : 0;
  d->scalar_gate = (p->flags & FIX_FLAG_SCALAR_GATE) ? 1 : 0;
  long long nch = 0;
  if (p->cu_seqlens) {
    if (p->batch != 1) return FIX_ERR_SHAPE;
    if (!p->cu_seqlens_host || p->num_seqs < 1) return FIX_ERR_CU_SEQLENS;
    const int64_t* c = p->cu_seqlens_host;
    if (c[0] != 0 || c[p->num_seqs] != p->seqlen) return FIX_ERR_CU_SEQLENS;
    for (int i = 0; i < p->num_seqs; ++i) {
      if (c[i + 1] < c[i]) return FIX_ERR_CU_SEQLENS;
      nch += (c[i + 1] - c[i] + FIX_CHUNK - 1) / FIX_CHUNK;
    }
    d->nseq = p->num_seqs;
  } else {
    if (p->num_seqs != 0 || p->cu_seqlens_host) return FIX_ERR_CU_SEQLENS;
    d->nseq = p->batch;
    nch = (long long)p->batch * ((p->seqlen + FIX_CHUNK - 1) / FIX_CHUNK);
  }
  d->nchunks = (int)nch;
  return FIX_OK;
}

// Work split of the dk/dv kernel: each key chunk's tiles (q heads x 64-row
// query tiles) are taken in two kinds, those of the chunk itself (the
// diagonal) and those of the later chunks of its sequence, and each kind is
// cut into runs of at most P tiles, P chosen so that about two runs per SM
// cover the problem.  Every run (part) owns one slot of fp32 partial sums.
// Planned with the B200's 148 SMs whatever the device: the split only affects
// load balance, and the plan must not depend on a device query so that the
// workspace size agrees between sizing and calling.
struct SplitPlan {
  int P = 0;
  long long nparts = 0, nslots = 0;
};

static int tiles64_host(long long L, int j) {
  return (int)((L - (long long)j * FIX_CHUNK + 63) / 64);
}

static SplitPlan plan_split(const fix_attn_problem* p, const Dims& d) {
  SplitPlan sp;
  auto each_seq = [&](auto fn) {
    if (p->cu_seqlens) {
      for (int i = 0; i < p->num_seqs; ++i) fn(p->cu_seqlens_host[i + 1] - p->cu_seqlens_host[i], 1);
    } else {
      fn((long long)p->seqlen, (long long)p->batch);
    }
  };
  long long total = 0;
  each_seq([&](long long L, long long mult) {
    const int nc = (int)((L + FIX_CHUNK - 1) / FIX_CHUNK);
    for (int j = 0; j < nc; ++j) total += mult * d.grp * tiles64_host(L, j);
  });
  total *= d.Hkv;
  // about one part per SM: each dk/dv CTA's set-up (barriers, TMEM, its key
  // chunk's K and V) and epilogue are paid once per part, and fewer parts
  // mean fewer partial slots for the combine to read
  constexpr int kSMs = 148;
  long long P = (total + kSMs - 1) / kSMs;
  if (P < 4) P = 4;
  if (P > (1 << 30)) P = 1 << 30;
  sp.P = (int)P;
  // the split: per key chunk, its diagonal tiles and its later tiles, each
  // in runs of at most P
  each_seq([&](long long L, long long mult) {
    const int nc = (int)((L + FIX_CHUNK - 1) / FIX_CHUNK);
    for (int j = 0; j < nc; ++j) {
      const long long h = fix_halves((int)L, j);
      const long long nd = ((long long)d.grp * h + P - 1) / P;
      const long long no = ((long long)d.grp * (tiles64_host(L, j) - h) + P - 1) / P;
      sp.nparts += mult * (nd + no);
    }
  });
  sp.nslots = sp.nparts;   // every part writes its own slot
  return sp;
}

// Workspace layout (all offsets 256-byte aligned).
struct Ws {
  size_t status, chunks, order, safe, L, Lt, vt, vm, vml, tot, rho, hr, lvt;   // forward and backward
  size_t dow, dot, domh, doml, dsafe, hmax, ptt, delta, A, dG, dtot, dwp, dgf;   // backward only
  size_t parts, cpart, partial;                            // dk/dv work split
  size_t total;
};

static Ws layout(const Dims& d, bool bwd, const SplitPlan& sp) {
  Ws w{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  const size_t nkv = (size_t)d.N * d.Hkv * d.Dv;
  const size_t nch = (size_t)d.nchunks * d.Hkv * d.Dv;
  w.status = take(256);
  w.chunks = take((size_t)(d.nchunks > 0 ? d.nchunks : 1) * sizeof(Chunk));
  w.order = take((size_t)(d.nchunks > 0 ? d.nchunks : 1) * sizeof(int));
  w.safe = take((size_t)(d.nchunks > 0 ? d.nchunks : 1) * d.Hkv * sizeof(int));
  w.L = take(nkv * 4);
  w.Lt = take(nkv * 4);   // L channel-major [Hkv][Dv][N], for the forward's epilogue
  w.vt = take(nkv * 2);
  w.vm = take(nkv * 2);
  w.vml = take(nkv * 2);
  w.tot = take(nch * 4);
  w.rho = take(nch * 4);
  w.hr = take(nch * 4);
  w.lvt = take(nch * 4);
  if (bwd) {
    w.dow = take((size_t)d.N * d.Hq * d.Dv * 4);
    w.dot = take((size_t)d.N * d.Hq * d.Dv * 2);
    w.domh = take((size_t)d.N * d.Hq * d.Dv * 2);
    w.doml = take((size_t)d.N * d.Hq * d.Dv * 2);
    w.dsafe = take((size_t)(d.nchunks > 0 ? d.nchunks : 1) * d.Hq * sizeof(int));
    w.hmax = take((size_t)(d.nchunks > 0 ? d.nchunks : 1) * d.Hq * sizeof(int));
    w.ptt = take((size_t)d.N * d.Hq * sizeof(float));
    w.delta = take((size_t)d.N * d.Hq * sizeof(float));
    w.A = take(nkv * 4);
    w.dG = take(nkv * 4);
    w.dtot = take(nch * 4);
    w.dwp = take((size_t)(d.nchunks > 0 ? d.nchunks : 1) * kPreSplit * d.Hkv * d.Dv * 4);
    w.parts = take((size_t)(sp.nparts > 0 ? sp.nparts : 1) * sizeof(Part));
    w.cpart = take((size_t)(d.nchunks > 0 ? d.nchunks : 1) * sizeof(int2));
    w.partial = take((size_t)sp.nslots * d.Hkv * FIX_CHUNK * (d.Dk + d.Dv) * 4);
    // a scalar gate's per-channel dg, summed over the channels at the end
    w.dgf = d.scalar_gate ? take(nkv * 4) : 0;
  }
  w.total = o;
  return w;
}

static fix_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FIX_ERR_CUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return FIX_ERR_CUDA;
  return major == 10 ? FIX_OK : FIX_ERR_ARCH;
}

#ifdef FIX_TEST_HOOKS
int g_test_last_cuda_error = 0;   // test builds: the last launch error seen
#endif
fix_status launch_status() {
  const cudaError_t e = cudaGetLastError();
#ifdef FIX_TEST_HOOKS
  if (e != cudaSuccess) g_test_last_cuda_error = (int)e;
#endif
  return e == cudaSuccess ? FIX_OK : FIX_ERR_CUDA;
}
static fix_status launched() { return launch_status(); }

// Records the profiling event of `stage` (begin = 0 / end = 1) if requested.
static fix_status mark(const fix_attn_problem* p, int stage, int end, cudaStream_t st) {
  if (!p->events) return FIX_OK;
  cudaEvent_t e = static_cast<cudaEvent_t>(p->events[2 * stage + end]);
  if (!e) return FIX_OK;
  return cudaEventRecord(e, st) == cudaSuccess ? FIX_OK : FIX_ERR_CUDA;
}

#define FIX_TRY(expr)                 \
  do {                                \
    fix_status _s = (expr);           \
    if (_s != FIX_OK) return _s;      \
  } while (0)

static size_t simt_fwd_smem(const Dims& d) {
  return sizeof(float) * (size_t)(ST_ROWS * (2 * d.Dk + 1 + 3 * d.Dv));
}
static size_t simt_dq_smem(const Dims& d) {
  return sizeof(float) * (size_t)(ST_ROWS * d.Dk + 2 * ST_ROWS * d.Dv + ST_ROWS + d.Dv +
                                  ST_ROWS * (d.Dk + 1) + 2 * ST_ROWS * (d.Dv + 1));
}
static size_t simt_dkv_smem(const Dims& d) {
  return sizeof(float) * (size_t)(ST_ROWS * d.Dk + 2 * ST_ROWS * d.Dv + ST_ROWS);
}

bool set_smem_limit(const void* func, int bytes) {
  struct Entry {
    const void* func;
    int dev, bytes;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(mu);
  for (Entry& e : done)
    if (e.func == func && e.dev == dev) {
      if (bytes <= e.bytes) return true;
      if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
          cudaSuccess)
        return launch_status() == FIX_OK;
      e.bytes = bytes;
      return true;
    }
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return launch_status() == FIX_OK;   // records the error (it is pending)
  done.push_back(Entry{func, dev, bytes});
  return true;
}

// Copies `bytes` (a multiple of 4) from host memory to the device through
// the parameter blocks of upload launches, in pieces of at most 31 KB.
static fix_status upload(void* dst, const uint32_t* src, size_t bytes, cudaStream_t st) {
  size_t words = bytes / 4, off = 0;
  while (off < words) {
    const size_t n = std::min(words - off, (size_t)kBlobMaxWords);
    uint32_t* to = static_cast<uint32_t*>(dst) + off;
    auto send = [&](auto blob) {
      std::memcpy(blob.w, src + off, n * 4);
      upload_kernel<sizeof(blob.w) / 4><<<1, 256, 0, st>>>(blob, to, (int)n);
    };
    if (n <= 256) send(Blob<256>{});
    else if (n <= 1024) send(Blob<1024>{});
    else if (n <= 4096) send(Blob<4096>{});
    else send(Blob<kBlobMaxWords>{});
    FIX_TRY(launched());
    off += n;
  }
  return FIX_OK;
}

// Launches that upload() makes for `bytes`.
static int upload_launches(size_t bytes) {
  return (int)((bytes / 4 + kBlobMaxWords - 1) / kBlobMaxWords);
}

// Sequence lengths of the problem, in order (B sequences of T tokens, or the
// packed lengths of the host mirror of cu_seqlens).
template <class Fn>
static void each_sequence(const fix_attn_problem* p, Fn fn) {
  if (p->cu_seqlens) {
    for (int i = 0; i < p->num_seqs; ++i)
      fn(p->cu_seqlens_host[i], p->cu_seqlens_host[i + 1] - p->cu_seqlens_host[i]);
  } else {
    for (int b = 0; b < p->batch; ++b) fn((long long)b * p->seqlen, (long long)p->seqlen);
  }
}

// Builds the schedule on the host and uploads it into the workspace:
//   chunks[]  the chunk table, sequences in order, 128-token chunks from each
//             sequence's first token (followed by safe[] = 1, see the prefix
//             pass);
//   order[]   chunk ids by decreasing chunk index j (the number of key blocks
//             before the diagonal; ties in table order), so that grids
//             walking order[] start the longest causal rows first;
//   with the dk/dv split plan `sp`: parts[] holds every later-block part
//   first (sequences, then chunks, in order), then every diagonal part; a key
//   chunk's slots are consecutive, its diagonal parts' first, and
//   cpart[ci] = {number of parts, first slot}.
// With `tables_kept` (the backward reusing its forward's workspace) only the
// split is uploaded: the chunk table and order are the forward's.
static fix_status upload_schedule(const fix_attn_problem* p, const Dims& d, const Ws& ws,
                                  char* base, const SplitPlan* sp, bool tables_kept,
                                  cudaStream_t st) {
  if (d.nchunks == 0) return FIX_OK;
  thread_local std::vector<uint32_t> bufA, bufB;
  // chunk table, order, and the fp16-safe flags of the prefix pass set to 1
  // (its CTAs AND their part in)
  const size_t spanA = ws.safe - ws.chunks + (size_t)d.nchunks * d.Hkv * sizeof(int);
  bufA.assign(spanA / 4, 0u);
  std::fill(bufA.begin() + (ws.safe - ws.chunks) / 4, bufA.end(), 1u);
  Chunk* chunks = reinterpret_cast<Chunk*>(bufA.data());
  int* order = reinterpret_cast<int*>(reinterpret_cast<char*>(bufA.data()) + (ws.order - ws.chunks));
  int ci = 0, maxj = 0;
  each_sequence(p, [&](long long s0, long long L) {
    const int nc = (int)((L + FIX_CHUNK - 1) / FIX_CHUNK);
    for (int j = 0; j < nc; ++j, ++ci) {
      chunks[ci] = Chunk{(int)(s0 + (long long)j * FIX_CHUNK),
                         (int)std::min<long long>(FIX_CHUNK, L - (long long)j * FIX_CHUNK), j, nc};
      maxj = std::max(maxj, j);
    }
  });
  if (ci != d.nchunks) return FIX_ERR_CU_SEQLENS;
  {
    std::vector<int> count(maxj + 2, 0);
    for (int i = 0; i < ci; ++i) ++count[maxj - chunks[i].j + 1];
    for (int k = 1; k <= maxj + 1; ++k) count[k] += count[k - 1];
    for (int i = 0; i < ci; ++i) order[count[maxj - chunks[i].j]++] = i;
  }
  if (!tables_kept) FIX_TRY(upload(base + ws.chunks, bufA.data(), spanA, st));
  if (!sp) return FIX_OK;
  const size_t spanB = ws.cpart - ws.parts + (size_t)d.nchunks * sizeof(int2);
  bufB.assign(spanB / 4, 0u);
  Part* parts = reinterpret_cast<Part*>(bufB.data());
  int2* cpart = reinterpret_cast<int2*>(reinterpret_cast<char*>(bufB.data()) + (ws.cpart - ws.parts));
  const long long P = sp->P;
  auto n_diag = [&](long long L, int j) { return ((long long)d.grp * fix_halves((int)L, j) + P - 1) / P; };
  auto n_off = [&](long long L, int j) {
    return ((long long)d.grp * (tiles64_host(L, j) - fix_halves((int)L, j)) + P - 1) / P;
  };
  long long total_off = 0;
  each_sequence(p, [&](long long, long long L) {
    const int nc = (int)((L + FIX_CHUNK - 1) / FIX_CHUNK);
    for (int j = 0; j < nc; ++j) total_off += n_off(L, j);
  });
  long long o = 0, e = total_off, slot = 0;
  int c = 0;
  each_sequence(p, [&](long long, long long L) {
    const int nc = (int)((L + FIX_CHUNK - 1) / FIX_CHUNK);
    for (int j = 0; j < nc; ++j, ++c) {
      const long long nd = n_diag(L, j), no = n_off(L, j);
      cpart[c] = make_int2((int)(nd + no), (int)slot);
      for (long long q = 0; q < nd; ++q) parts[e++] = Part{c, (int)q, (int)(slot + q), 1};
      for (long long q = 0; q < no; ++q) parts[o++] = Part{c, (int)q, (int)(slot + nd + q), 0};
      slot += nd + no;
    }
  });
  if (e != sp->nparts || slot != sp->nslots) return FIX_ERR_CU_SEQLENS;
  return upload(base + ws.parts, bufB.data(), spanB, st);
}

static fix_status run_prefix(const Dims& d, const fix_attn_problem* p, const Ws& ws, char* base,
                             const float* g, const void* v, bool want_vt, bool want_lt,
                             const SplitPlan* sp, int* hmax, bool reuse, cudaStream_t st) {
  const Chunk* chunks = reinterpret_cast<const Chunk*>(base + ws.chunks);
  FIX_TRY(upload_schedule(p, d, ws, base, sp, reuse, st));
  if (d.nchunks == 0) return FIX_OK;
  if (reuse) {
    // the forward's prefix results stay; only the per-(chunk, q head) max
    // |do| of this backward starts from zero
    if (hmax && cudaMemsetAsync(hmax, 0, (size_t)d.nchunks * d.Hq * sizeof(int), st) != cudaSuccess)
      return FIX_ERR_CUDA;
    return FIX_OK;
  }
  const size_t psmem = prefix_smem_bytes(d.Dv, want_lt);
  if (!set_smem_limit(reinterpret_cast<const void*>(prefix_kernel), (int)psmem)) return FIX_ERR_CUDA;
  prefix_kernel<<<dim3(d.nchunks, d.Hkv, prefix_slices(d.Dv)), 256, psmem, st>>>(
      d, chunks, g, static_cast<const __nv_bfloat16*>(v), reinterpret_cast<float*>(base + ws.L),
      want_lt ? reinterpret_cast<float*>(base + ws.Lt) : nullptr,
      want_vt ? reinterpret_cast<uint16_t*>(base + ws.vt) : nullptr,
      reinterpret_cast<__nv_bfloat16*>(base + ws.vm),
      reinterpret_cast<__nv_bfloat16*>(base + ws.vml), reinterpret_cast<float*>(base + ws.tot),
      reinterpret_cast<float*>(base + ws.rho), reinterpret_cast<float*>(base + ws.hr),
      reinterpret_cast<float*>(base + ws.lvt), reinterpret_cast<int*>(base + ws.safe),
      reinterpret_cast<int*>(base + ws.status) + 1, hmax);
  return launched();
}

}  // namespace fix

using namespace fix;

extern "C" {

size_t fix_attn_workspace_bytes(const fix_attn_problem* p, int backward) {
  Dims d;
  if (make_dims(p, &d) != FIX_OK) return 0;
  return layout(d, backward != 0, backward ? plan_split(p, d) : SplitPlan{}).total;
}

const char* fix_attn_status_string(int s) {
  switch (s) {
    case FIX_OK: return "FIX_OK";
    case FIX_ERR_NULL: return "FIX_ERR_NULL: a required pointer is NULL";
    case FIX_ERR_SHAPE: return "FIX_ERR_SHAPE: invalid or inconsistent sizes";
    case FIX_ERR_HEAD_DIM: return "FIX_ERR_HEAD_DIM: head dims must be 16, 32, 64 or 128";
    case FIX_ERR_GQA: return "FIX_ERR_GQA: num_q_heads must be a multiple of num_kv_heads";
    case FIX_ERR_CU_SEQLENS: return "FIX_ERR_CU_SEQLENS: cu_seqlens must rise from 0 to the token count";
    case FIX_ERR_ALIGN: return "FIX_ERR_ALIGN: pointers must be 16-byte aligned";
    case FIX_ERR_WORKSPACE: return "FIX_ERR_WORKSPACE: workspace missing or too small";
    case FIX_ERR_DTYPE: return "FIX_ERR_DTYPE: unknown y_dtype or algo";
    case FIX_ERR_CUDA: return "FIX_ERR_CUDA: a CUDA call or kernel launch failed";
    case FIX_ERR_DEVICE_TIMEOUT: return "FIX_ERR_DEVICE_TIMEOUT: a bounded device wait expired";
    case FIX_ERR_ARCH: return "FIX_ERR_ARCH: the current device is not sm_100";
    default: return "unknown fix_status";
  }
}

fix_status fix_attn_fwd(const fix_attn_problem* p, const void* q, const void* k, const void* v,
                        const float* g, const void* w, const void* z, void* y, float* o_s,
                        float* m_s, float* rstd_s, void* workspace, size_t ws_bytes,
                        void* stream) {
  Dims d;
  FIX_TRY(make_dims(p, &d));
  if (!q || !k || !v || !g || (!w && !d.no_norm) || !y || !workspace) return FIX_ERR_NULL;
  const int nsaved = (o_s != nullptr) + (m_s != nullptr) + (rstd_s != nullptr);
  if (nsaved != 0 && nsaved != 3) return FIX_ERR_NULL;
  for (const void* ptr : {q, k, v, (const void*)g, w, z, (const void*)y, (const void*)workspace})
    if (ptr && !aligned16(ptr)) return FIX_ERR_ALIGN;
  if (nsaved && (!aligned16(o_s) || !aligned16(m_s) || !aligned16(rstd_s))) return FIX_ERR_ALIGN;
  const Ws ws = layout(d, false, SplitPlan{});
  if (ws_bytes < ws.total) return FIX_ERR_WORKSPACE;
  FIX_TRY(check_device());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(workspace);
  // status word and the out-of-range flag of the prefix pass start at zero
  if (cudaMemsetAsync(base + ws.status, 0, 8, st) != cudaSuccess) return FIX_ERR_CUDA;
  if (d.N == 0) return FIX_OK;
  const bool tc = p->algo != FIX_ALGO_SIMT && tc_fwd_supported(d);
  FIX_TRY(mark(p, FIX_STAGE_FWD_PREFIX, 0, st));
  FIX_TRY(run_prefix(d, p, ws, base, g, v, tc, tc, nullptr, nullptr, false, st));
  FIX_TRY(mark(p, FIX_STAGE_FWD_PREFIX, 1, st));
  const Chunk* chunks = reinterpret_cast<const Chunk*>(base + ws.chunks);
  const float* L = reinterpret_cast<const float*>(base + ws.L);
  const float* tot = reinterpret_cast<const float*>(base + ws.tot);
  FIX_TRY(mark(p, FIX_STAGE_FWD_ATTN, 0, st));
  if (tc) {
    FIX_TRY(tc_fwd(d, chunks, reinterpret_cast<const int*>(base + ws.order), q, k,
                   reinterpret_cast<const uint16_t*>(base + ws.vt),
                   reinterpret_cast<const __nv_bfloat16*>(base + ws.vm),
                   reinterpret_cast<const __nv_bfloat16*>(base + ws.vml), v, L,
                   reinterpret_cast<const float*>(base + ws.Lt), tot,
                   reinterpret_cast<const float*>(base + ws.rho),
                   reinterpret_cast<const float*>(base + ws.hr),
                   reinterpret_cast<const float*>(base + ws.lvt),
                   reinterpret_cast<const int*>(base + ws.safe), w, z, y,
                   p->y_dtype == FIX_DTYPE_F32, o_s, m_s, rstd_s,
                   reinterpret_cast<int*>(base + ws.status), st));
  } else {
    const size_t smem = simt_fwd_smem(d);
    if (!set_smem_limit(reinterpret_cast<const void*>(fwd_simt_kernel), (int)smem))
      return FIX_ERR_CUDA;
    fwd_simt_kernel<<<dim3(d.nchunks * 4, d.Hq), 256, smem, st>>>(
        d, chunks, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), L, tot, static_cast<const __nv_bfloat16*>(w),
        static_cast<const __nv_bfloat16*>(z), y, p->y_dtype == FIX_DTYPE_F32, o_s, m_s, rstd_s);
    FIX_TRY(launched());
  }
  return mark(p, FIX_STAGE_FWD_ATTN, 1, st);
}

fix_status fix_attn_bwd(const fix_attn_problem* p, const void* q, const void* k, const void* v,
                        const float* g, const void* w, const void* z, const void* dy,
                        const float* o_s, const float* m_s, const float* rstd_s, void* dq,
                        void* dk, void* dv, float* dg, void* dw, void* dz, void* workspace,
                        size_t ws_bytes, void* stream) {
  Dims d;
  FIX_TRY(make_dims(p, &d));
  if (!q || !k || !v || !g || (!w && !d.no_norm) || !dy || !o_s || !m_s || !rstd_s || !dq || !dk ||
      !dv || !dg || (!dw && !d.no_norm) || !workspace || (!z != !dz))
    return FIX_ERR_NULL;
  for (const void* ptr : {q, k, v, (const void*)g, w, z, dy, (const void*)o_s, (const void*)m_s,
                          (const void*)rstd_s, (const void*)dq, (const void*)dk, (const void*)dv,
                          (const void*)dg, (const void*)dw, (const void*)dz,
                          (const void*)workspace})
    if (ptr && !aligned16(ptr)) return FIX_ERR_ALIGN;
  const SplitPlan sp = plan_split(p, d);
  const Ws ws = layout(d, true, sp);
  if (ws_bytes < ws.total) return FIX_ERR_WORKSPACE;
  FIX_TRY(check_device());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(workspace);
  const bool tc = p->algo != FIX_ALGO_SIMT && tc_bwd_supported(d);
  // The forward's prefix results can stand in for the backward's when the
  // caller says the workspace is the forward's and the forward produced what
  // this backward reads (the 16-bit operands only on its tensor-core path).
  const bool fwd_tc = p->algo != FIX_ALGO_SIMT && tc_fwd_supported(d);
  const bool reuse = (p->flags & FIX_FLAG_REUSE_FWD_WORKSPACE) && (!tc || fwd_tc);
  // status word, and (unless reused) the prefix pass's out-of-range flag
  if (cudaMemsetAsync(base + ws.status, 0, reuse ? 4 : 8, st) != cudaSuccess) return FIX_ERR_CUDA;
  if (d.N == 0) {
    if (dw && cudaMemsetAsync(dw, 0, (size_t)d.Dv * 2, st) != cudaSuccess) return FIX_ERR_CUDA;
    return FIX_OK;
  }
  FIX_TRY(mark(p, FIX_STAGE_BWD_PREFIX, 0, st));
  FIX_TRY(run_prefix(d, p, ws, base, g, v, tc, false, tc ? &sp : nullptr,
                     tc ? reinterpret_cast<int*>(base + ws.hmax) : nullptr, reuse, st));
  FIX_TRY(mark(p, FIX_STAGE_BWD_PREFIX, 1, st));
  const Chunk* chunks = reinterpret_cast<const Chunk*>(base + ws.chunks);
  const float* L = reinterpret_cast<const float*>(base + ws.L);
  const float* tot = reinterpret_cast<const float*>(base + ws.tot);
  float* dow = reinterpret_cast<float*>(base + ws.dow);
  uint16_t* dot = reinterpret_cast<uint16_t*>(base + ws.dot);
  __nv_bfloat16* domh = reinterpret_cast<__nv_bfloat16*>(base + ws.domh);
  __nv_bfloat16* doml = reinterpret_cast<__nv_bfloat16*>(base + ws.doml);
  int* dsafe = reinterpret_cast<int*>(base + ws.dsafe);
  float* A = reinterpret_cast<float*>(base + ws.A);
  float* dG = reinterpret_cast<float*>(base + ws.dG);
  float* dtot = reinterpret_cast<float*>(base + ws.dtot);
  float* dwp = reinterpret_cast<float*>(base + ws.dwp);
  const int* badflag = reinterpret_cast<const int*>(base + ws.status) + 1;
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k);
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(v);
  FIX_TRY(mark(p, FIX_STAGE_BWD_PRE, 0, st));
  int* hmax = reinterpret_cast<int*>(base + ws.hmax);
  float* delta = reinterpret_cast<float*>(base + ws.delta);
  const size_t pre_smem = bwd_pre_smem_bytes(d.grp);
  if (!set_smem_limit(reinterpret_cast<const void*>(bwd_pre_kernel), (int)pre_smem)) return FIX_ERR_CUDA;
  bwd_pre_kernel<<<dim3(d.nchunks * kPreSplit, d.Hkv), 256, pre_smem, st>>>(
      d, chunks, qb, kb, vb, o_s, m_s, rstd_s, static_cast<const __nv_bfloat16*>(dy),
      static_cast<const __nv_bfloat16*>(w), static_cast<const __nv_bfloat16*>(z),
      static_cast<__nv_bfloat16*>(dz), dow, A, delta, dwp, tc ? hmax : nullptr,
      tc ? reinterpret_cast<float*>(base + ws.ptt) : nullptr);
  FIX_TRY(launched());
  if (tc) {
    bwd_pre_ops_kernel<<<dim3(d.nchunks * kPreOpsSplit, d.Hkv), 256, 0, st>>>(
        d, chunks, L, reinterpret_cast<const float*>(base + ws.rho),
        reinterpret_cast<const float*>(base + ws.hr), reinterpret_cast<const int*>(base + ws.safe),
        dow, hmax, dot, domh, doml, dsafe);
    FIX_TRY(launched());
  }
  if (!d.no_norm) {
    dw_reduce_kernel<<<(d.Dv + 31) / 32, 1024, 0, st>>>(dwp, d.nchunks * kPreSplit * d.Hkv, d.Dv,
                                                       static_cast<__nv_bfloat16*>(dw));
    FIX_TRY(launched());
  } else if (dw && cudaMemsetAsync(dw, 0, (size_t)d.Dv * 2, st) != cudaSuccess) {
    return FIX_ERR_CUDA;   // no weight without the norm: its gradient is zero
  }
  FIX_TRY(mark(p, FIX_STAGE_BWD_PRE, 1, st));
  TcBwdArgs ta{};
  if (tc) {
    ta.chunks = chunks;
    ta.order = reinterpret_cast<const int*>(base + ws.order);
    ta.q = q;
    ta.k = k;
    ta.v = v;
    ta.vt = reinterpret_cast<const uint16_t*>(base + ws.vt);
    ta.vm = reinterpret_cast<const __nv_bfloat16*>(base + ws.vm);
    ta.L = L;
    ta.tot = tot;
    ta.rho = reinterpret_cast<const float*>(base + ws.rho);
    ta.hr = reinterpret_cast<const float*>(base + ws.hr);
    ta.lvt = reinterpret_cast<const float*>(base + ws.lvt);
    ta.safe = reinterpret_cast<const int*>(base + ws.safe);
    ta.dsafe = dsafe;
    ta.m_s = m_s;
    ta.do_ws = dow;
    ta.dot = dot;
    ta.domh = domh;
    ta.doml = doml;
    ta.A = A;
    ta.ptt = reinterpret_cast<const float*>(base + ws.ptt);
    ta.delta = d.no_norm ? delta : nullptr;
    ta.badflag = badflag;
    ta.parts = reinterpret_cast<const Part*>(base + ws.parts);
    ta.cpart = reinterpret_cast<const int2*>(base + ws.cpart);
    ta.tiles_per_part = sp.P;
    ta.nparts = sp.nparts;
    ta.nslots = sp.nslots;
    ta.partial = reinterpret_cast<float*>(base + ws.partial);
    ta.dq = dq;
    ta.dk = dk;
    ta.dv = dv;
    ta.dG = dG;
    ta.status = reinterpret_cast<int*>(base + ws.status);
  }
  const size_t smq = simt_dq_smem(d), smkv = simt_dkv_smem(d);
  if (!tc && (!set_smem_limit(reinterpret_cast<const void*>(dq_simt_kernel), (int)smq) ||
              !set_smem_limit(reinterpret_cast<const void*>(dkv_simt_kernel), (int)smkv)))
    return FIX_ERR_CUDA;
  FIX_TRY(mark(p, FIX_STAGE_BWD_DQ, 0, st));
  if (tc) FIX_TRY(tc_bwd(p, d, ta, 0, st));
  else
    dq_simt_kernel<<<dim3(d.nchunks * 4, d.Hq), 256, smq, st>>>(
        d, chunks, qb, kb, vb, L, tot, m_s, dow, d.no_norm ? delta : nullptr,
        static_cast<__nv_bfloat16*>(dq), nullptr);
  FIX_TRY(launched());
  FIX_TRY(mark(p, FIX_STAGE_BWD_DQ, 1, st));
  FIX_TRY(mark(p, FIX_STAGE_BWD_DKV, 0, st));
  if (tc) FIX_TRY(tc_bwd(p, d, ta, 1, st));
  else
    dkv_simt_kernel<<<dim3(d.nchunks * 4, d.Hkv), 256, smkv, st>>>(
        d, chunks, qb, kb, vb, L, tot, m_s, dow, d.no_norm ? delta : nullptr, A,
        static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv), dG, nullptr);
  FIX_TRY(launched());
  FIX_TRY(mark(p, FIX_STAGE_BWD_DKV, 1, st));
  FIX_TRY(mark(p, FIX_STAGE_BWD_FINISH, 0, st));
  if (tc) FIX_TRY(tc_bwd(p, d, ta, 2, st));
  FIX_TRY(mark(p, FIX_STAGE_BWD_FINISH, 1, st));
  FIX_TRY(mark(p, FIX_STAGE_BWD_DG, 0, st));
  chunk_total_kernel<<<dim3(d.nchunks, d.Hkv, prefix_slices(d.Dv)), 256, 0, st>>>(d, chunks, dG, dtot);
  FIX_TRY(launched());
  float* dgf = d.scalar_gate ? reinterpret_cast<float*>(base + ws.dgf) : dg;
  reverse_cumsum_kernel<<<dim3(d.nchunks, d.Hkv, prefix_slices(d.Dv)), 256, 0, st>>>(d, chunks, dG, dtot, dgf);
  FIX_TRY(launched());
  if (d.scalar_gate) {
    // a scalar gate acts on every channel: its gradient is the channel sum
    const long long rows = (long long)d.N * d.Hkv;
    channel_sum_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(dgf, rows, d.Dv, dg);
    FIX_TRY(launched());
  }
  return mark(p, FIX_STAGE_BWD_DG, 1, st);
}

int fix_attn_kernel_count(const fix_attn_problem* p, int backward) {
  Dims d;
  if (make_dims(p, &d) != FIX_OK) return 0;
  if (d.N == 0) return 0;
  const SplitPlan sp = backward ? plan_split(p, d) : SplitPlan{};
  const Ws ws = layout(d, backward != 0, sp);
  const int upA =
      d.nchunks ? upload_launches(ws.safe - ws.chunks + (size_t)d.nchunks * d.Hkv * 4) : 0;
  if (!backward) {
    const bool tc = p->algo != FIX_ALGO_SIMT && tc_fwd_supported(d);
    // schedule upload, prefix pass, attention
    return upA + 1 + (tc ? tc_fwd_kernel_count(d) : 1);
  }
  const bool tc = p->algo != FIX_ALGO_SIMT && tc_bwd_supported(d);
  const bool fwd_tc = p->algo != FIX_ALGO_SIMT && tc_fwd_supported(d);
  const bool reuse = (p->flags & FIX_FLAG_REUSE_FWD_WORKSPACE) && (!tc || fwd_tc);
  const int upB = (tc && d.nchunks) ? upload_launches(ws.cpart - ws.parts + (size_t)d.nchunks * 8) : 0;
  // schedule uploads (the split only when the forward's tables are reused),
  // the prefix pass unless reused, the preprocess (2, or 3 with the
  // tensor-core operands), then either tensor-core dq / dk/dv / exact
  // out-of-range terms / combine or the exact kernels (2), the dG reverse
  // cumsum (2)
  const bool has_dw = !d.no_norm;   // dw is optional only without the norm
  return (reuse ? 0 : upA + 1) + upB + (tc ? 2 : 1) + (has_dw ? 1 : 0) +
         (tc ? tc_bwd_kernel_count(d, sp.nslots) : 2) + 2 + (d.scalar_gate ? 1 : 0);
}

fix_status fix_attn_device_status(const void* workspace, void* stream) {
  if (!workspace) return FIX_ERR_NULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return FIX_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return FIX_ERR_CUDA;
  return word == 0 ? FIX_OK : FIX_ERR_DEVICE_TIMEOUT;
}

}  // extern "C"
