/*
 * fix_attn.h -- C ABI of the FiX attention library (libfixattn.so), sm_100a.
 *
 * FiX ("FiX: Introducing Fine-grained Forget Gate into Softmax Attention",
 * ICML 2026 poster, abstract) is causal softmax attention whose forget gate
 * acts element-wise on the value channels.  Because an RMSNorm over the value
 * dimension follows, the softmax denominator is dropped and any per-row shift
 * of the logits is free.  Per sequence, q head h and its kv head
 * kv(h) = h / (Hq / Hkv), for positions 0 <= s <= t < L:
 *
 *     S_ts    = scale * <q_t, k_s>,      m_t = max_{s<=t} S_ts
 *     G_t[c]  = sum_{r<=t} g_r[c]        (restarts at every sequence)
 *     o_t[c]  = sum_{s<=t} exp(S_ts - m_t) * exp(G_t[c] - G_s[c]) * v_s[c]
 *     y_t     = o_t * (mean_c o_t[c]^2 + eps)^(-1/2) * w
 *
 * Shapes and constraints follow the FiX README ("Quick Start" and its closing
 * note): q [B,T,Hq,Dk], k [B,T,Hkv,Dk], v [B,T,Hkv,Dv], g [B,T,Hkv,Dv] in
 * float32, o_norm weight w [Dv]; packed sequences through int64 cu_seqlens as
 * in FlashAttention; head dims in {16, 32, 64, 128}.
 *
 * Conventions for every entry point:
 *   - Ownership: the caller allocates and owns every buffer.  The library never
 *     allocates, frees or synchronises (except the two device-status readers)
 *     and keeps no mutable global state besides cached kernel attributes, with
 *     one exception: the fixed device array behind fix_attn_fwd_noalloc (and
 *     its per-device address cache), described beside that entry point.
 *   - Execution: calls are asynchronous and ordered on `stream` (a cudaStream_t
 *     passed as void*; NULL = legacy default stream).  Every element of every
 *     output is written.
 *   - Layout: all tensors are dense, token-major with heads interleaved
 *     ([N, H, D], N = B*T tokens, D fastest), base pointers 16-byte aligned.
 *   - Dtypes: q, k, v, w, dy, dq, dk, dv, dw are bf16; g, dg and the saved
 *     tensors o, m, rstd are float32; y is bf16 or float32 (problem.y_dtype).
 *   - Errors: a status code is returned; nothing is thrown.  Argument errors
 *     are detected on the host before any launch; a failed launch returns
 *     FIX_ERR_CUDA.  Bounded device-side waits that expire record
 *     FIX_ERR_DEVICE_TIMEOUT in the workspace status word, which
 *     fix_attn_device_status() reads.
 */
#ifndef FIX_ATTN_H_
#define FIX_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FIX_OK = 0,
  FIX_ERR_NULL = 1,            /* a required pointer is NULL */
  FIX_ERR_SHAPE = 2,           /* non-positive / inconsistent sizes, B > 1 with cu_seqlens */
  FIX_ERR_HEAD_DIM = 3,        /* Dk or Dv not in {16, 32, 64, 128} */
  FIX_ERR_GQA = 4,             /* Hq not a multiple of Hkv */
  FIX_ERR_CU_SEQLENS = 5,      /* host mirror not 0 = c0 <= c1 <= ... = N */
  FIX_ERR_ALIGN = 6,           /* a pointer is not 16-byte aligned */
  FIX_ERR_WORKSPACE = 7,       /* workspace NULL or smaller than required */
  FIX_ERR_DTYPE = 8,           /* unknown y_dtype / algo */
  FIX_ERR_CUDA = 9,            /* a CUDA runtime call or launch failed */
  FIX_ERR_DEVICE_TIMEOUT = 10, /* a bounded device wait expired (see above) */
  FIX_ERR_ARCH = 11            /* the current device is not sm_100 */
} fix_status;

enum { FIX_DTYPE_BF16 = 0, FIX_DTYPE_F32 = 1 };

/* Kernel family.  FIX_ALGO_AUTO picks the tensor-core (tcgen05) kernels
 * where they apply: Dk and Dv in {64, 128}, at least 128 tokens in all, and
 * for the backward at most 16 q heads per kv head; other problems run on the
 * exact kernels.  FIX_ALGO_SIMT runs the exact fp32 CUDA-core kernels (every
 * decay factor exp(G_t - G_s) formed element by element); it is much slower
 * and serves as a second, independent GPU path for cross-checks. */
enum { FIX_ALGO_AUTO = 0, FIX_ALGO_SIMT = 1, FIX_ALGO_TC = 2 };

/* fix_attn_problem.flags.
 * FIX_FLAG_REUSE_FWD_WORKSPACE (fix_attn_bwd only): the caller promises that
 *   `workspace` is the one the matching training-mode fix_attn_fwd call used
 *   (same problem, q, k, v, g) and that nothing has written it since.  The
 *   backward then reuses the forward's gate prefix results (the prefix pass
 *   of the README's "Code Structure": chunk-local cumsums and pre-decayed
 *   values) instead of recomputing them.  Undefined results if the promise
 *   does not hold.
 * FIX_FLAG_NO_NORM: the README's o_norm = False.  No RMSNorm and no weight:
 *   y_t = o_t / l_t with the softmax denominator l_t = sum_{s<=t} exp(S_ts
 *   - m_t), i.e. the attention average with the element-wise decay on v (for
 *   g = 0 ordinary causal softmax attention).  o_norm_weight may be NULL;
 *   the saved tensors are then o_t / l_t, the log-sum-exp m_t + log l_t and
 *   ones; the backward is the exact one and fills dw (if given) with zeros.
 * FIX_FLAG_SCALAR_GATE: g (and dg) have shape [N, Hkv]: one log forget gate
 *   per token and kv head, applied to every value channel (the Forgetting
 *   Transformer's scalar gate, FoX abstract); dg is its gradient.
 * Both must be set identically for a forward and its backward.  Any other
 * bit: FIX_ERR_SHAPE. */
enum { FIX_FLAG_REUSE_FWD_WORKSPACE = 1, FIX_FLAG_NO_NORM = 2, FIX_FLAG_SCALAR_GATE = 4 };

typedef struct {
  int32_t batch;          /* B; must be 1 when cu_seqlens is given           */
  int32_t seqlen;         /* T; the total token count N when packed          */
  int32_t num_q_heads;    /* Hq                                               */
  int32_t num_kv_heads;   /* Hkv; Hq % Hkv == 0 (q head h uses kv h/(Hq/Hkv)) */
  int32_t head_dim_k;     /* Dk in {16,32,64,128}                            */
  int32_t head_dim_v;     /* Dv in {16,32,64,128}                            */
  int32_t num_seqs;       /* packed sequence count S (0 when not packed)      */
  int32_t y_dtype;        /* FIX_DTYPE_BF16 or FIX_DTYPE_F32                  */
  int32_t algo;           /* FIX_ALGO_*                                       */
  int32_t flags;          /* FIX_FLAG_* bits; 0 by default                    */
  const int64_t *cu_seqlens;      /* device [S+1] or NULL                     */
  const int64_t *cu_seqlens_host; /* host mirror [S+1]; required with cu_seqlens */
  float scale;            /* logit scale; <= 0 selects Dk^-1/2                */
  float eps;              /* RMSNorm epsilon (>= 0)                           */
  void *const *events;    /* NULL, or FIX_NUM_STAGES*2 cudaEvent_t: the call records
                             events[2*i] before and events[2*i+1] after stage i
                             on `stream` (profiling; stages it does not run are
                             recorded back to back)                            */
} fix_attn_problem;

/* Stages that fix_attn_problem.events brackets. */
enum {
  FIX_STAGE_FWD_PREFIX = 0, /* schedule + gate prefix sums + pre-decayed v   */
  FIX_STAGE_FWD_ATTN = 1,   /* attention forward with the fused RMSNorm      */
  FIX_STAGE_BWD_PREFIX = 2, /* schedule + gate prefix sums + pre-decayed v   */
  FIX_STAGE_BWD_PRE = 3,    /* RMSNorm backward, dw                          */
  FIX_STAGE_BWD_DQ = 4,     /* dq (tensor-core kernel, else exact kernel)    */
  FIX_STAGE_BWD_DKV = 5,    /* dk/dv partial sums (tensor-core kernel, else  */
                            /* the exact dk, dv, dG kernel)                  */
  FIX_STAGE_BWD_DG = 6,     /* reverse cumsum dG -> dg                        */
  FIX_STAGE_BWD_FINISH = 7, /* tensor-core path: the exact diagonal terms of */
                            /* channels outside the split's range (returns   */
                            /* at once without them), then the combine of    */
                            /* the dk/dv partials into dk, dv, dG            */
  FIX_NUM_STAGES = 8
};

/* Bytes of device workspace that fix_attn_fwd (backward = 0) or fix_attn_bwd
 * (backward = 1) needs for this problem; 0 if the problem is invalid.  The
 * workspace holds the chunked gate prefix sums, the pre-decayed values, the
 * packed-sequence schedule, backward accumulators and a status word.  Its
 * contents need no initialisation and are meaningless between calls. */
size_t fix_attn_workspace_bytes(const fix_attn_problem *p, int backward);

/* Forward (training or inference).
 *   q [N,Hq,Dk] bf16, k [N,Hkv,Dk] bf16, v [N,Hkv,Dv] bf16, g [N,Hkv,Dv] f32
 *   ([N,Hkv] with FIX_FLAG_SCALAR_GATE), o_norm_weight [Dv] bf16 (NULL allowed
 *   with FIX_FLAG_NO_NORM), o_gate [N,Hq,Dv] bf16 or NULL
 *   ->  y [N,Hq,Dv] (bf16 or f32, problem.y_dtype).
 * With o_gate z, y is multiplied element-wise by swish(z) = z sigmoid(z)
 * after the norm and its weight (the README's o_gate argument; the
 * activation is not on the pages: swish is the output-gate form of the
 * library FiX is forked from).
 * Saved tensors for fix_attn_bwd (pass all three, or all NULL for inference):
 *   o_saved [N,Hq,Dv] f32 (o before the norm and gate), m_saved [N,Hq] f32
 *   (row shift m_t), rstd_saved [N,Hq] f32.
 * g should be <= 0 (a log forget gate); positive values are computed the same
 * way but the factors exp(G_t - G_s) are then only safe while they stay inside
 * the float32 range.  Definition: FiX poster abstract; shapes and arguments:
 * FiX README, "Quick Start". */
fix_status fix_attn_fwd(const fix_attn_problem *p, const void *q, const void *k,
                        const void *v, const float *g, const void *o_norm_weight,
                        const void *o_gate, void *y, float *o_saved, float *m_saved,
                        float *rstd_saved, void *workspace, size_t workspace_bytes,
                        void *stream);

/* Backward of L = sum(dy * y) with the row shift m_t held constant (the exact
 * derivative with FIX_FLAG_NO_NORM, where y does not depend on m_t).
 *   dy [N,Hq,Dv] bf16, o_gate as given to the forward, and the saved o, m,
 *   rstd of the matching forward call
 *   -> dq [N,Hq,Dk], dk [N,Hkv,Dk], dv [N,Hkv,Dv] bf16, dg f32 (g's shape),
 *      dw [Dv] bf16 (gradient of o_norm_weight; may be NULL with
 *      FIX_FLAG_NO_NORM), d_o_gate [N,Hq,Dv] bf16 (NULL iff o_gate is NULL).
 * dk, dv and dg sum over the q heads of each kv group. */
fix_status fix_attn_bwd(const fix_attn_problem *p, const void *q, const void *k,
                        const void *v, const float *g, const void *o_norm_weight,
                        const void *o_gate, const void *dy, const float *o_saved,
                        const float *m_saved, const float *rstd_saved, void *dq, void *dk,
                        void *dv, float *dg, void *dw, void *d_o_gate, void *workspace,
                        size_t workspace_bytes, void *stream);

/* Decode: one new query per sequence against the cache of its tokens.
 * The problem gives batch = B sequences, seqlen = Tmax (cache capacity),
 * heads, head dims, scale, eps, y_dtype and the flags FIX_FLAG_NO_NORM /
 * FIX_FLAG_SCALAR_GATE; cu_seqlens must be NULL and num_seqs 0.
 *   seqlens   device int32 [B]: L_b, the tokens in sequence b's cache, the
 *             new token included (0 < L_b <= Tmax; L_b = 0 gives y = 0)
 *   q         [B,Hq,Dk] bf16: the new token's queries
 *   k_cache   [B,Tmax,Hkv,Dk] bf16, v_cache [B,Tmax,Hkv,Dv] bf16,
 *   g_cache   [B,Tmax,Hkv,Dv] f32 ([B,Tmax,Hkv] with the scalar gate): the
 *             keys, values and log forget gates of tokens 0..L_b-1
 *   o_norm_weight [Dv] bf16 (NULL allowed without the norm), o_gate [B,Hq,Dv]
 *             bf16 or NULL  ->  y [B,Hq,Dv] (bf16 or f32)
 * y is row t = L_b - 1 of fix_attn_fwd on the same sequence (the FiX poster
 * abstract names inference memory as a challenge FiX addresses; the pages
 * give no decode algorithm, so this evaluates the definition for the last
 * row).  Requires Hq/Hkv * Dv <= 2048 (FIX_ERR_GQA otherwise).  The cache is
 * read once, split over CTAs by key ranges. */
size_t fix_attn_decode_workspace_bytes(const fix_attn_problem *p);
fix_status fix_attn_decode(const fix_attn_problem *p, const int32_t *seqlens, const void *q,
                           const void *k_cache, const void *v_cache, const float *g_cache,
                           const void *o_norm_weight, const void *o_gate, void *y,
                           void *workspace, size_t workspace_bytes, void *stream);

/* Synchronises `stream`, then returns the device status word that the last
 * call on this workspace left (FIX_OK or FIX_ERR_DEVICE_TIMEOUT), or
 * FIX_ERR_CUDA if the stream reports an error.  The word is reset by every
 * fix_attn_fwd / fix_attn_bwd call. */
fix_status fix_attn_device_status(const void *workspace, void *stream);

/* Largest workspace fix_attn_fwd_noalloc can provide: 16 MiB.  The forward's
 * workspace is about 14 bytes per (token, kv head, value channel) plus a few
 * KB, so the array covers N * Hkv * Dv up to about 1.18 million: e.g. 2,300
 * tokens x 4 kv heads x Dv 128, or 4,600 tokens x 4 kv heads x Dv 64.
 * fix_attn_workspace_bytes(p, 0) gives the exact figure for a problem. */
#define FIX_NOALLOC_MAX_WORKSPACE_BYTES (16u * 1024u * 1024u)

/* Forward for callers that cannot allocate device memory.  (The FiX pages
 * have no counterpart to this entry point; it only changes where the
 * workspace lives.)
 *
 * Some callers cannot obtain a device workspace when they call: host code
 * handed only tensors and a stream, or a runtime whose device memory is
 * reserved up front, where an allocation would fail or synchronise.  This
 * call runs exactly fix_attn_fwd, with the same arguments except the
 * workspace, which it takes from one library-owned device array of
 * FIX_NOALLOC_MAX_WORKSPACE_BYTES that every GPU loading the library holds
 * until the process exits.  It calls no allocator.
 *   - Returns FIX_ERR_WORKSPACE if fix_attn_workspace_bytes(p, 0) exceeds
 *     FIX_NOALLOC_MAX_WORKSPACE_BYTES, and fix_attn_fwd's codes otherwise.
 *   - The first call on a device, with that device current, looks up the
 *     array's device address (cudaGetSymbolAddress) and caches it; make that
 *     first call before any stream capture.
 *   - All calls on a device share the array, which keeps the last call's
 *     contents; calls that overlap on the GPU (other streams or unordered
 *     host threads) race on it.  Order them on one stream.
 *   - A bounded device wait that expires records FIX_ERR_DEVICE_TIMEOUT in
 *     the array's status word; fix_attn_noalloc_device_status reads it. */
fix_status fix_attn_fwd_noalloc(const fix_attn_problem *p, const void *q, const void *k,
                                const void *v, const float *g, const void *o_norm_weight,
                                const void *o_gate, void *y, float *o_saved, float *m_saved,
                                float *rstd_saved, void *stream);

/* fix_attn_device_status for fix_attn_fwd_noalloc: synchronises `stream`,
 * then returns the status word that the last fix_attn_fwd_noalloc call on
 * the current device left in the library's array (FIX_OK or
 * FIX_ERR_DEVICE_TIMEOUT; FIX_OK before any such call), or FIX_ERR_CUDA if
 * the stream reports an error.  Allocates nothing. */
fix_status fix_attn_noalloc_device_status(void *stream);

/* Number of kernels that fix_attn_fwd (backward = 0) or fix_attn_bwd
 * (backward = 1) launches for this problem (0 if it is invalid). */
int fix_attn_kernel_count(const fix_attn_problem *p, int backward);

/* Static, human-readable name of a status code. */
const char *fix_attn_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* FIX_ATTN_H_ */
