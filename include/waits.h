/*
 * waits.h -- C ABI of libwaits.so, the B200 (sm_100a) WAITS prefill
 * KV-eviction path: score -> select -> compact.
 *
 * Method source: the WAITS README (stig.sh/Dirac-Notation/A2SF).
 *   - Opening summary: keys are retained by an accumulative attention score
 *     whose query rows are weighted by the sigmoid forgetting curve
 *     w[q] = 1 / (1 + exp(-a * (q - (N - b - 0.5)))).
 *   - Quickstart: init_cache keys "sigmoid_a" (a), "recent_budget" (R) and
 *     "select_budget" (B); Evaluation: the window b is the --window flag.
 *
 * Conventions shared by every entry point
 *   Layout    Packed varlen ("THD"): Q is [T, Hq, d], K and V are [T, Hkv, d],
 *             bf16, row-major, d contiguous; sequence i owns tokens
 *             [cu_seqlens[i], cu_seqlens[i+1]).  T = total_tokens.  Query
 *             head h reads KV head h / G with G = Hq / Hkv.
 *   Positions Sequence-local and 0-based: q, k in [0, N_i).
 *   Memory    Every pointer is DEVICE memory owned by the caller unless its
 *             comment says HOST.  The library allocates nothing and keeps no
 *             state between calls; scratch lives in the caller's workspace.
 *             The one exception is waits_score_static (below): its scratch
 *             is a fixed array inside the library, one per device, shared by
 *             every call on that device, so those calls must be serialised.
 *             Q, K, V must be 16-byte aligned.
 *   Streams   `stream` is a cudaStream_t passed as void* (NULL = legacy
 *             default stream).  Calls only enqueue work on it and return; the
 *             outputs are valid once the stream reaches that point.
 *   Errors    Arguments are validated on the host before anything is
 *             enqueued; a non-OK status means nothing was launched.  Problems
 *             only the device can see (malformed cu_seqlens, an index out of
 *             range handed to waits_compact, a bounded wait that gave up) set
 *             bits of a status word in the workspace and the affected work is
 *             skipped, never performed out of bounds; read it with
 *             waits_read_device_status().
 *   Inputs    Q and K must be finite (non-finite values give unspecified
 *             scores but never out-of-bounds accesses).
 */
#ifndef WAITS_H
#define WAITS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define WAITS_ABI_VERSION 1

typedef enum waits_status {
  WAITS_OK = 0,
  WAITS_ERR_ARG = 1,          /* null pointer, misalignment, bad a/b/R/B   */
  WAITS_ERR_SHAPE = 2,        /* inconsistent or out-of-range shape        */
  WAITS_ERR_UNSUPPORTED = 3,  /* head_dim not 64/128, G > 128, ...         */
  WAITS_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than required   */
  WAITS_ERR_CUDA = 5,         /* a CUDA runtime call failed                */
  WAITS_ERR_TIMEOUT = 6,      /* device status: a bounded wait gave up     */
  WAITS_ERR_DEVICE = 7        /* device status: other device-side problem  */
} waits_status;

/* Bits of the device status word (waits_read_device_status). */
#define WAITS_DEV_TIMEOUT        0x1u  /* a bounded spin/mbarrier wait expired */
#define WAITS_DEV_BAD_SEQLENS    0x2u  /* cu_seqlens not 0 <= ... <= T, or N > max_seqlen */
#define WAITS_DEV_PLAN_OVERFLOW  0x4u  /* internal: plan larger than its bound */
#define WAITS_DEV_BAD_INDEX      0x8u  /* waits_compact saw idx outside [0, N) */
#define WAITS_DEV_BAD_CURVE      0x10u /* a routed call's a or b was invalid for some sequence */

typedef struct waits_shape {
  int32_t nseq;             /* sequences in the packed batch, >= 1             */
  int32_t total_tokens;     /* T = cu_seqlens[nseq], >= 1                      */
  int32_t max_seqlen;       /* upper bound on every N_i (host-side value)      */
  int32_t num_q_heads;      /* Hq, a multiple of num_kv_heads                  */
  int32_t num_kv_heads;     /* Hkv >= 1                                        */
  int32_t head_dim;         /* d, 64 or 128                                    */
  const int32_t* cu_seqlens;/* DEVICE, int32 [nseq + 1], cu[0] = 0, non-decreasing */
} waits_shape;

/* Library ABI version (WAITS_ABI_VERSION of the build). */
int32_t waits_abi_version(void);

/* Static, NUL-terminated description of a status code. */
const char* waits_strerror(waits_status status);

/*
 * Description of the last CUDA runtime failure seen by a call on this host
 * thread (which step failed and CUDA's error name), "" if none.  The string
 * is owned by the library and stays valid until the next call that fails.
 */
const char* waits_last_error(void);

/*
 * Bytes of device workspace that waits_score / waits_compress need for
 * `shape` (any a, b, R, B).  Host-only; touches no device state.
 * Errors: WAITS_ERR_ARG if shape or bytes is NULL; shape errors as below.
 */
waits_status waits_workspace_size(const waits_shape* shape, size_t* bytes);

/*
 * Number of kernels one waits_score call with this shape, a and b enqueues:
 * 2 (the two scorer passes) when every scorer CTA can rebuild the work plan
 * itself -- at most 32 sequences and, from a bound on the rows whose fp32
 * weight is non-zero (about b + 89/a per sequence), at most 32 planned
 * entries per pass with all active rows of a sequence in 4 Q tiles -- else
 * 4 (a planner kernel first, and between the passes a kernel that merges
 * every row's bias once; 3, without it, under WAITS_SCORER=tc).  Either way
 * the results are the same.  The environment variable
 * WAITS_PLANNER_KERNEL=1 makes every call take the planner kernel (a
 * debugging aid).
 * Host-only; touches no device state.
 * Errors: WAITS_ERR_ARG if shape or kernels is NULL, or a < 0 / non-finite,
 * or b < 0; shape errors as below.
 */
waits_status waits_score_kernels(const waits_shape* shape, float a, int32_t b,
                                 int32_t* kernels);

/*
 * Accumulative forgetting-curve score (README opening summary).  For every
 * sequence, KV head g and key k:
 *   scores[g * T + cu[i] + k] =
 *     sum_{h in group g} sum_{q >= k} w[q] * softmax_k'(Q[q,h].K[k',g] / sqrt(d))[k]
 * with w from the forgetting curve, N = N_i, and the sum restricted to rows
 * whose fp32 weight 1.0f/(1.0f+expf(-a*(q-c))) is non-zero (the others add
 * less than 1e-37 each).
 *   Q, K       bf16 [T, Hq, d] / [T, Hkv, d]
 *   a          slope, finite and >= 0 (0 gives H2O; 1e4 a step)
 *   b          window, >= 0
 *   scores     fp32 [Hkv, T], written for every token
 *   workspace  >= waits_workspace_size() bytes, 256-byte aligned
 * Errors: ARG (null, misaligned, a < 0 or non-finite, b < 0), SHAPE,
 * UNSUPPORTED, WORKSPACE, CUDA.
 */
waits_status waits_score(const waits_shape* shape, const void* Q, const void* K,
                         float a, int32_t b, float* scores, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * waits_score with the softmax normalisers supplied by the caller: the
 * prefill attention that precedes the scorer (the README's opening summary
 * has WAITS registered as an attention function, so it runs right after
 * the layer's attention) has already computed every row's log-sum-exp, as a
 * FlashAttention forward returns it.  The first pass (row statistics) is
 * then skipped and only the weighted column sums run, half the work.
 *   lse   DEVICE fp32 [Hq, T]: lse[h * T + t] = natural log of
 *         sum_{k <= q} exp(Q[t,h] . K[k,g] / sqrt(d)), q the sequence-local
 *         position of packed token t (keys of its own sequence only); read
 *         only for rows whose fp32 weight is non-zero
 *   other arguments, layouts and results as waits_score; with the exact
 *   LSE the scores equal waits_score's within fp32 rounding.
 * Errors: as waits_score, plus ARG if lse is NULL or not 4-byte aligned.
 */
waits_status waits_score_with_lse(const waits_shape* shape, const void* Q, const void* K,
                                  const float* lse, float a, int32_t b, float* scores,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * waits_score with a forgetting curve per sequence: the README's routed
 * WAITS ("Training the routing policy" and Evaluation's --waits_table) picks
 * one (a, b) action per sample, so one packed batch mixes curves.
 *   a     DEVICE fp32 [nseq]: slope of sequence i, finite and >= 0
 *   b     DEVICE int32 [nseq]: window of sequence i, >= 0
 *   other arguments, layouts and results as waits_score, each sequence
 *   scored with its own (a[i], b[i]).  The work plan is built on the device
 *   (3 kernels).  A sequence whose a or b is invalid sets WAITS_DEV_BAD_CURVE
 *   and gets zero scores.
 * Errors: as waits_score, plus ARG if a or b is NULL or misaligned.
 */
waits_status waits_score_routed(const waits_shape* shape, const void* Q, const void* K,
                                const float* a, const int32_t* b, float* scores,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * waits_score_routed followed by waits_select_compact (per-sequence curves,
 * then selection and compaction), all enqueued on `stream`.
 */
waits_status waits_compress_routed(const waits_shape* shape, const void* Q, const void* K,
                                   const void* V, const float* a, const int32_t* b, int32_t R,
                                   int32_t B, float* scores, int32_t* idx, int32_t* kept_len,
                                   void* K_out, void* V_out, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * Selection (README Quickstart budgets).  Per sequence i and KV head g:
 * keep the recent window [N-R, N) and the B-R positions of [0, N-R) with the
 * largest score, ties to the lower index; N <= B keeps every position.
 *   idx        int32 [nseq, Hkv, B]: kept positions, sequence-local,
 *              ascending; entries j >= kept_len[i] are -1
 *   kept_len   int32 [nseq]: min(N_i, B)
 *   workspace  may be NULL (this call needs none); kept for ABI symmetry
 * Errors: ARG (null, R < 0, R > B, B < 1), SHAPE, CUDA.
 */
waits_status waits_select(const waits_shape* shape, const float* scores,
                          int32_t R, int32_t B, int32_t* idx, int32_t* kept_len,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * Compaction ("retaining key-value pairs", README opening summary):
 *   K_out[i, g, j, :] = K[cu[i] + idx[i, g, j], g, :] for j < kept_len[i],
 *   zero for j >= kept_len[i]; same for V.  Bit-exact copy.
 *   K_out, V_out  bf16 [nseq, Hkv, B, d], 16-byte aligned
 * An idx entry outside [0, N_i) sets WAITS_DEV_BAD_INDEX (in `workspace` if
 * given) and that row is written as zeros.
 * Errors: ARG, SHAPE, UNSUPPORTED, CUDA.
 */
waits_status waits_compact(const waits_shape* shape, const void* K, const void* V,
                           const int32_t* idx, const int32_t* kept_len, int32_t B,
                           void* K_out, void* V_out, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * waits_select followed by waits_compact, in one kernel: the same idx,
 * kept_len, K_out and V_out bit for bit.  The selecting CTAs copy the K and
 * V rows of the positions they keep as soon as those positions are known, so
 * the compaction costs no launch or wait of its own.  (waits_compress uses
 * it.)  Arguments as in the two calls; the indices come from the selection,
 * so WAITS_DEV_BAD_INDEX cannot arise.
 * Errors: ARG, SHAPE, UNSUPPORTED, CUDA.
 */
waits_status waits_select_compact(const waits_shape* shape, const float* scores,
                                  const void* K, const void* V, int32_t R, int32_t B,
                                  int32_t* idx, int32_t* kept_len, void* K_out, void* V_out,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * score -> select -> compact in one call, all enqueued on `stream`.
 * Arguments as above; `scores` is an output too.
 */
waits_status waits_compress(const waits_shape* shape, const void* Q, const void* K,
                            const void* V, float a, int32_t b, int32_t R, int32_t B,
                            float* scores, int32_t* idx, int32_t* kept_len,
                            void* K_out, void* V_out, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * waits_compress for the KV heads [kv_head_begin, kv_head_end) of a layer,
 * reading the layer's own Q, K and V in place: a tensor-parallel rank that
 * owns those heads scores, selects and compacts exactly them (every KV head,
 * with its query heads, is independent of the others; no exchange between
 * ranks is needed, since a rank's compacted cache is what its decode reads).
 *   shape            the whole layer (num_q_heads, num_kv_heads of the tensors)
 *   Q, K, V          the whole layer's tensors, as for waits_compress
 *   scores           fp32 [Hs, T], Hs = kv_head_end - kv_head_begin: row i
 *                    is KV head kv_head_begin + i
 *   idx, kept_len    [nseq, Hs, B], [nseq]
 *   K_out, V_out     bf16 [nseq, Hs, B, d]
 *   workspace        >= waits_workspace_size() of the layer (a range needs no more)
 * The results equal the rows of a whole-layer call for those heads, up to
 * the fp32 rounding of sums whose order depends on the work split.
 * Errors: as waits_compress, plus ARG for an empty or out-of-range range.
 */
waits_status waits_compress_heads(const waits_shape* shape, int32_t kv_head_begin,
                                  int32_t kv_head_end, const void* Q, const void* K,
                                  const void* V, float a, int32_t b, int32_t R, int32_t B,
                                  float* scores, int32_t* idx, int32_t* kept_len, void* K_out,
                                  void* V_out, void* workspace, size_t workspace_bytes,
                                  void* stream);

/* Device buffers that waits_compress_host stages through (caller-owned). */
typedef struct waits_device_buffers {
  void* Q;          /* bf16 [T, Hq, d]  */
  void* K;          /* bf16 [T, Hkv, d] */
  void* V;          /* bf16 [T, Hkv, d] */
  float* scores;    /* fp32 [Hkv, T]    */
  int32_t* idx;     /* [nseq, Hkv, B]   */
  int32_t* kept_len;/* [nseq]           */
  void* K_out;      /* bf16 [nseq, Hkv, B, d] */
  void* V_out;      /* bf16 [nseq, Hkv, B, d] */
  int32_t* cu_seqlens; /* [nseq + 1]    */
} waits_device_buffers;

/*
 * Host-buffer variant of waits_compress: copies the inputs from HOST memory
 * (pinned memory makes the copies asynchronous), runs the path, and copies
 * idx, kept_len, K_out and V_out back to HOST memory, all on `stream`.
 * Only the rows the scorer can read are sent: each sequence's query rows
 * from a conservative lower bound of the first non-zero-weight row on, and
 * all of K.  V is read only where a row is kept: when V_host is page-locked
 * and mapped into the device's address space (cudaHostAlloc, cudaMallocHost
 * and cudaHostRegister memory under unified addressing, torch's
 * pin_memory), the compaction kernel reads the kept rows straight from it
 * over the bus and dev->V is not used; otherwise all of V is copied to
 * dev->V first.  The call returns once the work is enqueued; the host
 * outputs are valid after the stream is synchronised, and V_host must stay
 * unchanged until then.
 *   cu_seqlens_host  HOST int32 [nseq + 1]
 *   Q_host, K_host, V_host, idx_host, kept_len_host, K_out_host,
 *   V_out_host       HOST, same layouts as the device versions
 *   dev              device staging buffers; dev->cu_seqlens receives the
 *                    offsets and shape->cu_seqlens is ignored
 *   h2d_bytes, d2h_bytes  optional HOST out: bytes moved each way (the
 *                    kept V rows read over the bus count as host to device)
 * Errors: as waits_compress, plus SHAPE if cu_seqlens_host is inconsistent.
 */
waits_status waits_compress_host(const waits_shape* shape,
                                 const int32_t* cu_seqlens_host,
                                 const void* Q_host, const void* K_host,
                                 const void* V_host, float a, int32_t b,
                                 int32_t R, int32_t B, int32_t* idx_host,
                                 int32_t* kept_len_host, void* K_out_host,
                                 void* V_out_host,
                                 const waits_device_buffers* dev,
                                 void* workspace, size_t workspace_bytes,
                                 void* stream, size_t* h2d_bytes,
                                 size_t* d2h_bytes);

/*
 * Largest scratch waits_score_static can use: 32 MiB, enough for one
 * Llama-3.1-8B-shaped layer (N = 32768, 32/8 heads) whose
 * waits_workspace_size() is 13.3 MiB.
 */
#define WAITS_STATIC_WORKSPACE_BYTES (32u << 20)

/*
 * waits_score without a caller-supplied workspace.  The WAITS pages have no
 * counterpart of this call: it exists for callers that cannot allocate
 * device memory -- a plugin whose host engine owns the whole device pool, or
 * code running where an allocation is forbidden or would synchronise the
 * device.  The scorer's scratch lives in one file-scope device array of
 * WAITS_STATIC_WORKSPACE_BYTES that every GPU loading the library keeps
 * until the process exits; the call allocates nothing.
 *   Arguments, layouts and results as waits_score.
 *   Errors: as waits_score; WAITS_ERR_WORKSPACE when
 *   waits_workspace_size(shape) exceeds WAITS_STATIC_WORKSPACE_BYTES (nothing
 *   is launched).
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it for the
 *   device's current CUDA context; a new context (after cudaDeviceReset, for
 *   instance) looks it up again.  Make the first call on a device before any
 *   stream capture.
 *   Every call on a device shares the one array, which keeps the previous
 *   call's contents; every part of it a call reads is written earlier in
 *   that call, so nothing needs clearing.  Calls whose work overlaps on the
 *   GPU (other streams, other host threads) race on it: serialise them.
 *   The call's device status word lives in the array: read it with
 *   waits_read_static_status.
 */
waits_status waits_score_static(const waits_shape* shape, const void* Q, const void* K,
                                float a, int32_t b, float* scores, void* stream);

/*
 * Synchronise `stream` and read the device status word that the last
 * waits_score_static call on the current device left in the library's
 * static scratch (bits WAITS_DEV_*; 0 = clean).  Like that entry point, it
 * has no counterpart on the WAITS pages.  Errors: ARG (status_bits NULL),
 * CUDA.
 */
waits_status waits_read_static_status(void* stream, uint32_t* status_bits);

/*
 * Synchronise `stream` and read the device status word of `workspace`
 * (bits WAITS_DEV_*; 0 = clean).  The word is cleared at the start of every
 * waits_score / waits_compress.  Errors: ARG, WORKSPACE, CUDA.
 */
waits_status waits_read_device_status(const void* workspace,
                                      size_t workspace_bytes, void* stream,
                                      uint32_t* status_bits);

/*
 * Bytes of device workspace waits_decode_attention needs.  Host-only.
 * Errors: ARG (bytes NULL), SHAPE, UNSUPPORTED (head_dim not 64 or 128).
 */
waits_status waits_decode_workspace_size(int32_t nseq, int32_t num_q_heads, int32_t head_dim,
                                         int32_t capacity, size_t* bytes);

/*
 * One decode step of attention over the compacted cache: what the model
 * runs after prefill compression (README Quickstart: model.generate after
 * init_cache).  For sequence s and query head h, KV head g = h / G:
 *   out[s, h] = sum_{j < cache_len[s]} softmax_j(q[s, h] . K_cache[s, g, j] / sqrt(d))
 *               * V_cache[s, g, j]
 *   lse[s, h] = natural log of that softmax's normaliser (-inf, and out = 0,
 *               for an empty cache)
 *   q          DEVICE bf16 [nseq, Hq, d], 16-byte aligned
 *   K_cache, V_cache  DEVICE bf16 [nseq, Hkv, capacity, d] (waits_compress's
 *               K_out, V_out with capacity = B, or any cache of that layout;
 *               slots past cache_len[s] are not read)
 *   cache_len  DEVICE int32 [nseq]: valid slots (kept_len, plus any decoded
 *               tokens the caller appended); clamped to [0, capacity]
 *   out        DEVICE fp32 [nseq, Hq, d];  lse  DEVICE fp32 [nseq, Hq] or NULL
 *   workspace  >= waits_decode_workspace_size() bytes, 16-byte aligned
 * Two kernels on `stream` (per 256 cache slots, then the merge).  Hq / Hkv
 * at most 16.
 * Errors: ARG, SHAPE, UNSUPPORTED, WORKSPACE, CUDA.
 */
waits_status waits_decode_attention(int32_t nseq, int32_t num_q_heads, int32_t num_kv_heads,
                                    int32_t head_dim, int32_t capacity, const void* q,
                                    const void* K_cache, const void* V_cache,
                                    const int32_t* cache_len, float* out, float* lse,
                                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Testing aid, no counterpart on the WAITS pages: y[i] = the scorer's
 * FMA-pipe 2^x of x[i] (the exponential that part of the scorer's epilogue
 * runs instead of the MUFU ex2: a round-to-nearest split x = n + f, a cubic
 * in f with relative error 1.013e-4 (1.02e-4 with fp32 rounding), 2^n built
 * from the bits of the rounding sum).  x is first raised to at least -127,
 * so x <= -126.5 gives +0; defined for x <= 127 (the epilogue's arguments
 * never exceed 0 beyond rounding); exact powers of two at integers in
 * [-126, 127].  x and y are DEVICE fp32 arrays of n elements.  Errors: ARG
 * (null pointer, n < 0), CUDA.
 */
waits_status waits_test_exp2_poly(const float* x, float* y, int64_t n, void* stream);

/*
 * Environment variables read at each waits_score / waits_compress call
 * (testing aids): WAITS_WAIT_LIMIT_NS sets the limit of the scorer's
 * bounded waits in nanoseconds (default 2 s); WAITS_TEST_WITHHOLD_MMA=1
 * makes the scorer's MMA warp issue nothing, so the waits for its
 * accumulators run out: the call ends early, with WAITS_DEV_TIMEOUT set and
 * the scores unspecified, and leaves the context usable.  WAITS_SCORER=tc
 * makes both passes of every plan run the general scorer kernel (by
 * default the kernel with 256-column accumulators runs pass 1 of every plan
 * and pass 2 of the small ones; the scores are bit-identical either way).
 */

#ifdef __cplusplus
}
#endif

#endif /* WAITS_H */
