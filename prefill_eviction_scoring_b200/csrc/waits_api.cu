// C ABI of libwaits.so: host-side validation, workspace carving and launches
// on the caller's stream.  Declarations and contracts: include/waits.h.
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "plan_core.cuh"

#include <cstdarg>

using namespace waits;

namespace {

thread_local char g_last_error[512] = "";
thread_local char g_detail[256] = "";

waits_status cuda_fail(const char* what, cudaError_t err) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)%s%s", what, cudaGetErrorName(err),
           cudaGetErrorString(err), g_detail[0] ? "; " : "", g_detail);
  g_detail[0] = 0;
  return WAITS_ERR_CUDA;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

waits_status check_shape(const waits_shape* s) {
  if (!s || !s->cu_seqlens) return WAITS_ERR_ARG;
  if (s->nseq < 1 || s->total_tokens < 1 || s->max_seqlen < 1 || s->num_kv_heads < 1 ||
      s->num_q_heads < 1)
    return WAITS_ERR_SHAPE;
  if (s->num_q_heads % s->num_kv_heads) return WAITS_ERR_SHAPE;
  if (s->max_seqlen > s->total_tokens) return WAITS_ERR_SHAPE;
  if (s->head_dim != 64 && s->head_dim != 128) return WAITS_ERR_UNSUPPORTED;
  if (s->num_q_heads / s->num_kv_heads > kTile) return WAITS_ERR_UNSUPPORTED;
  // every flat index below fits comfortably in 64 bits; keep T*Hq*d in 2^40
  const double elems = (double)s->total_tokens * s->num_q_heads * s->head_dim;
  if (elems > 1099511627776.0 || s->nseq > s->total_tokens) return WAITS_ERR_SHAPE;
  return WAITS_OK;
}

Layout layout_of(const waits_shape* s) {
  return make_layout(s->nseq, s->total_tokens, s->num_q_heads, s->num_kv_heads);
}

waits_status check_ws(const waits_shape* s, const void* ws, size_t bytes) {
  if (!ws) return WAITS_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return WAITS_ERR_ARG;
  if (bytes < layout_of(s).total) return WAITS_ERR_WORKSPACE;
  return WAITS_OK;
}

waits_status check_budget(int32_t R, int32_t B) {
  if (B < 1 || R < 0 || R > B) return WAITS_ERR_ARG;
  return WAITS_OK;
}

int grid_size() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return sms < kMaxGrid ? sms : kMaxGrid;
}

// Whether every scorer CTA can rebuild the plan itself (plan_core.cuh): at
// most kLocalMax sequences and kLocalMax entries in each pass, and every
// sequence's active rows within the stationary Q tiles of one pass-2 entry.
// The bound on a sequence's active rows (those whose fp32 weight is not 0,
// about b + 89/a of them) is loose by a few rows; the device counts exactly
// and flags a plan overflow rather than run if the bound was ever short.
// WAITS_DEVICE_PLAN=1 (debugging, tests): a one-sequence batch is planned
// on the device like any other instead of by the host.
bool host_plan_allowed() {
  const char* force = std::getenv("WAITS_DEVICE_PLAN");
  return !(force && force[0] == '1');
}

// WAITS_WAIT_LIMIT_NS (testing aid): limit of the scorer's bounded waits in
// nanoseconds, default 2 s.  WAITS_TEST_WITHHOLD_MMA=1 (testing aid): the
// scorer's MMA warp issues nothing, so the waits for its accumulators run out
// and the call ends with WAITS_DEV_TIMEOUT set.
uint64_t wait_limit_ns() {
  const char* v = std::getenv("WAITS_WAIT_LIMIT_NS");
  if (!v || !v[0]) return 2000000000ull;
  char* end = nullptr;
  const unsigned long long x = std::strtoull(v, &end, 10);
  return end && *end == '\0' && x > 0 ? (uint64_t)x : 2000000000ull;
}

// WAITS_SCORER=tc (debugging, tests): local plans also run the general
// scorer kernel (128-column accumulators) instead of the sparse one.
bool force_tc_scorer() {
  const char* v = std::getenv("WAITS_SCORER");
  return v && v[0] == 't' && v[1] == 'c' && v[2] == '\0';
}

bool withhold_mma() {
  const char* v = std::getenv("WAITS_TEST_WITHHOLD_MMA");
  return v && v[0] == '1';
}

bool local_plan_fits(const waits_shape* s, float a, int32_t b) {
  // WAITS_PLANNER_KERNEL=1 (debugging, tests): always plan with the planner kernel
  const char* force = std::getenv("WAITS_PLANNER_KERNEL");
  if (force && force[0] == '1') return false;
  if (s->nseq > kLocalMax) return false;
  const int tokq = tokens_per_qtile(s->num_q_heads / s->num_kv_heads);
  double rows = s->max_seqlen;                       // a = 0: every row is active
  if (a > 0.0f)
    rows = std::fmin(rows, (double)b + 8.0 + std::ceil(89.0 / a) + s->max_seqlen / 4194304.0);
  const int64_t nqt = (int64_t)std::ceil(rows / tokq);
  if (nqt > kMaxStat) return false;
  const int64_t e1 = (int64_t)s->num_kv_heads * s->nseq * ((nqt + kMaxStat1 - 1) / kMaxStat1);
  const int64_t e2 = (int64_t)s->num_kv_heads * s->nseq;
  return e1 <= kLocalMax && e2 <= kLocalMax;
}

uint32_t* status_word(void* ws, size_t bytes) {
  if (!ws || bytes < sizeof(PlanHeader) || !aligned(ws, 256)) return nullptr;
  return &reinterpret_cast<PlanHeader*>(ws)->status;
}

waits_status enqueue_score(const waits_shape* s, const void* Q, const void* K, float a,
                           int32_t b, float* scores, void* ws, cudaStream_t st,
                           const float* lse = nullptr, const float* seq_a = nullptr,
                           const int32_t* seq_b = nullptr, int q_row_heads = 0,
                           int kv_row_heads = 0) {
  const Layout L = layout_of(s);
  uint8_t* base = static_cast<uint8_t*>(ws);
  const int grid = grid_size();
  if (grid <= 0) return cuda_fail("device query", cudaGetLastError());
  PlanArgs pa{};
  pa.cu = s->cu_seqlens;
  pa.nseq = s->nseq;
  pa.T = s->total_tokens;
  pa.max_seqlen = s->max_seqlen;
  pa.Hq = s->num_q_heads;
  pa.Hkv = s->num_kv_heads;
  pa.G = s->num_q_heads / s->num_kv_heads;
  pa.tokq = tokens_per_qtile(pa.G);
  pa.a = a;
  pa.b = b;
  pa.seq_a = seq_a;
  pa.seq_b = seq_b;
  pa.grid = grid;
  pa.hdr = reinterpret_cast<PlanHeader*>(base + L.header);
  pa.seqs = reinterpret_cast<SeqInfo*>(base + L.seqs);
  pa.e1 = reinterpret_cast<Entry*>(base + L.e1);
  pa.e2 = reinterpret_cast<Entry*>(base + L.e2);
  pa.c2 = reinterpret_cast<uint32_t*>(base + L.c2);
  pa.max_e1 = L.max_e1;
  pa.max_e2 = L.max_e2;
  pa.max_u1 = L.max_u1;
  pa.max_u2 = L.max_u2;
  pa.scores = scores;
  // routed calls plan on the device from the per-sequence parameters
  const bool local = !seq_a && local_plan_fits(s, a, b);
  cudaError_t err = cudaSuccess;
  if (!local) {
    err = launch_plan(pa, st);
    if (err != cudaSuccess) return cuda_fail("planner launch", err);
  }

  PassArgs p{};
  p.Q = static_cast<const uint16_t*>(Q);
  p.K = static_cast<const uint16_t*>(K);
  p.T = s->total_tokens;
  p.Hq = s->num_q_heads;
  p.Hkv = s->num_kv_heads;
  p.q_row_heads = q_row_heads > 0 ? q_row_heads : s->num_q_heads;
  p.kv_row_heads = kv_row_heads > 0 ? kv_row_heads : s->num_kv_heads;
  p.G = pa.G;
  p.tokq = pa.tokq;
  p.d = s->head_dim;
  p.a = a;
  p.b = b;
  p.scale2 = (float)(1.4426950408889634 / std::sqrt((double)s->head_dim));
  p.hdr = pa.hdr;
  p.seqs = pa.seqs;
  p.e1 = pa.e1;
  p.e2 = pa.e2;
  p.c2 = pa.c2;
  p.part1 = reinterpret_cast<float2*>(base + L.part1);
  p.part2 = reinterpret_cast<float*>(base + L.part2);
  p.scores = scores;
  p.status = &pa.hdr->status;
  p.local_plan = local ? 1 : 0;
  p.lse = lse;
  p.wait_ns = wait_limit_ns();
  p.withhold_mma = withhold_mma() ? 1 : 0;
  p.cu = s->cu_seqlens;
  p.nseq = s->nseq;
  p.max_seqlen = s->max_seqlen;
  HostPlan hp;
  p.host_plan = local && s->nseq == 1 && host_plan_allowed() &&
                        host_plan_single(p.T, p.max_seqlen, p.Hkv, p.tokq, a, b, grid, &hp)
                    ? 1
                    : 0;
  // local plans hold only P2Q entries in pass 2: the 256-column kernel for
  // both passes; the planner kernel's plans: its pass 1, and the general
  // kernel's pass 2 (which also handles stationary K tiles)
  if (force_tc_scorer())
    err = launch_score_passes(p, p.host_plan ? &hp : nullptr, grid, st);
  else if (local)
    err = launch_sparse_passes(p, p.host_plan ? &hp : nullptr, grid, st);
  else if (lse)
    err = launch_score_passes(p, nullptr, grid, st);   // pass 2 only
  else if ((err = launch_sparse_pass1(p, grid, st)) == cudaSuccess &&
           (err = launch_row_bias(p, L.max_e1, st)) == cudaSuccess) {
    PassArgs p2 = p;
    p2.bias_ready = 1;   // pass 2 reads the merged row biases
    err = launch_score_pass2(p2, grid, st);
  }
  if (err != cudaSuccess) return cuda_fail("scorer launch", err);
  return WAITS_OK;
}

waits_status check_score_args(const waits_shape* s, const void* Q, const void* K, float a,
                              int32_t b, const float* scores) {
  if (!Q || !K || !scores) return WAITS_ERR_ARG;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(scores, 4)) return WAITS_ERR_ARG;
  if (!std::isfinite(a) || a < 0.0f || b < 0) return WAITS_ERR_ARG;
  (void)s;
  return WAITS_OK;
}

waits_status check_select_args(const float* scores, int32_t R, int32_t B, const int32_t* idx,
                               const int32_t* kept_len) {
  if (!scores || !idx || !kept_len) return WAITS_ERR_ARG;
  return check_budget(R, B);
}

waits_status check_compact_args(const void* K, const void* V, const int32_t* idx,
                                const int32_t* kept_len, int32_t B, const void* Ko,
                                const void* Vo) {
  if (!K || !V || !idx || !kept_len || !Ko || !Vo) return WAITS_ERR_ARG;
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(Ko, 16) || !aligned(Vo, 16))
    return WAITS_ERR_ARG;
  if (B < 1) return WAITS_ERR_ARG;
  return WAITS_OK;
}

}  // namespace

namespace waits {
void set_error_detail(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
}
}  // namespace waits

extern "C" {

int32_t waits_abi_version(void) { return WAITS_ABI_VERSION; }

const char* waits_last_error(void) { return g_last_error; }

const char* waits_strerror(waits_status st) {
  switch (st) {
    case WAITS_OK: return "ok";
    case WAITS_ERR_ARG: return "invalid argument (null, misaligned, or a/b/R/B out of range)";
    case WAITS_ERR_SHAPE: return "invalid or inconsistent shape";
    case WAITS_ERR_UNSUPPORTED: return "unsupported configuration (head_dim must be 64 or 128, G <= 128)";
    case WAITS_ERR_WORKSPACE: return "workspace missing or smaller than waits_workspace_size()";
    case WAITS_ERR_CUDA: return "a CUDA runtime call failed";
    case WAITS_ERR_TIMEOUT: return "a bounded device-side wait expired";
    case WAITS_ERR_DEVICE: return "device-side error (see WAITS_DEV_* status bits)";
  }
  return "unknown status";
}

waits_status waits_workspace_size(const waits_shape* shape, size_t* bytes) {
  if (!bytes) return WAITS_ERR_ARG;
  const waits_status st = check_shape(shape);
  if (st != WAITS_OK) return st;
  *bytes = layout_of(shape).total;
  return WAITS_OK;
}

waits_status waits_score_kernels(const waits_shape* shape, float a, int32_t b,
                                 int32_t* kernels) {
  if (!kernels || !std::isfinite(a) || a < 0.0f || b < 0) return WAITS_ERR_ARG;
  const waits_status st = check_shape(shape);
  if (st != WAITS_OK) return st;
  *kernels = local_plan_fits(shape, a, b) ? 2 : (force_tc_scorer() ? 3 : 4);
  return WAITS_OK;
}

waits_status waits_score(const waits_shape* shape, const void* Q, const void* K, float a,
                         int32_t b, float* scores, void* workspace, size_t workspace_bytes,
                         void* stream) {
  waits_status st = check_shape(shape);
  if (st == WAITS_OK) st = check_score_args(shape, Q, K, a, b, scores);
  if (st == WAITS_OK) st = check_ws(shape, workspace, workspace_bytes);
  if (st != WAITS_OK) return st;
  return enqueue_score(shape, Q, K, a, b, scores, workspace, static_cast<cudaStream_t>(stream));
}

waits_status waits_score_with_lse(const waits_shape* shape, const void* Q, const void* K,
                                  const float* lse, float a, int32_t b, float* scores,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  waits_status st = check_shape(shape);
  if (st == WAITS_OK) st = check_score_args(shape, Q, K, a, b, scores);
  if (st == WAITS_OK && (!lse || !aligned(lse, 4))) st = WAITS_ERR_ARG;
  if (st == WAITS_OK) st = check_ws(shape, workspace, workspace_bytes);
  if (st != WAITS_OK) return st;
  return enqueue_score(shape, Q, K, a, b, scores, workspace, static_cast<cudaStream_t>(stream),
                       lse);
}

waits_status waits_score_routed(const waits_shape* shape, const void* Q, const void* K,
                                const float* a, const int32_t* b, float* scores,
                                void* workspace, size_t workspace_bytes, void* stream) {
  waits_status st = check_shape(shape);
  if (st == WAITS_OK) st = check_score_args(shape, Q, K, 0.0f, 0, scores);
  if (st == WAITS_OK && (!a || !b || !aligned(a, 4) || !aligned(b, 4))) st = WAITS_ERR_ARG;
  if (st == WAITS_OK) st = check_ws(shape, workspace, workspace_bytes);
  if (st != WAITS_OK) return st;
  return enqueue_score(shape, Q, K, 0.0f, 0, scores, workspace,
                       static_cast<cudaStream_t>(stream), nullptr, a, b);
}

waits_status waits_compress_routed(const waits_shape* shape, const void* Q, const void* K,
                                   const void* V, const float* a, const int32_t* b, int32_t R,
                                   int32_t B, float* scores, int32_t* idx, int32_t* kept_len,
                                   void* K_out, void* V_out, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  waits_status st = waits_score_routed(shape, Q, K, a, b, scores, workspace, workspace_bytes,
                                       stream);
  if (st != WAITS_OK) return st;
  return waits_select_compact(shape, scores, K, V, R, B, idx, kept_len, K_out, V_out, workspace,
                              workspace_bytes, stream);
}

waits_status waits_select(const waits_shape* shape, const float* scores, int32_t R, int32_t B,
                          int32_t* idx, int32_t* kept_len, void* workspace,
                          size_t workspace_bytes, void* stream) {
  waits_status st = check_shape(shape);
  if (st == WAITS_OK) st = check_select_args(scores, R, B, idx, kept_len);
  if (st != WAITS_OK) return st;
  const cudaError_t err = launch_select(scores, shape->cu_seqlens, shape->nseq,
                                        shape->total_tokens, shape->num_kv_heads, R, B, idx,
                                        kept_len, status_word(workspace, workspace_bytes),
                                        static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail("select launch", err);
  return WAITS_OK;
}

waits_status waits_compact(const waits_shape* shape, const void* K, const void* V,
                           const int32_t* idx, const int32_t* kept_len, int32_t B, void* K_out,
                           void* V_out, void* workspace, size_t workspace_bytes, void* stream) {
  waits_status st = check_shape(shape);
  if (st == WAITS_OK) st = check_compact_args(K, V, idx, kept_len, B, K_out, V_out);
  if (st != WAITS_OK) return st;
  const cudaError_t err = launch_compact(
      static_cast<const uint16_t*>(K), static_cast<const uint16_t*>(V), shape->cu_seqlens, idx,
      kept_len, shape->nseq, shape->num_kv_heads, shape->head_dim, B,
      static_cast<uint16_t*>(K_out), static_cast<uint16_t*>(V_out),
      status_word(workspace, workspace_bytes), static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail("compact launch", err);
  return WAITS_OK;
}

waits_status waits_compress(const waits_shape* shape, const void* Q, const void* K,
                            const void* V, float a, int32_t b, int32_t R, int32_t B,
                            float* scores, int32_t* idx, int32_t* kept_len, void* K_out,
                            void* V_out, void* workspace, size_t workspace_bytes,
                            void* stream) {
  waits_status st = check_shape(shape);
  if (st == WAITS_OK) st = check_score_args(shape, Q, K, a, b, scores);
  if (st == WAITS_OK) st = check_select_args(scores, R, B, idx, kept_len);
  if (st == WAITS_OK) st = check_compact_args(K, V, idx, kept_len, B, K_out, V_out);
  if (st == WAITS_OK) st = check_ws(shape, workspace, workspace_bytes);
  if (st != WAITS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = enqueue_score(shape, Q, K, a, b, scores, workspace, s);
  if (st != WAITS_OK) return st;
  const cudaError_t err = launch_select(
      scores, shape->cu_seqlens, shape->nseq, shape->total_tokens, shape->num_kv_heads, R, B,
      idx, kept_len, status_word(workspace, workspace_bytes), s, static_cast<const uint16_t*>(K),
      static_cast<const uint16_t*>(V), shape->head_dim, static_cast<uint16_t*>(K_out),
      static_cast<uint16_t*>(V_out));
  if (err != cudaSuccess) return cuda_fail("select-compact launch", err);
  return WAITS_OK;
}

waits_status waits_compress_heads(const waits_shape* shape, int32_t kv_head_begin,
                                  int32_t kv_head_end, const void* Q, const void* K,
                                  const void* V, float a, int32_t b, int32_t R, int32_t B,
                                  float* scores, int32_t* idx, int32_t* kept_len, void* K_out,
                                  void* V_out, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  waits_status st = check_shape(shape);
  if (st != WAITS_OK) return st;
  if (kv_head_begin < 0 || kv_head_end <= kv_head_begin || kv_head_end > shape->num_kv_heads)
    return WAITS_ERR_ARG;
  if (!Q || !K || !V) return WAITS_ERR_ARG;
  // the heads [begin, end) of the layer as a layer of their own: the same
  // token rows (rows keep the layer's head count), shifted base pointers
  const int G = shape->num_q_heads / shape->num_kv_heads, d = shape->head_dim;
  waits_shape sub = *shape;
  sub.num_kv_heads = kv_head_end - kv_head_begin;
  sub.num_q_heads = sub.num_kv_heads * G;
  const uint16_t* Qs = static_cast<const uint16_t*>(Q) + (size_t)kv_head_begin * G * d;
  const uint16_t* Ks = static_cast<const uint16_t*>(K) + (size_t)kv_head_begin * d;
  const uint16_t* Vs = static_cast<const uint16_t*>(V) + (size_t)kv_head_begin * d;
  st = check_score_args(&sub, Qs, Ks, a, b, scores);
  if (st == WAITS_OK) st = check_select_args(scores, R, B, idx, kept_len);
  if (st == WAITS_OK) st = check_compact_args(Ks, Vs, idx, kept_len, B, K_out, V_out);
  if (st == WAITS_OK) st = check_ws(&sub, workspace, workspace_bytes);
  if (st != WAITS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = enqueue_score(&sub, Qs, Ks, a, b, scores, workspace, s, nullptr, nullptr, nullptr,
                     shape->num_q_heads, shape->num_kv_heads);
  if (st != WAITS_OK) return st;
  const cudaError_t err = launch_select(
      scores, sub.cu_seqlens, sub.nseq, sub.total_tokens, sub.num_kv_heads, R, B, idx, kept_len,
      status_word(workspace, workspace_bytes), s, Ks, Vs, d, static_cast<uint16_t*>(K_out),
      static_cast<uint16_t*>(V_out), shape->num_kv_heads);
  if (err != cudaSuccess) return cuda_fail("select-compact launch", err);
  return WAITS_OK;
}

waits_status waits_select_compact(const waits_shape* shape, const float* scores,
                                  const void* K, const void* V, int32_t R, int32_t B,
                                  int32_t* idx, int32_t* kept_len, void* K_out, void* V_out,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  waits_status st = check_shape(shape);
  if (st == WAITS_OK) st = check_select_args(scores, R, B, idx, kept_len);
  if (st == WAITS_OK) st = check_compact_args(K, V, idx, kept_len, B, K_out, V_out);
  if (st != WAITS_OK) return st;
  const cudaError_t err = launch_select(
      scores, shape->cu_seqlens, shape->nseq, shape->total_tokens, shape->num_kv_heads, R, B,
      idx, kept_len, status_word(workspace, workspace_bytes), static_cast<cudaStream_t>(stream),
      static_cast<const uint16_t*>(K), static_cast<const uint16_t*>(V), shape->head_dim,
      static_cast<uint16_t*>(K_out), static_cast<uint16_t*>(V_out));
  if (err != cudaSuccess) return cuda_fail("select-compact launch", err);
  return WAITS_OK;
}

waits_status waits_compress_host(const waits_shape* shape, const int32_t* cu_host,
                                 const void* Q_host, const void* K_host, const void* V_host,
                                 float a, int32_t b, int32_t R, int32_t B, int32_t* idx_host,
                                 int32_t* kept_len_host, void* K_out_host, void* V_out_host,
                                 const waits_device_buffers* dev, void* workspace,
                                 size_t workspace_bytes, void* stream, size_t* h2d_bytes,
                                 size_t* d2h_bytes) {
  if (!shape || !cu_host || !dev || !Q_host || !K_host || !V_host || !idx_host ||
      !kept_len_host || !K_out_host || !V_out_host || !dev->cu_seqlens)
    return WAITS_ERR_ARG;
  waits_shape sh = *shape;
  sh.cu_seqlens = dev->cu_seqlens;
  waits_status st = check_shape(&sh);
  if (st != WAITS_OK) return st;
  // host copy of the offsets: validate before sending anything
  if (cu_host[0] != 0 || cu_host[sh.nseq] != sh.total_tokens) return WAITS_ERR_SHAPE;
  for (int i = 0; i < sh.nseq; ++i) {
    const int n = cu_host[i + 1] - cu_host[i];
    if (n < 0 || n > sh.max_seqlen) return WAITS_ERR_SHAPE;
  }
  st = check_score_args(&sh, dev->Q, dev->K, a, b, dev->scores);
  if (st == WAITS_OK) st = check_select_args(dev->scores, R, B, dev->idx, dev->kept_len);
  if (st == WAITS_OK)
    st = check_compact_args(dev->K, dev->V, dev->idx, dev->kept_len, B, dev->K_out, dev->V_out);
  if (st == WAITS_OK) st = check_ws(&sh, workspace, workspace_bytes);
  if (st != WAITS_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t qrow = (size_t)sh.num_q_heads * sh.head_dim * 2;
  const size_t krow = (size_t)sh.num_kv_heads * sh.head_dim * 2;
  size_t up = 0, down = 0;
  auto h2d = [&](void* dst, const void* src, size_t n) {
    up += n;
    return cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, s) == cudaSuccess;
  };
  auto d2h = [&](void* dst, const void* src, size_t n) {
    down += n;
    return cudaMemcpyAsync(dst, src, n, cudaMemcpyDeviceToHost, s) == cudaSuccess;
  };
  bool ok = h2d(dev->cu_seqlens, cu_host, sizeof(int32_t) * (sh.nseq + 1));
  // Query rows below this bound have -a*(q-c) > 88.73, so their fp32 weight
  // is exactly 0 and the scorer never reads them.
  for (int i = 0; i < sh.nseq && ok; ++i) {
    const int lo = cu_host[i], N = cu_host[i + 1] - lo;
    long long q_lo = 0;
    if (a > 0.0f) {
      const double c = (double)N - (double)b - 0.5;
      q_lo = (long long)std::floor(c - 90.0 / (double)a) - 2;
      if (q_lo < 0) q_lo = 0;
      if (q_lo > N) q_lo = N;
    }
    const size_t off = (size_t)(lo + q_lo) * qrow;
    if (N > q_lo) ok = h2d(static_cast<uint8_t*>(dev->Q) + off,
                           static_cast<const uint8_t*>(Q_host) + off, (size_t)(N - q_lo) * qrow);
  }
  ok = ok && h2d(dev->K, K_host, (size_t)sh.total_tokens * krow);
  // V: only the kept rows are ever read.  Page-locked host memory mapped
  // into the device's address space is read in place by the compaction
  // (min(B, N) rows per sequence and KV head cross the bus); anything else
  // is copied whole first.
  const void* V_src = dev->V;
  cudaPointerAttributes attr{};
  if (cudaPointerGetAttributes(&attr, V_host) == cudaSuccess &&
      attr.type == cudaMemoryTypeHost && attr.devicePointer != nullptr &&
      aligned(attr.devicePointer, 16)) {
    V_src = attr.devicePointer;
    for (int i = 0; i < sh.nseq; ++i) {
      const int N = cu_host[i + 1] - cu_host[i];
      up += (size_t)(N < B ? N : B) * krow;
    }
  } else {
    cudaGetLastError();   // an unregistered pointer is not an error here
    ok = ok && h2d(dev->V, V_host, (size_t)sh.total_tokens * krow);
  }
  if (!ok) return WAITS_ERR_CUDA;
  st = waits_compress(&sh, dev->Q, dev->K, V_src, a, b, R, B, dev->scores, dev->idx,
                      dev->kept_len, dev->K_out, dev->V_out, workspace, workspace_bytes, stream);
  if (st != WAITS_OK) return st;
  const size_t nidx = (size_t)sh.nseq * sh.num_kv_heads * B;
  const size_t nout = nidx * sh.head_dim * 2;
  ok = d2h(idx_host, dev->idx, nidx * sizeof(int32_t)) &&
       d2h(kept_len_host, dev->kept_len, sh.nseq * sizeof(int32_t)) &&
       d2h(K_out_host, dev->K_out, nout) && d2h(V_out_host, dev->V_out, nout);
  if (!ok) return WAITS_ERR_CUDA;
  if (h2d_bytes) *h2d_bytes = up;
  if (d2h_bytes) *d2h_bytes = down;
  return WAITS_OK;
}

waits_status decode_dims_ok(int32_t nseq, int32_t Hq, int32_t Hkv, int32_t d, int32_t C) {
  if (nseq < 1 || Hq < 1 || Hkv < 1 || C < 1 || Hq % Hkv) return WAITS_ERR_SHAPE;
  if (d != 64 && d != 128) return WAITS_ERR_UNSUPPORTED;
  if (Hq / Hkv > decode_max_group()) return WAITS_ERR_UNSUPPORTED;
  if ((int64_t)nseq * Hkv > 65535LL * 65535LL || Hq > 65535 || nseq > 65535)
    return WAITS_ERR_SHAPE;
  return WAITS_OK;
}

waits_status waits_decode_workspace_size(int32_t nseq, int32_t num_q_heads, int32_t head_dim,
                                         int32_t capacity, size_t* bytes) {
  if (!bytes) return WAITS_ERR_ARG;
  if (nseq < 1 || num_q_heads < 1 || capacity < 1) return WAITS_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128) return WAITS_ERR_UNSUPPORTED;
  *bytes = decode_workspace_bytes(nseq, num_q_heads, head_dim, capacity);
  return WAITS_OK;
}

waits_status waits_decode_attention(int32_t nseq, int32_t num_q_heads, int32_t num_kv_heads,
                                    int32_t head_dim, int32_t capacity, const void* q,
                                    const void* K_cache, const void* V_cache,
                                    const int32_t* cache_len, float* out, float* lse,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  waits_status st = decode_dims_ok(nseq, num_q_heads, num_kv_heads, head_dim, capacity);
  if (st != WAITS_OK) return st;
  if (!q || !K_cache || !V_cache || !cache_len || !out) return WAITS_ERR_ARG;
  if (!aligned(q, 16) || !aligned(K_cache, 16) || !aligned(V_cache, 16) || !aligned(out, 4) ||
      !aligned(cache_len, 4) || (lse && !aligned(lse, 4)))
    return WAITS_ERR_ARG;
  if (!workspace || !aligned(workspace, 16) ||
      workspace_bytes < decode_workspace_bytes(nseq, num_q_heads, head_dim, capacity))
    return WAITS_ERR_WORKSPACE;
  const cudaError_t err = launch_decode(
      nseq, num_q_heads, num_kv_heads, head_dim, capacity, static_cast<const uint16_t*>(q),
      static_cast<const uint16_t*>(K_cache), static_cast<const uint16_t*>(V_cache), cache_len,
      out, lse, static_cast<float*>(workspace), static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail("decode launch", err);
  return WAITS_OK;
}

waits_status waits_test_exp2_poly(const float* x, float* y, int64_t n, void* stream) {
  if (!x || !y || n < 0) return WAITS_ERR_ARG;
  if (n == 0) return WAITS_OK;
  const cudaError_t err = launch_exp2_poly(x, y, n, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail("exp2 test launch", err);
  return WAITS_OK;
}

waits_status waits_read_device_status(const void* workspace, size_t workspace_bytes,
                                      void* stream, uint32_t* status_bits) {
  if (!status_bits) return WAITS_ERR_ARG;
  if (!workspace || workspace_bytes < sizeof(PlanHeader)) return WAITS_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return WAITS_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, &reinterpret_cast<const PlanHeader*>(workspace)->status,
                      sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return WAITS_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return WAITS_ERR_CUDA;
  *status_bits = v;
  return WAITS_OK;
}

}  // extern "C"
