// Internal definitions shared by the libwaits translation units: the
// workspace layout, the work plan written by the planner kernel, the fp32
// forgetting-curve weight, and small block-level helpers.
#pragma once

#include <cmath>
#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda_runtime.h>

#include "waits.h"

namespace waits {

// ---------------------------------------------------------------- tiling ---
constexpr int kTile = 128;      // keys per K tile; max packed rows per Q tile
constexpr int kMaxStat = 4;     // stationary tiles held by one work unit (at most)
constexpr int kMaxStat1 = 2;    // pass 1: Q tiles per unit (leaves room for 4 K stages)
constexpr int kMaxGrid = 1024;  // upper bound on persistent CTAs (sizing)
constexpr int kPlanThreads = 256;

// A Q tile packs `tokq` consecutive query positions x G heads of one KV
// group: packed row r <-> position q0 + j*tokq + r / G, head g*G + r % G.
__host__ __device__ inline int tokens_per_qtile(int G) { return kTile / G; }

// ----------------------------------------------------------- plan types ---
enum EntryMode : int32_t {
  kModeP1 = 0,   // pass 1: stationary Q tiles, streamed K tiles
  kModeP2Q = 1,  // pass 2: stationary Q tiles (all active rows), streamed K
  kModeP2K = 2,  // pass 2: stationary K tiles, streamed Q tiles
};

struct SeqInfo {
  int32_t start;   // cu_seqlens[s]
  int32_t len;     // N
  int32_t q0;      // first row with non-zero fp32 weight (len if none)
  int32_t nqt;     // Q tiles covering rows [q0, N)
  int32_t nkt;     // K tiles covering keys [0, N)
  int32_t e1;      // first pass-1 entry of this sequence
  int32_t e2;      // first pass-2 entry of this sequence
  int32_t b;       // this sequence's forgetting-curve window and slope
  float a;
  int32_t pad[3];  // 48 bytes: arrays of entries after it stay 16-byte aligned
};

// An entry is one (sequence, KV head, stationary group) with a contiguous
// range of streamed tiles ("steps").  Steps are split over CTAs by global
// step index; the CTAs covering an entry are consecutive.
struct Entry {
  int32_t seq, g, grp, mode;
  int32_t stat0;     // first stationary tile index (Q tile or K tile)
  int32_t n_stat;    // stationary tiles in the group (1..4)
  int32_t step0;     // first streamed tile index
  int32_t n_steps;   // streamed tiles
  int64_t sbase;     // global index of this entry's first step
  int32_t unit_base; // partial-result slot of this entry's first unit
  int32_t n_units;   // CTAs (units) covering the entry
  int32_t first_cta;
  int32_t n_masked;  // trailing steps that reach the causal diagonal (slower)
  int32_t pad[2];
};

// Cost of a step on the causal diagonal (masked exp path) in units of an
// unmasked step, for splitting an entry's steps evenly by time.
constexpr int kMaskedCost = 3;   // measured: 2 and 3 alike, 1% better than 1

struct PlanHeader {
  uint32_t status;     // WAITS_DEV_* bits, cleared by the planner
  int32_t n_e1, n_e2;  // entries per pass
  int32_t n_u1, n_u2;  // units per pass
  int32_t p1, p2;      // CTAs that own work per pass (<= grid)
  int32_t pad0;
  int64_t s1, s2;      // total steps per pass
  int32_t aligned1, aligned2;  // per pass: CTAs split entry by entry (1) or by global step (0)
  int32_t pad[2];
};

// ------------------------------------------------------ workspace layout ---
struct Layout {
  size_t header, seqs, e1, e2, c2, part1, part2, total;
  int64_t max_e1, max_e2, max_u1, max_u2;
};

__host__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Upper bounds that hold for every a, b (a = 0 activates every row).
__host__ inline Layout make_layout(int64_t nseq, int64_t T, int64_t Hq, int64_t Hkv) {
  Layout L{};
  const int64_t G = Hq / Hkv;
  const int64_t tokq = tokens_per_qtile((int)G);
  L.max_e1 = Hkv * (T / (kMaxStat1 * tokq) + nseq);
  L.max_e2 = Hkv * (T / (kMaxStat * kTile) + nseq);
  L.max_u1 = L.max_e1 + kMaxGrid;
  L.max_u2 = L.max_e2 + kMaxGrid;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
  L.header = take(sizeof(PlanHeader));
  L.seqs = take(sizeof(SeqInfo) * (size_t)nseq);
  L.e1 = take(sizeof(Entry) * (size_t)L.max_e1);
  L.e2 = take(sizeof(Entry) * (size_t)L.max_e2);
  L.c2 = take(sizeof(uint32_t) * (size_t)L.max_e2);
  L.part1 = take(sizeof(float2) * (size_t)L.max_u1 * kMaxStat1 * kTile);
  L.part2 = take(sizeof(float) * (size_t)L.max_u2 * kMaxStat * kTile);
  L.total = off;
  return L;
}

// ---------------------------------------------------------- L2 policies ---
// Policy under which lines are the first to be evicted from L2: for data
// that streams through once (or twice) per call, so that it does not push
// out what every call reuses.
__device__ inline uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 16-byte load through the coherent path (plain ld.global, no read-only
// cache): valid for device memory and for mapped page-locked host memory.
__device__ inline uint4 ld_global_v4(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ------------------------------------------------------------ the curve ---
// fp32 forgetting-curve weight (WAITS README, opening summary):
// w = 1 / (1 + exp(-a (q - (N - b - 0.5)))), IEEE division, no flush to zero.
__device__ inline float curve_weight(int q, int N, float a, int b) {
  const float c = (float)N - (float)b - 0.5f;
  const float t = -a * ((float)q - c);
  return 1.0f / (1.0f + expf(t));
}

// First row whose fp32 weight is non-zero (N if none).  For a > 0 the weight
// is non-decreasing in q and vanishes once -a (q - c) passes ~88.7 (expf
// overflows), so the search starts from that estimate and walks to the
// exact boundary, falling back to bisection if the walk is long; a = 0
// weights every row by 1/2.
__host__ __device__ inline int first_active_row(int N, float a, int b) {
  if (N <= 0) return 0;
  if (a == 0.0f) return 0;
  const float c = (float)N - (float)b - 0.5f;
  // curve_weight(q) != 0 exactly when expf(t) is finite: 1 + expf(t) is then
  // at most FLT_MAX and its IEEE reciprocal at least 2.9e-39 (no flush to
  // zero); this test skips the division
  auto active = [&](int q) { return expf(-a * ((float)q - c)) != INFINITY; };
  if (!active(N - 1)) return N;
  float est = ceilf(c - 88.72284f / a);
  int q = est < 0.f ? 0 : (est > (float)(N - 1) ? N - 1 : (int)est);
  for (int step = 0; step < 8; ++step) {
    const bool on = active(q);
    if (on && (q == 0 || !active(q - 1))) return q;
    q += on ? -1 : 1;
    if (q < 0 || q > N - 1) break;
  }
  int lo = 0, hi = N - 1;
  while (lo < hi) {
    const int mid = lo + (hi - lo) / 2;
    if (active(mid)) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// --------------------------------------------------------- block scans ---
// Exclusive prefix sum over the threads of a block (a multiple of 32, <= 1024).
// A one-warp block scans with shuffles alone, without barriers.
__device__ inline int64_t block_exclusive_scan(int64_t v, int64_t* total, int64_t* sh /*[32]*/) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (blockDim.x == 32) {
    int64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    *total = __shfl_sync(0xffffffffu, x, 31);
    return x - v;
  }
  int64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int64_t s = lane < nw ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int64_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    sh[lane] = s;  // inclusive warp totals
  }
  __syncthreads();
  const int64_t before = (warp ? sh[warp - 1] : 0) + x - v;
  *total = sh[(blockDim.x >> 5) - 1];
  __syncthreads();
  return before;
}

// -------------------------------------------------------- kernel params ---
struct PlanArgs {
  const int32_t* cu;
  int nseq, T, max_seqlen, Hq, Hkv, G, tokq;
  float a;
  int b;
  // per-sequence curve parameters (DEVICE [nseq]; routed calls), else null
  const float* seq_a;
  const int32_t* seq_b;
  int grid;
  PlanHeader* hdr;
  SeqInfo* seqs;
  Entry* e1;
  Entry* e2;
  uint32_t* c2;        // pass-2 unit counters (last-arriver merges), zeroed
  int64_t max_e1, max_e2, max_u1, max_u2;
  float* scores;  // zero-filled for sequences without active rows
};

struct PassArgs {
  const uint16_t* Q;   // bf16 bits [T, Hq, d] (rows of q_row_heads heads)
  const uint16_t* K;   // bf16 bits [T, Hkv, d] (rows of kv_row_heads heads)
  int T, Hq, Hkv, G, tokq, d;
  int q_row_heads, kv_row_heads;   // heads per token row in memory (>= Hq, Hkv)
  float a;
  int b;
  float scale2;        // log2(e) / sqrt(d)
  const PlanHeader* hdr;
  const SeqInfo* seqs;
  const Entry* e1;
  const Entry* e2;
  uint32_t* c2;
  float2* part1;       // [units, 2, 128] (reference max, sum) in log2 units
  float* part2;        // [units, 4, 128] partial column sums
  float* scores;       // [Hkv, T]
  uint32_t* status;
  // local plan: every CTA rebuilds the (small) plan in shared memory from
  // cu_seqlens, and no planner kernel runs; with host_plan it copies the
  // plan the host built (one sequence) and only checks cu_seqlens
  int local_plan;
  int host_plan;
  const int32_t* cu;
  int nseq, max_seqlen;
  // natural-log row LSE [Hq, T] given by the caller (waits_score_with_lse):
  // pass 1 is not run and pass 2 takes its row biases from it; else null
  const float* lse;
  // 1: every pass-1 entry's merged row biases sit in the first unit's
  // partial slots (bias in .x; row_bias_kernel ran after pass 1)
  int bias_ready;
  // limit of every bounded wait in the main loops (ns); testing aid: with
  // withhold_mma the MMA warp issues nothing, so those waits run out
  uint64_t wait_ns;
  int withhold_mma;
};

// ------------------------------------------- programmatic dependent launch ---
// Every kernel of the path is launched with programmatic stream
// serialisation: it may start while the previous kernel on the stream is
// still running, does only its private set-up (shared memory, barriers,
// tensor memory), then waits for the previous grid to complete and its
// memory to be visible before it touches global memory.  It lets the next
// kernel start launching at once; that kernel waits the same way.
__device__ inline void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ inline void pdl_allow_next() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Same, launched as thread-block clusters of `cluster` CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, int cluster,
                               size_t smem, cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Extra text appended to the next waits_last_error() message (host only).
void set_error_detail(const char* fmt, ...);

// Host-side launchers (one per translation unit).
cudaError_t launch_plan(const PlanArgs& a, cudaStream_t s);
struct HostPlan;
// hp: the host-built plan when a.host_plan (else unused, may be null).
cudaError_t launch_score_passes(const PassArgs& a, const HostPlan* hp, int grid, cudaStream_t s);
// The same two passes for a local plan (every entry of pass 2 in mode P2Q):
// 256-column accumulators, bit-identical scores.
cudaError_t launch_sparse_passes(const PassArgs& a, const HostPlan* hp, int grid, cudaStream_t s);
// Large plans (the planner kernel's, in the workspace): pass 1 by the
// 256-column kernel (bit-identical row partials), pass 2 by score_tc.cu's.
cudaError_t launch_sparse_pass1(const PassArgs& a, int grid, cudaStream_t s);
cudaError_t launch_score_pass2(const PassArgs& a, int grid, cudaStream_t s);
// Between the passes of a planner-kernel plan: every row's bias, merged
// once from its pass-1 partials (max_e1 bounds the plan's pass-1 entries).
cudaError_t launch_row_bias(const PassArgs& a, int64_t max_e1, cudaStream_t s);
cudaError_t launch_exp2_poly(const float* x, float* y, int64_t n, cudaStream_t s);
// K == nullptr: selection only; else also the compaction of K and V into
// Ko, Vo (the rows of the kept positions, zeros past kept_len).
cudaError_t launch_select(const float* scores, const int32_t* cu, int nseq, int T,
                          int Hkv, int R, int B, int32_t* idx, int32_t* kept_len,
                          uint32_t* status, cudaStream_t s, const uint16_t* K = nullptr,
                          const uint16_t* V = nullptr, int d = 0, uint16_t* Ko = nullptr,
                          uint16_t* Vo = nullptr, int kv_row_heads = 0);
cudaError_t launch_compact(const uint16_t* K, const uint16_t* V, const int32_t* cu,
                           const int32_t* idx, const int32_t* kept_len, int nseq,
                           int Hkv, int d, int B, uint16_t* Ko, uint16_t* Vo,
                           uint32_t* status, cudaStream_t s, int kv_row_heads = 0);
// Decode attention over the compacted cache (decode.cu).
size_t decode_workspace_bytes(int64_t nseq, int64_t Hq, int64_t d, int64_t C);
int decode_max_group();
cudaError_t launch_decode(int nseq, int Hq, int Hkv, int d, int C, const uint16_t* q,
                          const uint16_t* Kc, const uint16_t* Vc, const int32_t* len, float* out,
                          float* lse, float* part, cudaStream_t st);

}  // namespace waits
