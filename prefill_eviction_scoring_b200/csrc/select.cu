// Per (sequence, KV head) selection (WAITS README, Quickstart budgets): keep
// the recent window [N-R, N) and the B-R highest scores of [0, N-R), ties to
// the lower index, reported in ascending order.
//
// One thread-block cluster of kCta CTAs per (sequence, KV head); CTA r owns
// a contiguous slice of the pool [0, N-R), staged in its shared memory.  The
// (B-R)-th largest key tau is found exactly by a radix select over three
// digits (11 + 11 + 10 bits of a monotone 32-bit image of the fp32 score):
// each CTA histograms its slice, each CTA then sums one slice of the bins
// over the cluster through distributed shared memory, and every CTA reads the
// merged counts to pick the same digit.  The kept positions are written in
// index order: per-thread counts, block scans, and a scan over the cluster's
// CTAs (again through distributed shared memory); threshold ties are taken
// lowest index first.
#include <cooperative_groups.h>

#include "waits_internal.cuh"

namespace cg = cooperative_groups;

namespace waits {
namespace {

constexpr int kCta = 8;               // CTAs per cluster (portable cluster size)
constexpr int kSelThreads = 512;
constexpr int kMaxBins = 2048;        // 11-bit digits
constexpr int kStage = 16384;         // keys staged per CTA (64 KB): pools up to 131072
// digit d covers bits [shift(d), shift(d) + bits(d)) of the key
__device__ constexpr int digit_shift(int d) { return d == 0 ? 21 : (d == 1 ? 10 : 0); }
__device__ constexpr int digit_bits(int d) { return d == 2 ? 10 : 11; }

// Monotone map of fp32 to uint32: a < b (as floats, -0 == +0) iff
// key(a) < key(b).  Scores from waits_score are >= 0, but waits_select takes
// any finite fp32 input.
__device__ inline uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;                       // -0 ranks with +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Histogram add from every active lane: lanes holding the same bin are
// merged first, so a warp issues one shared-memory atomic per distinct bin
// (scores cluster in a few bins; unmerged atomics would serialise).
__device__ inline void hist_add(uint32_t* hist, uint32_t bin) {
  const unsigned peers = __match_any_sync(__activemask(), bin);
  if ((threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

struct SelSmem {
  uint32_t hist[kMaxBins];        // this CTA's histogram of the current digit
  uint32_t merged[kMaxBins / kCta];  // cluster sums of this CTA's slice of bins
  uint32_t slice_total;           // sum of merged[]
  uint32_t n_gt, n_eq;            // this CTA's keys above / equal to tau
  uint32_t digit;
  int32_t above;
  int64_t scan[32];
};

// Warp 0: pick the digit whose bin holds the need-th largest key, given the
// merged histogram spread over the cluster (CTA c holds bins
// [c*per, (c+1)*per) of nb).  Every CTA computes the same answer.
__device__ void find_digit(cg::cluster_group& cl, SelSmem& sm, int nb, int need) {
  const int lane = threadIdx.x & 31;
  if (threadIdx.x >= 32) return;
  const int per = nb / kCta;
  // slice totals, highest bins (last CTA) first
  uint32_t v = 0;
  if (lane < kCta) v = *cl.map_shared_rank(&sm.slice_total, kCta - 1 - lane);
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t excl = incl - v;
  const unsigned hit = __ballot_sync(0xffffffffu, lane < kCta && (int)excl < need &&
                                                      (int)incl >= need);
  const int l0 = __ffs(hit) - 1;                       // exactly one lane
  const int slice = kCta - 1 - l0;
  const int above0 = (int)__shfl_sync(0xffffffffu, excl, l0);
  const uint32_t* bins = cl.map_shared_rank(sm.merged, slice);
  // descending bins of that slice: lane l owns positions [l*k, l*k + k)
  const int k = per / 32;
  uint32_t tot = 0;
  for (int i = 0; i < k; ++i) tot += bins[per - 1 - (lane * k + i)];
  uint32_t inc2 = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc2, o);
    if (lane >= o) inc2 += y;
  }
  const int rem = need - above0;
  const uint32_t ex2 = inc2 - tot;
  if ((int)ex2 < rem && (int)inc2 >= rem) {
    uint32_t cum = ex2;
    for (int i = 0; i < k; ++i) {
      const int pos = per - 1 - (lane * k + i);
      const uint32_t c = bins[pos];
      if ((int)(cum + c) >= rem) {
        sm.digit = (uint32_t)(slice * per + pos);
        sm.above = above0 + (int)cum;
        break;
      }
      cum += c;
    }
  }
}

__global__ void __cluster_dims__(kCta, 1, 1) __launch_bounds__(kSelThreads) select_kernel(
    const float* __restrict__ scores, const int32_t* __restrict__ cu, int nseq, int T,
    int Hkv, int R, int B, int32_t* __restrict__ idx, int32_t* __restrict__ kept_len,
    uint32_t* status) {
  extern __shared__ uint32_t stage[];       // [kStage] keys of this CTA's slice
  __shared__ SelSmem sm;
  cg::cluster_group cl = cg::this_cluster();
  const int tid = threadIdx.x;
  pdl_allow_next();
  pdl_wait();
  const int r = (int)cl.block_rank();
  const int sg = blockIdx.x / kCta;
  const int s = sg / Hkv, g = sg % Hkv;
  const int lo = cu[s], hi = cu[s + 1];
  int32_t* out = idx + ((size_t)s * Hkv + g) * B;
  // Every branch below depends only on (s, g), so all CTAs of a cluster take
  // it together and the cluster barriers match.
  const bool bad = (s == 0 && lo != 0) || hi < lo || hi > T || (s == nseq - 1 && hi != T);
  if (bad) {
    for (int j = r * kSelThreads + tid; j < B; j += kCta * kSelThreads) out[j] = -1;
    if (r == 0 && tid == 0) {
      if (g == 0) kept_len[s] = 0;
      if (status) atomicOr(status, WAITS_DEV_BAD_SEQLENS);
    }
    return;
  }
  const int N = hi - lo;
  if (r == 0 && g == 0 && tid == 0) kept_len[s] = N < B ? N : B;
  if (N <= B) {
    for (int j = r * kSelThreads + tid; j < B; j += kCta * kSelThreads) out[j] = j < N ? j : -1;
    return;
  }
  const int want = B - R;            // positions taken from the pool by score
  const int pool = N - R;            // > want because N > B
  // recent window: always kept, after the want pool positions
  for (int j = r * kSelThreads + tid; j < R; j += kCta * kSelThreads) out[want + j] = pool + j;
  if (want == 0) return;

  const float* sc = scores + (size_t)g * T + lo;
  const int per = (pool + kCta - 1) / kCta;
  const int a0 = min(pool, r * per);
  const int n = min(pool, a0 + per) - a0;
  const bool staged = per <= kStage;     // uniform over the cluster
  if (staged)
    for (int i = tid; i < n; i += kSelThreads) stage[i] = order_key(__ldg(sc + a0 + i));
  auto key = [&](int i) -> uint32_t {
    return staged ? stage[i] : order_key(__ldg(sc + a0 + i));
  };

  // ---- radix select of the want-th largest key
  uint32_t prefix = 0, pmask = 0;
  int need = want;
#pragma unroll 1
  for (int d = 0; d < 3; ++d) {
    const int nb = 1 << digit_bits(d), shift = digit_shift(d);
    for (int i = tid; i < nb; i += kSelThreads) sm.hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kSelThreads) {
      const uint32_t u = key(i);
      if ((u & pmask) == prefix) hist_add(sm.hist, (u >> shift) & (uint32_t)(nb - 1));
    }
    cl.sync();   // every CTA's histogram is complete
    const int pb = nb / kCta;
    uint32_t part = 0;
    for (int b = tid; b < pb; b += kSelThreads) {
      uint32_t sum = 0;
#pragma unroll
      for (int c = 0; c < kCta; ++c) sum += cl.map_shared_rank(sm.hist, c)[r * pb + b];
      sm.merged[b] = sum;
      part += sum;
    }
    int64_t tot;
    block_exclusive_scan((int64_t)part, &tot, sm.scan);
    if (tid == 0) sm.slice_total = (uint32_t)tot;
    cl.sync();   // merged slices and their totals are visible
    find_digit(cl, sm, nb, need);
    __syncthreads();
    prefix |= sm.digit << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    need -= sm.above;
  }
  const uint32_t tau = prefix;    // need = ties of tau to keep, lowest index first

  // ---- ascending output: thread tid owns positions [c0, c1) of the slice
  const int pt = (n + kSelThreads - 1) / kSelThreads;
  const int c0 = min(n, tid * pt), c1 = min(n, c0 + pt);
  int gt = 0, eq = 0;
  for (int i = c0; i < c1; ++i) {
    const uint32_t u = key(i);
    gt += u > tau;
    eq += u == tau;
  }
  int64_t t_gt, t_eq;
  const int gt_before = (int)block_exclusive_scan(gt, &t_gt, sm.scan);
  const int eq_before = (int)block_exclusive_scan(eq, &t_eq, sm.scan);
  if (tid == 0) {
    sm.n_gt = (uint32_t)t_gt;
    sm.n_eq = (uint32_t)t_eq;
  }
  cl.sync();   // per-CTA counts visible
  __shared__ int s_cta_gt, s_cta_eq;
  if (tid < 32) {
    uint32_t vg = 0, ve = 0;
    if (tid < r) {
      vg = *cl.map_shared_rank(&sm.n_gt, tid);
      ve = *cl.map_shared_rank(&sm.n_eq, tid);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      vg += __shfl_down_sync(0xffffffffu, vg, o);
      ve += __shfl_down_sync(0xffffffffu, ve, o);
    }
    if (tid == 0) {
      s_cta_gt = (int)vg;
      s_cta_eq = (int)ve;
    }
  }
  __syncthreads();
  const int eq_prev = s_cta_eq + eq_before;            // tau keys before this thread
  const int take_eq = max(0, min(eq, need - eq_prev));
  int pos = s_cta_gt + gt_before + min(need, eq_prev);
  int taken = 0;
  for (int i = c0; i < c1; ++i) {
    const uint32_t u = key(i);
    bool keep = u > tau;
    if (u == tau) {
      keep = taken < take_eq;
      ++taken;
    }
    if (keep && pos < want) out[pos++] = a0 + i;
  }
  cl.sync();   // no CTA leaves while another may still read its shared memory
}

}  // namespace

cudaError_t launch_select(const float* scores, const int32_t* cu, int nseq, int T, int Hkv,
                          int R, int B, int32_t* idx, int32_t* kept_len, uint32_t* status,
                          cudaStream_t s) {
  const int dyn = kStage * (int)sizeof(uint32_t);
  cudaError_t err = cudaFuncSetAttribute(select_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
  if (err != cudaSuccess) return err;
  const int64_t grid = (int64_t)nseq * Hkv * kCta;
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  return launch_pdl(select_kernel, dim3((unsigned)grid), dim3(kSelThreads), (size_t)dyn, s,
                    scores, cu, nseq, T, Hkv, R, B, idx, kept_len, status);
}

}  // namespace waits
