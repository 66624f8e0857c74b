// Per (sequence, KV head) selection (WAITS README, Quickstart budgets): keep
// the recent window [N-R, N) and the B-R highest scores of [0, N-R), ties to
// the lower index, reported in ascending order.
//
// One CTA per (sequence, KV head).  The (B-R)-th largest score is found by an
// exact 4-round radix select on the fp32 bit pattern (non-negative floats
// order like their bits); the kept set is then written in index order with
// block prefix sums, taking threshold ties lowest index first.
#include "waits_internal.cuh"

namespace waits {
namespace {

constexpr int kSelThreads = 1024;

__device__ inline uint32_t order_key(float s) {
  const uint32_t u = __float_as_uint(s);
  return u == 0x80000000u ? 0u : u;   // -0 ranks with +0
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(
    const float* __restrict__ scores, const int32_t* __restrict__ cu, int nseq, int T,
    int Hkv, int R, int B, int32_t* __restrict__ idx, int32_t* __restrict__ kept_len,
    uint32_t* status) {
  __shared__ uint32_t hist[256];
  __shared__ int64_t sh[32];
  __shared__ uint32_t s_digit;
  __shared__ int s_above;
  const int tid = threadIdx.x;
  const int s = blockIdx.x / Hkv, g = blockIdx.x % Hkv;
  const int lo = cu[s], hi = cu[s + 1];
  int32_t* out = idx + ((size_t)s * Hkv + g) * B;
  const bool bad = (s == 0 && lo != 0) || hi < lo || hi > T || (s == nseq - 1 && hi != T);
  if (bad) {
    for (int j = tid; j < B; j += blockDim.x) out[j] = -1;
    if (tid == 0) {
      if (g == 0) kept_len[s] = 0;
      if (status) atomicOr(status, WAITS_DEV_BAD_SEQLENS);
    }
    return;
  }
  const int N = hi - lo;
  if (g == 0 && tid == 0) kept_len[s] = N < B ? N : B;
  if (N <= B) {
    for (int j = tid; j < B; j += blockDim.x) out[j] = j < N ? j : -1;
    return;
  }
  const int want = B - R;          // positions taken from the pool by score
  const int pool = N - R;
  const float* sc = scores + (size_t)g * T + lo;
  const int lane = tid & 31, warp = tid >> 5;

  uint32_t prefix = 0, pmask = 0;
  int need = want;
  if (want > 0) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
      __syncthreads();
      for (int k = tid; k < pool; k += blockDim.x) {
        const uint32_t u = order_key(sc[k]);
        const bool match = (u & pmask) == prefix;
        const uint32_t dg = (u >> shift) & 255u;
        const unsigned m = __ballot_sync(__activemask(), match);
        if (match) {
          const unsigned peers = __match_any_sync(m, dg);
          if (lane == __ffs(peers) - 1) atomicAdd(&hist[dg], (uint32_t)__popc(peers));
        }
      }
      __syncthreads();
      if (warp == 0) {
        // lane L owns bins 255-8L ... 248-8L (descending)
        uint32_t c[8];
        uint32_t tot = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { c[i] = hist[255 - 8 * lane - i]; tot += c[i]; }
        uint32_t incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const uint32_t excl = incl - tot;
        if ((int)excl < need && (int)incl >= need) {
          uint32_t cum = excl;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if ((int)(cum + c[i]) >= need) { s_digit = 255 - 8 * lane - i; s_above = (int)cum; break; }
            cum += c[i];
          }
        }
      }
      __syncthreads();
      prefix |= s_digit << shift;
      pmask |= 255u << shift;
      need -= s_above;
      __syncthreads();
    }
  }
  const uint32_t tau = prefix;

  // ascending output: thread tid owns positions [c0, c1)
  const int per = (N + blockDim.x - 1) / blockDim.x;
  const int c0 = min(N, tid * per), c1 = min(N, c0 + per);
  int n_gt = 0, n_eq = 0;
  if (want > 0) {
    for (int k = c0; k < min(c1, pool); ++k) {
      const uint32_t u = order_key(sc[k]);
      n_gt += u > tau;
      n_eq += u == tau;
    }
  }
  int64_t tot;
  const int eq_before = (int)block_exclusive_scan(n_eq, &tot, sh);
  const int take_eq = max(0, min(n_eq, need - eq_before));
  const int n_rec = max(0, c1 - max(c0, pool));
  int pos = (int)block_exclusive_scan(n_gt + take_eq + n_rec, &tot, sh);
  int eq_seen = 0;
  for (int k = c0; k < c1; ++k) {
    bool keep = k >= pool;
    if (!keep && want > 0) {
      const uint32_t u = order_key(sc[k]);
      if (u > tau) keep = true;
      else if (u == tau) { keep = eq_seen < take_eq; ++eq_seen; }
    }
    if (keep && pos < B) out[pos++] = k;
  }
}

}  // namespace

cudaError_t launch_select(const float* scores, const int32_t* cu, int nseq, int T, int Hkv,
                          int R, int B, int32_t* idx, int32_t* kept_len, uint32_t* status,
                          cudaStream_t s) {
  select_kernel<<<nseq * Hkv, kSelThreads, 0, s>>>(scores, cu, nseq, T, Hkv, R, B, idx,
                                                   kept_len, status);
  return cudaGetLastError();
}

}  // namespace waits
