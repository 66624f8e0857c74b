// Per (sequence, KV head) selection (WAITS README, Quickstart budgets): keep
// the recent window [N-R, N) and the B-R highest scores of [0, N-R), ties to
// the lower index, reported in ascending order.
//
// One CTA per (sequence, KV head).  Scores are non-negative, so their fp32
// bit patterns order like the values.  The (B-R)-th largest pattern tau is
// found exactly by a radix select over 12 + 10 + 10 bits; after the first
// digit only the candidates that still match the prefix are kept (compacted
// in shared memory), so later rounds touch few elements.  The kept set is
// then written in index order with block prefix sums, taking threshold ties
// lowest index first.  The pool is staged in shared memory when it fits.
#include "waits_internal.cuh"

namespace waits {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kBins1 = 4096;          // first digit: bits 20..31
constexpr int kBins2 = 1024;          // then bits 10..19 and 0..9
constexpr int kCand = 4096;           // candidate list capacity (smem)
constexpr int kCache = 45056;         // pool entries staged in smem (~176 KB)
// Staged key k lives at k + k/32: one pad word per 32 keeps both the
// strided visits and the per-thread contiguous output scan conflict-free.
__device__ inline int cpos(int k) { return k + (k >> 5); }
constexpr int kCacheWords = kCache + kCache / 32;
constexpr int kBatch = 8;             // loads in flight per thread when streaming

__device__ inline uint32_t order_key(float s) {
  const uint32_t u = __float_as_uint(s);
  return u == 0x80000000u ? 0u : u;   // -0 ranks with +0
}

// Histogram add from every active lane: lanes holding the same bin are
// merged first, so a warp issues one shared-memory atomic per distinct bin
// (scores cluster in a few bins; unmerged atomics would serialise).
__device__ inline void hist_add(uint32_t* hist, uint32_t bin) {
  const unsigned peers = __match_any_sync(__activemask(), bin);
  if ((threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

// Append k to the candidate list with one atomic per warp.
__device__ inline void cand_push(int* cand, int* count, bool take, int k) {
  const unsigned act = __activemask();
  const unsigned m = __ballot_sync(act, take);
  if (!m) return;
  const int lane = threadIdx.x & 31;
  const int leader = __ffs(m) - 1;
  int base = 0;
  if (lane == leader) base = atomicAdd(count, __popc(m));
  base = __shfl_sync(act, base, leader);
  if (take) {
    const int slot = base + __popc(m & ((1u << lane) - 1u));
    if (slot < kCand) cand[slot] = k;
  }
}

// Warp 0 scans `hist[0..nb)` from the top bin down and finds the digit whose
// bin holds the need-th largest element; returns it (and the count above it)
// through shared memory.
__device__ void find_digit(const uint32_t* hist, int nb, int need, uint32_t* s_digit,
                           int* s_above) {
  const int lane = threadIdx.x & 31;
  if (threadIdx.x >= 32) return;
  const int per = nb / 32;                 // bins per lane, descending
  const int top = nb - 1 - lane * per;
  uint32_t tot = 0;
  for (int i = 0; i < per; ++i) tot += hist[top - i];
  uint32_t incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t excl = incl - tot;
  if ((int)excl < need && (int)incl >= need) {
    uint32_t cum = excl;
    for (int i = 0; i < per; ++i) {
      const uint32_t c = hist[top - i];
      if ((int)(cum + c) >= need) { *s_digit = (uint32_t)(top - i); *s_above = (int)cum; break; }
      cum += c;
    }
  }
}

// ------------------------------------------------------------ fast path ---
// Pools of up to kSelThreads * kPer keys: every thread holds a contiguous run
// of kPer keys in registers.  A sorted sample of one key per thread brackets
// the (want)-th largest key; one pass counts the keys above the bracket and
// collects those inside it (value, index); a bitonic sort of the collected
// keys (value descending, index ascending) gives the exact threshold and how
// many of its ties are taken.  Returns false (nothing written) when the
// bracket misses or overflows, and the caller runs the radix path.
constexpr int kPer = 32;
constexpr int kFastCand = 2048;

__device__ inline void bitonic_desc_u32(uint32_t* a, int n) {
  for (int k = 2; k <= n; k <<= 1)
    for (int j = k >> 1; j > 0; j >>= 1) {
      __syncthreads();
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int ij = i ^ j;
        if (ij > i) {
          const uint32_t x = a[i], y = a[ij];
          if (((i & k) == 0) == (x < y)) { a[i] = y; a[ij] = x; }
        }
      }
    }
  __syncthreads();
}

__device__ inline void bitonic_desc_u64(uint64_t* a, int n) {
  for (int k = 2; k <= n; k <<= 1)
    for (int j = k >> 1; j > 0; j >>= 1) {
      __syncthreads();
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int ij = i ^ j;
        if (ij > i) {
          const uint64_t x = a[i], y = a[ij];
          if (((i & k) == 0) == (x < y)) { a[i] = y; a[ij] = x; }
        }
      }
    }
  __syncthreads();
}

__device__ bool select_fast(const float* __restrict__ sc, int pool, int N, int want, int B,
                            int32_t* __restrict__ out, uint32_t* smem, int64_t* sh,
                            int* s_ncand) {
  __shared__ uint32_t s_tau;
  __shared__ int s_need, s_ok;
  const int tid = threadIdx.x;
  const int base = tid * kPer;
  uint32_t u[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) u[j] = base + j < pool ? order_key(__ldg(sc + base + j)) : 0u;
  int64_t tot;
  uint32_t tau = 0;
  int need = want;
  if (want > 0) {
    // sample: the first key of every thread's run (runs past the pool: 0)
    uint32_t* samp = smem;
    const int S = (pool + kPer - 1) / kPer;
    samp[tid] = base < pool ? u[0] : 0u;
    bitonic_desc_u32(samp, kSelThreads);
    const double p = (double)want / pool;
    const int r = (int)((double)want * S / pool);
    const int delta = (int)ceilf(4.0f * sqrtf((float)(S * p * (1.0 - p)))) + 4;
    const int hr = r - delta, lr = r + delta;
    const uint32_t t_hi = hr >= 0 ? samp[hr] : 0xFFFFFFFFu;
    const uint32_t t_lo = lr < S ? samp[lr] : 0u;
    __syncthreads();
    // count keys above the bracket, collect those inside it
    uint64_t* cand = reinterpret_cast<uint64_t*>(smem + kSelThreads);
    if (tid == 0) *s_ncand = 0;
    __syncthreads();
    int above = 0;
    const int lane = tid & 31;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const bool valid = base + j < pool;
      above += valid && u[j] > t_hi;
      const bool take = valid && u[j] <= t_hi && u[j] >= t_lo;
      const unsigned m = __ballot_sync(0xffffffffu, take);
      int slot0 = 0;
      if (m) {
        if (lane == __ffs(m) - 1) slot0 = atomicAdd(s_ncand, __popc(m));
        slot0 = __shfl_sync(0xffffffffu, slot0, __ffs(m) - 1);
        if (take) {
          const int slot = slot0 + __popc(m & ((1u << lane) - 1u));
          if (slot < kFastCand)
            cand[slot] = ((uint64_t)u[j] << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)(base + j));
        }
      }
    }
    const int n_above = (int)block_exclusive_scan(above, &tot, sh);
    (void)n_above;
    const int ab = (int)tot;
    const int nc = *s_ncand;
    const bool ok = nc <= kFastCand && ab < want && ab + nc >= want;
    if (!ok) return false;    // uniform: every thread saw the same totals
    int n2 = 1;
    while (n2 < nc) n2 <<= 1;
    for (int i = nc + tid; i < n2; i += blockDim.x) cand[i] = 0ull;
    bitonic_desc_u64(cand, n2);
    if (tid == 0) {
      const int k = want - ab - 1;                 // the threshold key's place
      const uint32_t t = (uint32_t)(cand[k] >> 32);
      int first = k;
      while (first > 0 && (uint32_t)(cand[first - 1] >> 32) == t) --first;
      s_tau = t;
      s_need = (want - ab) - first;                // ties of t that are kept
    }
    __syncthreads();
    tau = s_tau;
    need = s_need;
  }
  // ascending output from the register runs
  int n_gt = 0, n_eq = 0;
  if (want > 0) {
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const bool valid = base + j < pool;
      n_gt += valid && u[j] > tau;
      n_eq += valid && u[j] == tau;
    }
  }
  const int c0 = min(N, base), c1 = min(N, base + kPer);
  const int eq_before = (int)block_exclusive_scan(n_eq, &tot, sh);
  const int take_eq = max(0, min(n_eq, need - eq_before));
  const int n_rec = max(0, c1 - max(c0, pool));
  int pos = (int)block_exclusive_scan(n_gt + take_eq + n_rec, &tot, sh);
  int eq_seen = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int k = base + j;
    if (k >= N) break;
    bool keep = k >= pool;
    if (!keep && want > 0) {
      if (u[j] > tau) keep = true;
      else if (u[j] == tau) { keep = eq_seen < take_eq; ++eq_seen; }
    }
    if (keep && pos < B) out[pos++] = k;
  }
  return true;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(
    const float* __restrict__ scores, const int32_t* __restrict__ cu, int nseq, int T,
    int Hkv, int R, int B, int32_t* __restrict__ idx, int32_t* __restrict__ kept_len,
    uint32_t* status) {
  extern __shared__ uint32_t dyn_smem[];
  uint32_t* cache = dyn_smem;                                  // staged keys (padded)
  int* cand = reinterpret_cast<int*>(dyn_smem + kCacheWords);  // [kCand] candidates
  __shared__ uint32_t hist[kBins1];
  __shared__ int64_t sh[32];
  __shared__ uint32_t s_digit;
  __shared__ int s_above, s_ncand;
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
  if (N <= kSelThreads * kPer &&
      select_fast(sc, pool, N, want, B, out, dyn_smem, sh, &s_ncand))
    return;
  const bool cached = pool <= kCache;
  // Visit every pool position k (in no particular order) with its key; keys
  // come from shared memory when staged, else from global memory with
  // kBatch independent loads in flight per thread.
  auto for_each = [&](auto&& f) {
    const int step = kBatch * (int)blockDim.x;
    for (int base = tid; base < pool; base += step) {
      uint32_t u[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int k = base + i * (int)blockDim.x;
        u[i] = k < pool ? (cached ? cache[cpos(k)] : order_key(__ldg(sc + k))) : 0u;
      }
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int k = base + i * (int)blockDim.x;
        if (k < pool) f(k, u[i]);
      }
    }
  };
  if (cached) {
    const int step = kBatch * (int)blockDim.x;
    for (int base = tid; base < pool; base += step) {
      float x[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int k = base + i * (int)blockDim.x;
        x[i] = k < pool ? __ldg(sc + k) : 0.f;
      }
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int k = base + i * (int)blockDim.x;
        if (k < pool) cache[cpos(k)] = order_key(x[i]);
      }
    }
    __syncthreads();
  }
  auto key = [&](int k) -> uint32_t {
    return cached ? cache[cpos(k)] : order_key(__ldg(sc + k));
  };

  uint32_t tau = 0;
  int need = want;
  if (want > 0) {
    // ---- digit 1: bits 20..31 over the whole pool
    for (int i = tid; i < kBins1; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for_each([&](int, uint32_t u) { hist_add(hist, u >> 20); });
    __syncthreads();
    find_digit(hist, kBins1, need, &s_digit, &s_above);
    __syncthreads();
    uint32_t prefix = s_digit << 20, pmask = 0xFFF00000u;
    need -= s_above;
    // ---- digits 2 and 3 (bits 10..19, 0..9) over the matching candidates
    if (tid == 0) s_ncand = 0;
    for (int i = tid; i < kBins2; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for_each([&](int k, uint32_t u) {
      const bool take = (u & pmask) == prefix;
      cand_push(cand, &s_ncand, take, k);
      if (take) hist_add(hist, (u >> 10) & 1023u);
    });
    __syncthreads();
    const int ncand = s_ncand;
    const bool listed = ncand <= kCand;
    for (int shift = 10; shift >= 0; shift -= 10) {
      if (shift == 0) {
        for (int i = tid; i < kBins2; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        if (listed) {
          for (int q = tid; q < ncand; q += blockDim.x) {
            const uint32_t u = key(cand[q]);
            if ((u & pmask) == prefix) hist_add(hist, u & 1023u);
          }
        } else {
          for_each([&](int, uint32_t u) {
            if ((u & pmask) == prefix) hist_add(hist, u & 1023u);
          });
        }
        __syncthreads();
      }
      find_digit(hist, kBins2, need, &s_digit, &s_above);
      __syncthreads();
      prefix |= s_digit << shift;
      pmask |= 1023u << shift;
      need -= s_above;
      __syncthreads();
    }
    tau = prefix;
  }

  // ---- ascending output: thread tid owns positions [c0, c1)
  const int per = (N + blockDim.x - 1) / blockDim.x;
  const int c0 = min(N, tid * per), c1 = min(N, c0 + per);
  int n_gt = 0, n_eq = 0;
  if (want > 0) {
    for (int k = c0; k < min(c1, pool); ++k) {
      const uint32_t u = key(k);
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
      const uint32_t u = key(k);
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
  const int dyn = (kCacheWords + kCand) * (int)sizeof(uint32_t);
  cudaError_t err = cudaFuncSetAttribute(select_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
  if (err != cudaSuccess) return err;
  select_kernel<<<nseq * Hkv, kSelThreads, dyn, s>>>(scores, cu, nseq, T, Hkv, R, B, idx,
                                                     kept_len, status);
  return cudaGetLastError();
}

}  // namespace waits
