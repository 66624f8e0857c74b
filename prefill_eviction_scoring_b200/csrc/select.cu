// Per (sequence, KV head) selection (WAITS README, Quickstart budgets): keep
// the recent window [N-R, N) and the B-R highest scores of [0, N-R), ties to
// the lower index, reported in ascending order.
//
// One 1024-thread CTA per (sequence, KV head).  Scores are mapped to a
// monotone 32-bit image; the (B-R)-th largest image tau is found exactly by
// a three-digit radix select (12 + 10 + 10 bits):
//   1. one pass stages the pool's images in shared memory (16-byte loads)
//      and histograms their top 12 bits;
//   2. a block scan over the bins finds the bin that holds the (B-R)-th
//      largest image;
//   3. the images in that bin are copied to a candidate list, and the two
//      lower digits are resolved on the candidates alone (on the whole pool
//      when the bin holds more than the list's capacity);
//   4. the output pass gives each thread 32 consecutive positions; one block
//      scan of packed (above tau, equal to tau) counts per chunk of 32768
//      positions places every kept position, threshold ties taken lowest
//      index first.
// Pools larger than the staging buffer are re-read from global memory
// (L2) in each pass instead.
#include "waits_internal.cuh"

namespace waits {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kGroupsPerThread = 8;              // output pass: 32 consecutive positions
constexpr int kStageKeys = kSelThreads * kGroupsPerThread * 4;   // 32768 (128 KB)
constexpr int kBins1 = 4096;                     // bits 20..31
constexpr int kCopies = 4;                       // first-digit histograms (by warp % 4)
constexpr int kBins2 = 1024;                     // bits 10..19, then 0..9
constexpr int kCand = 4096;                      // candidate list capacity

// Monotone map of fp32 to uint32: a < b (as floats, -0 == +0) iff
// key(a) < key(b).  Scores from waits_score are >= 0, but waits_select takes
// any finite fp32 input.
__device__ inline uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;                       // -0 ranks with +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct SelSmem {
  uint32_t hist[kCopies * kBins1];
  uint32_t cand[kCand];
  int64_t scan[32];
  uint32_t digit;
  int32_t above;
  int32_t count;
  int32_t ncand;
};

// The pool seen as aligned 16-byte groups: group i holds positions
// 4i - off .. 4i - off + 3 (off = misalignment of the first score in
// floats); positions outside [0, pool) are invalid.
struct Pool {
  const float* base;   // 16-byte aligned, = scores of position -off
  int off, pool, ngroups;
  const uint4* stage;  // staged images, or null
  __device__ uint4 image(int i, float4 f) const {
    const int p = 4 * i - off;
    return make_uint4(p + 0 >= 0 && p + 0 < pool ? order_key(f.x) : 0u,
                      p + 1 >= 0 && p + 1 < pool ? order_key(f.y) : 0u,
                      p + 2 >= 0 && p + 2 < pool ? order_key(f.z) : 0u,
                      p + 3 >= 0 && p + 3 < pool ? order_key(f.w) : 0u);
  }
  __device__ uint4 group(int i) const {
    if (stage) return stage[swz(i)];
    return image(i, __ldg(reinterpret_cast<const float4*>(base) + i));
  }
  // Staged slot of group i: the eight groups of each 128-byte block are
  // permuted by bits 3..5 of i, so both 32 consecutive groups (passes 1-3)
  // and groups 8t + j of threads t = 0..31 (output pass) hit all 32 banks.
  __device__ static int swz(int i) { return i ^ ((i >> 3) & 7); }
  // validity of the four positions of group i, as bits
  __device__ uint32_t valid(int i) const {
    const int p = 4 * i - off;
    uint32_t m = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) m |= (uint32_t)(p + e >= 0 && p + e < pool) << e;
    return m;
  }
};

__device__ inline uint32_t comp(const uint4& v, int e) {
  return e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w;
}

// Find the bin (bins in descending order) holding the need-th largest image
// among `nb` bins of sm.hist (summed over `copies` histograms of nb bins);
// result in sm.digit / sm.above, the bin's count in sm.count.  nb / 1024
// bins per thread (1 or 4).  Ends with a barrier.
__device__ void find_bin(SelSmem& sm, int nb, int copies, int need) {
  const int per = nb / kSelThreads;
  const int top = nb - 1 - (int)threadIdx.x * per;
  uint32_t c[4] = {0, 0, 0, 0}, sum = 0;
  for (int i = 0; i < per; ++i) {
    for (int k = 0; k < copies; ++k) c[i] += sm.hist[k * nb + top - i];
    sum += c[i];
  }
  int64_t tot;
  const int64_t ex = block_exclusive_scan((int64_t)sum, &tot, sm.scan);
  if (ex < need && ex + sum >= need) {
    int64_t cum = ex;
    for (int i = 0; i < per; ++i) {
      if (cum + c[i] >= need) {
        sm.digit = (uint32_t)(top - i);
        sm.above = (int)cum;
        sm.count = (int)c[i];
        break;
      }
      cum += c[i];
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(
    const float* __restrict__ scores, const int32_t* __restrict__ cu, int nseq, int T,
    int Hkv, int R, int B, int32_t* __restrict__ idx, int32_t* __restrict__ kept_len,
    uint32_t* status) {
  extern __shared__ uint4 stage_raw[];      // [kStageKeys / 4] staged groups, then SelSmem
  SelSmem& sm = *reinterpret_cast<SelSmem*>(stage_raw + kStageKeys / 4);
  const int tid = threadIdx.x;
  pdl_allow_next();
  pdl_wait();
  const int s = blockIdx.x / Hkv, g = blockIdx.x % Hkv;
  const int lo = cu[s], hi = cu[s + 1];
  int32_t* out = idx + ((size_t)s * Hkv + g) * B;
  const bool bad = (s == 0 && lo != 0) || hi < lo || hi > T || (s == nseq - 1 && hi != T);
  if (bad) {
    for (int j = tid; j < B; j += kSelThreads) out[j] = -1;
    if (tid == 0) {
      if (g == 0) kept_len[s] = 0;
      if (status) atomicOr(status, WAITS_DEV_BAD_SEQLENS);
    }
    return;
  }
  const int N = hi - lo;
  if (g == 0 && tid == 0) kept_len[s] = N < B ? N : B;
  if (N <= B) {
    for (int j = tid; j < B; j += kSelThreads) out[j] = j < N ? j : -1;
    return;
  }
  const int want = B - R;            // positions taken from the pool by score
  const int pool = N - R;            // > want because N > B
  for (int j = tid; j < R; j += kSelThreads) out[want + j] = pool + j;   // recent window
  if (want == 0) return;

  // ---- 1. stage the images (if they fit) and histogram the top 12 bits
  const float* sc = scores + (size_t)g * T + lo;
  Pool P;
  P.off = (int)((reinterpret_cast<uintptr_t>(sc) >> 2) & 3u);
  P.base = sc - P.off;
  P.pool = pool;
  P.ngroups = (pool + P.off + 3) / 4;
  P.stage = nullptr;
  const bool staged = 4 * P.ngroups <= kStageKeys;
  for (int i = tid; i < kCopies * kBins1; i += kSelThreads) sm.hist[i] = 0u;
  if (tid == 0) sm.ncand = 0;
  __syncthreads();
  {
    uint32_t* hist = sm.hist + ((tid >> 5) & (kCopies - 1)) * kBins1;
    constexpr int kUnroll = 4;
    for (int i0 = 0; i0 < P.ngroups; i0 += kUnroll * kSelThreads) {
      float4 f[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int i = i0 + u * kSelThreads + tid;
        f[u] = i < P.ngroups ? __ldg(reinterpret_cast<const float4*>(P.base) + i)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int i = i0 + u * kSelThreads + tid;
        if (i < P.ngroups) {
          const uint4 v = P.image(i, f[u]);
          if (staged) stage_raw[Pool::swz(i)] = v;
          const uint32_t ok = P.valid(i);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if ((ok >> e) & 1u) atomicAdd(&hist[comp(v, e) >> 20], 1u);
        }
      }
    }
  }
  if (staged) P.stage = stage_raw;
  __syncthreads();

  // ---- 2. threshold bin of the first digit
  int need = want;
  find_bin(sm, kBins1, kCopies, need);
  uint32_t prefix = sm.digit << 20, pmask = 0xFFF00000u;
  need -= sm.above;
  const int nbin = sm.count;
  __syncthreads();

  // ---- 3. the two lower digits, on the bin's candidates when they fit
  const bool listed = nbin <= kCand;
  if (listed) {
    for (int i0 = 0; i0 < P.ngroups; i0 += kSelThreads) {    // whole warps iterate
      const int i = i0 + tid;
      uint4 v = make_uint4(0, 0, 0, 0);
      uint32_t ok = 0;
      if (i < P.ngroups) { v = P.group(i); ok = P.valid(i); }
      uint32_t take = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        take |= (uint32_t)(((ok >> e) & 1u) && (comp(v, e) & pmask) == prefix) << e;
      // one shared-memory atomic per warp for the whole warp's candidates
      const int n = __popc(take);
      int incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if ((tid & 31) >= o) incl += y;
      }
      const int wtot = __shfl_sync(0xffffffffu, incl, 31);
      int base = 0;
      if ((tid & 31) == 31 && wtot) base = atomicAdd(&sm.ncand, wtot);
      base = __shfl_sync(0xffffffffu, base, 31) + incl - n;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if ((take >> e) & 1u) {
          if (base < kCand) sm.cand[base] = comp(v, e);    // base < nbin <= kCand
          ++base;
        }
    }
    __syncthreads();
  }
#pragma unroll 1
  for (int shift = 10; shift >= 0; shift -= 10) {
    for (int i = tid; i < kBins2; i += kSelThreads) sm.hist[i] = 0u;
    __syncthreads();
    if (listed) {
      for (int q = tid; q < nbin; q += kSelThreads) {
        const uint32_t x = sm.cand[q];
        if ((x & pmask) == prefix) atomicAdd(&sm.hist[(x >> shift) & 1023u], 1u);
      }
    } else {
      for (int i = tid; i < P.ngroups; i += kSelThreads) {
        const uint4 v = P.group(i);
        const uint32_t ok = P.valid(i);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t x = comp(v, e);
          if (((ok >> e) & 1u) && (x & pmask) == prefix)
            atomicAdd(&sm.hist[(x >> shift) & 1023u], 1u);
        }
      }
    }
    __syncthreads();
    find_bin(sm, kBins2, 1, need);
    prefix |= sm.digit << shift;
    pmask |= 1023u << shift;
    need -= sm.above;
    __syncthreads();
  }
  const uint32_t tau = prefix;   // need = ties of tau to keep, lowest index first

  // ---- 4. ascending output: thread t walks groups 8t .. 8t+7 of a chunk of
  // 8192 groups (32 consecutive positions); one block scan per chunk
  int64_t gt_base = 0, eq_base = 0;
  for (int c0 = 0; c0 < P.ngroups; c0 += kSelThreads * kGroupsPerThread) {
    const int g0 = c0 + kGroupsPerThread * tid;
    uint32_t gtm = 0, eqm = 0;     // bit 4j + e: position 4(g0 + j) + e - off
#pragma unroll
    for (int j = 0; j < kGroupsPerThread; ++j) {
      if (g0 + j < P.ngroups) {
        const uint4 v = P.group(g0 + j);
        const uint32_t ok = P.valid(g0 + j);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t x = comp(v, e);
          gtm |= (uint32_t)(((ok >> e) & 1u) && x > tau) << (4 * j + e);
          eqm |= (uint32_t)(((ok >> e) & 1u) && x == tau) << (4 * j + e);
        }
      }
    }
    // packed counts: above tau in the high half, ties in the low half
    const int64_t mine = ((int64_t)__popc(gtm) << 32) | (int64_t)__popc(eqm);
    int64_t tot;
    const int64_t ex = block_exclusive_scan(mine, &tot, sm.scan);
    int64_t gt_before = gt_base + (ex >> 32), eq_before = eq_base + (ex & 0xFFFFFFFFll);
    const int p0 = 4 * g0 - P.off;
    uint32_t any = gtm | eqm;
    while (any) {
      const int b = __ffs(any) - 1;
      any &= any - 1;
      const int64_t gb = gt_before + __popc(gtm & ((1u << b) - 1u));
      const int64_t eb = eq_before + __popc(eqm & ((1u << b) - 1u));
      const bool gt = (gtm >> b) & 1u;
      if (gt || eb < need) {
        const int64_t pos = gb + (eb < need ? eb : (int64_t)need);
        if (pos < want) out[pos] = p0 + b;
      }
    }
    gt_base += tot >> 32;
    eq_base += tot & 0xFFFFFFFFll;
  }
}

}  // namespace

cudaError_t launch_select(const float* scores, const int32_t* cu, int nseq, int T, int Hkv,
                          int R, int B, int32_t* idx, int32_t* kept_len, uint32_t* status,
                          cudaStream_t s) {
  const int64_t grid = (int64_t)nseq * Hkv;
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  const int dyn = kStageKeys * (int)sizeof(uint32_t) + (int)sizeof(SelSmem);
  cudaError_t err = cudaFuncSetAttribute(select_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
  if (err != cudaSuccess) return err;
  return launch_pdl(select_kernel, dim3((unsigned)grid), dim3(kSelThreads), (size_t)dyn, s,
                    scores, cu, nseq, T, Hkv, R, B, idx, kept_len, status);
}

}  // namespace waits
