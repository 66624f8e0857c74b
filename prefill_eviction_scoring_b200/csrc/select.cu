// Per (sequence, KV head) selection (WAITS README, Quickstart budgets): keep
// the recent window [N-R, N) and the B-R highest scores of [0, N-R), ties to
// the lower index, reported in ascending order.
//
// One thread-block cluster of kC CTAs per (sequence, KV head); CTA r of the
// cluster owns slice r of the pool (a contiguous range of 16-byte groups).
// Scores are mapped to a monotone 32-bit image; the (B-R)-th largest image
// tau is found exactly by a radix select over digits of 12 + 10 + 10 bits.
// For each digit every CTA histograms the images of its slice that carry the
// digits found so far and sends the histogram to every CTA of the cluster
// (distributed shared memory): the first digit's non-empty bins are added
// into each CTA's cluster histogram; the second digit's into the CTA that
// owns the bin (rank = bin / 128), from which every CTA gathers the sums
// after the barrier; the third digit's histogram is stored per sending CTA.
// Every CTA then finds the same digit itself, so a digit costs one cluster
// barrier.  With the second and third digits each
// CTA also sends how many of its images lie above the previous digit's bin;
// from those counts and the per-CTA third-digit histograms every CTA knows
// how many images above tau and equal to tau the slices before its own hold,
// and places its kept positions with block scans, ties to tau taken lowest
// index first.  The first pass stages the slice's images in shared memory,
// so the later passes read no global memory.
//
// With the KV copy (waits_select_compact, waits_compress) the same kernel
// also compacts K and V: after each output round the CTA copies the rows of
// the slots it has just filled (a contiguous range of slots, their source
// positions staged in shared memory), and the CTAs of the cluster share the
// recent window's rows and any zero rows.
#include "waits_internal.cuh"

namespace waits {
namespace {

constexpr int kC = 8;                            // CTAs per cluster (portable maximum)
constexpr int kSelThreads = 512;
constexpr int kStageGroups = 2048;               // per CTA: 8192 staged images (32 KB)
constexpr int kBins1 = 4096;                     // bits 20..31
constexpr int kCopies = 4;                       // local first-digit histograms (warp % 4)
constexpr int kBins2 = 1024;                     // bits 10..19, then 0..9
constexpr int kMaxPer = kBins1 / kSelThreads;    // bins per thread in find_bin
constexpr int kOutGroups = 2;                    // output pass: groups per thread and round
constexpr int kRoundKeys = 4 * kOutGroups * kSelThreads;   // positions per output round

// Monotone map of fp32 to uint32: a < b (as floats, -0 == +0) iff
// key(a) < key(b).  Scores from waits_score are >= 0, but waits_select takes
// any finite fp32 input.
__device__ inline uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;                       // -0 ranks with +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct SelSmem {
  uint32_t hist[kCopies * kBins1];   // this CTA's histograms
  uint32_t g1[kBins1];               // the cluster's first-digit histogram
  uint32_t g2[kBins2];               // the cluster's second-digit histogram (owned bins)
  uint32_t h3[kC][kBins2];           // third-digit histogram of each slice
  uint32_t above1[kC];               // per slice: images above the first digit's bin
  uint32_t above2[kC];               // per slice: images in it, above the second's
  int64_t scan[32];
  uint32_t digit;                    // find_bin's result
  int32_t above;
  int32_t src[kRoundKeys];           // KV copy: source position of each slot of a round
};

// K / V of the compaction (null K: selection only).  Rows are d / 8 16-byte
// vectors (1 << log_cpr).
struct KVCopy {
  const uint4* K;
  const uint4* V;
  uint4* Ko;
  uint4* Vo;
  int log_cpr;
  int row_heads;   // heads per token row of K and V in memory
};

// Output rows [r0, r1) of (sequence s, KV head g): slot j gets source
// position src_of(j) of the sequence (starting at token lo), or zeros when
// src_of(j) < 0.  All threads of the CTA, one 16-byte vector of K and of V
// each per turn, kCopyUnroll turns with their loads in flight before the
// stores.  V may be page-locked host memory mapped into the device's address
// space (the host-buffer entry point), so it is read with plain coherent
// loads.
template <typename F>
__device__ inline void copy_rows(const KVCopy& c, int Hkv, int B, int s, int g, int lo, int r0,
                                 int r1, F src_of) {
  constexpr int kCopyUnroll = 4;
  const uint4* __restrict__ K = c.K;
  const uint4* V = c.V;
  uint4* __restrict__ Ko = c.Ko;
  uint4* __restrict__ Vo = c.Vo;
  const int cpr = 1 << c.log_cpr;
  const int n = (r1 - r0) << c.log_cpr;
  const int nt = (int)blockDim.x;
  const size_t out0 = ((size_t)s * Hkv + g) * (size_t)B;
  for (int v0 = (int)threadIdx.x; v0 < n; v0 += kCopyUnroll * nt) {
    uint4 kx[kCopyUnroll], vx[kCopyUnroll];
    size_t dst[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      const int v = v0 + u * nt;
      kx[u] = make_uint4(0, 0, 0, 0);
      vx[u] = kx[u];
      dst[u] = 0;
      if (v < n) {
        const int j = r0 + (v >> c.log_cpr), col = v & (cpr - 1);
        const int src = src_of(j);
        dst[u] = ((out0 + j) << c.log_cpr) + col;
        if (src >= 0) {
          const size_t from = ((((size_t)lo + src) * c.row_heads + g) << c.log_cpr) + col;
          kx[u] = __ldg(K + from);
          vx[u] = ld_global_v4(V + from);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      if (v0 + u * nt < n) {
        Ko[dst[u]] = kx[u];
        Vo[dst[u]] = vx[u];
      }
    }
  }
}

// ---------------------------------------------------------- cluster ops ---
__device__ inline uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Every thread of every CTA in the cluster; orders shared-memory writes
// (local and remote) before the barrier with reads after it.
__device__ inline void cluster_sync() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ inline uint32_t peer(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(r)
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))), "r"(rank));
  return r;
}
__device__ inline void peer_add(uint32_t addr, uint32_t v) {
  asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ inline uint32_t peer_ld32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ inline void peer_st32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// The pool seen as aligned 16-byte groups: group i holds positions
// 4i - off .. 4i - off + 3 (off = misalignment of the first score in
// floats); positions outside [0, pool) are invalid.
struct Pool {
  const float* base;   // 16-byte aligned, = scores of position -off
  int off, pool, ngroups;
  __device__ uint4 image(int i, float4 f) const {
    const int p = 4 * i - off;
    return make_uint4(p + 0 >= 0 && p + 0 < pool ? order_key(f.x) : 0u,
                      p + 1 >= 0 && p + 1 < pool ? order_key(f.y) : 0u,
                      p + 2 >= 0 && p + 2 < pool ? order_key(f.z) : 0u,
                      p + 3 >= 0 && p + 3 < pool ? order_key(f.w) : 0u);
  }
  __device__ uint4 load(int i) const {
    return image(i, __ldg(reinterpret_cast<const float4*>(base) + i));
  }
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
// among the nb bins of h; result in sm.digit / sm.above.  Ends with a barrier.
__device__ void find_bin(SelSmem& sm, const uint32_t* h, int nb, int need) {
  const int per = nb / kSelThreads;
  const int top = nb - 1 - (int)threadIdx.x * per;
  uint32_t c[kMaxPer], sum = 0;
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    c[i] = i < per ? h[top - i] : 0u;
    sum += c[i];
  }
  int64_t tot;
  const int64_t ex = block_exclusive_scan((int64_t)sum, &tot, sm.scan);
  if (ex < need && ex + sum >= need) {
    int64_t cum = ex;
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i) {
      if (i < per && cum + c[i] >= need) {
        sm.digit = (uint32_t)(top - i);
        sm.above = (int)cum;
        break;
      }
      cum += c[i];
    }
  }
  __syncthreads();
}

template <bool COPY>
__global__ void __launch_bounds__(kSelThreads) select_kernel(
    const float* __restrict__ scores, const int32_t* __restrict__ cu, int nseq, int T,
    int Hkv, int R, int B, int32_t* __restrict__ idx, int32_t* __restrict__ kept_len,
    uint32_t* status, KVCopy kv) {
  extern __shared__ uint4 dyn_smem[];
  uint4* stage = dyn_smem;                                     // [kStageGroups]
  SelSmem& sm = *reinterpret_cast<SelSmem*>(dyn_smem + kStageGroups);
  const int tid = threadIdx.x;
  const uint32_t rank = cluster_rank();
  pdl_allow_next();
  // nothing here depends on the previous kernel: zero the histograms and
  // meet the cluster (every CTA runs before any shared memory is shared)
  for (int i = tid; i < kCopies * kBins1; i += kSelThreads) sm.hist[i] = 0u;
  for (int i = tid; i < kBins1; i += kSelThreads) sm.g1[i] = 0u;
  for (int i = tid; i < kBins2; i += kSelThreads) sm.g2[i] = 0u;
  for (int i = tid; i < kC * kBins2; i += kSelThreads) (&sm.h3[0][0])[i] = 0u;
  __syncthreads();
  cluster_sync();
  pdl_wait();
  // every branch below is taken by all CTAs of a cluster alike
  const int sg = blockIdx.x / kC;
  const int s = sg / Hkv, g = sg % Hkv;
  const int lo = cu[s], hi = cu[s + 1];
  int32_t* out = idx + ((size_t)s * Hkv + g) * B;
  const bool bad = (s == 0 && lo != 0) || hi < lo || hi > T || (s == nseq - 1 && hi != T);
  // the cluster's share of output rows [0, n): rank r takes [n r / kC, n (r + 1) / kC)
  auto share = [&](int n, int& r0, int& r1) {
    r0 = (int)((int64_t)n * rank / kC);
    r1 = (int)((int64_t)n * (rank + 1) / kC);
  };
  if (bad) {
    if (rank == 0) {
      for (int j = tid; j < B; j += kSelThreads) out[j] = -1;
      if (tid == 0) {
        if (g == 0) kept_len[s] = 0;
        if (status) atomicOr(status, WAITS_DEV_BAD_SEQLENS);
      }
    }
    if (COPY) {
      int r0, r1;
      share(B, r0, r1);
      copy_rows(kv, Hkv, B, s, g, 0, r0, r1, [](int) { return -1; });
    }
    return;
  }
  const int N = hi - lo;
  if (rank == 0 && g == 0 && tid == 0) kept_len[s] = N < B ? N : B;
  if (N <= B) {
    if (rank == 0)
      for (int j = tid; j < B; j += kSelThreads) out[j] = j < N ? j : -1;
    if (COPY) {
      int r0, r1;
      share(B, r0, r1);
      copy_rows(kv, Hkv, B, s, g, lo, r0, r1, [N](int j) { return j < N ? j : -1; });
    }
    return;
  }
  const int want = B - R;            // positions taken from the pool by score
  const int pool = N - R;            // > want because N > B
  if (rank == 0)
    for (int j = tid; j < R; j += kSelThreads) out[want + j] = pool + j;   // recent window
  if (COPY) {
    int r0, r1;
    share(R, r0, r1);
    copy_rows(kv, Hkv, B, s, g, lo, want + r0, want + r1,
              [want, pool](int j) { return pool + (j - want); });
  }
  if (want == 0) return;

  const float* sc = scores + (size_t)g * T + lo;
  Pool P;
  P.off = (int)((reinterpret_cast<uintptr_t>(sc) >> 2) & 3u);
  P.base = sc - P.off;
  P.pool = pool;
  P.ngroups = (pool + P.off + 3) / 4;
  // this CTA's slice of groups
  const int g_lo = (int)((int64_t)P.ngroups * rank / kC);
  const int g_hi = (int)((int64_t)P.ngroups * (rank + 1) / kC);
  const bool staged = g_hi - g_lo <= kStageGroups;
  auto group = [&](int i) { return staged ? stage[i - g_lo] : P.load(i); };
  uint32_t* loc2 = sm.hist + kBins1;       // this slice's second-digit histogram
  uint32_t* loc3 = sm.hist + 2 * kBins1;   // this slice's third-digit histogram

  // ---- first digit: stage the slice and histogram its top 12 bits
  {
    uint32_t* hist = sm.hist + ((tid >> 5) & (kCopies - 1)) * kBins1;
    constexpr int kUnroll = 4;
    for (int i0 = g_lo; i0 < g_hi; i0 += kUnroll * kSelThreads) {
      float4 f[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int i = i0 + u * kSelThreads + tid;
        f[u] = i < g_hi ? __ldg(reinterpret_cast<const float4*>(P.base) + i)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int i = i0 + u * kSelThreads + tid;
        if (i < g_hi) {
          const uint4 v = P.image(i, f[u]);
          if (staged) stage[i - g_lo] = v;
          const uint32_t ok = P.valid(i);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if ((ok >> e) & 1u) atomicAdd(&hist[comp(v, e) >> 20], 1u);
        }
      }
    }
  }
  __syncthreads();
  // copy 0 keeps this slice's histogram (summed over the copies); its
  // non-empty bins are added into every CTA's cluster histogram
  for (int b = tid; b < kBins1; b += kSelThreads) {
    uint32_t c = 0;
#pragma unroll
    for (int k = 0; k < kCopies; ++k) c += sm.hist[k * kBins1 + b];
    sm.hist[b] = c;
    if (c) {
#pragma unroll
      for (int r = 0; r < kC; ++r) peer_add(peer(&sm.g1[b], (uint32_t)r), c);
    }
  }
  cluster_sync();   // every CTA holds the cluster's first-digit histogram
  find_bin(sm, sm.g1, kBins1, want);
  const uint32_t d1 = sm.digit;
  int need = want - sm.above;

  // ---- second digit: bits 10..19 of the images in bin d1
  {
    uint32_t above = 0;
    for (int b = tid; b < kBins1; b += kSelThreads) above += (uint32_t)b > d1 ? sm.hist[b] : 0u;
    for (int b = tid; b < kBins2; b += kSelThreads) loc2[b] = 0u;
    int64_t tot;
    block_exclusive_scan((int64_t)above, &tot, sm.scan);   // barrier: loc2 is zero
    if (tid < kC) peer_st32(peer(&sm.above1[rank], (uint32_t)tid), (uint32_t)tot);
    for (int i = g_lo + tid; i < g_hi; i += kSelThreads) {
      const uint4 v = group(i);
      const uint32_t ok = P.valid(i);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t x = comp(v, e);
        if (((ok >> e) & 1u) && (x >> 20) == d1) atomicAdd(&loc2[(x >> 10) & (kBins2 - 1)], 1u);
      }
    }
    __syncthreads();
    for (int b = tid; b < kBins2; b += kSelThreads) {
      const uint32_t c = loc2[b];
      if (c) peer_add(peer(&sm.g2[b], (uint32_t)(b / (kBins2 / kC))), c);
    }
  }
  cluster_sync();   // the owners hold the second-digit histogram; every CTA the counts
  // gather the owners' bins (into loc3, zeroed again below)
  for (int b = tid; b < kBins2; b += kSelThreads)
    loc3[b] = peer_ld32(peer(&sm.g2[b], (uint32_t)(b / (kBins2 / kC))));
  __syncthreads();
  find_bin(sm, loc3, kBins2, need);
  const uint32_t d2 = sm.digit;
  need -= sm.above;
  const uint32_t pre2 = (d1 << 10) | d2;   // top 22 bits of tau

  // ---- third digit: bits 0..9 of the images carrying pre2, per slice
  {
    uint32_t above = 0;
    for (int b = tid; b < kBins2; b += kSelThreads) above += (uint32_t)b > d2 ? loc2[b] : 0u;
    for (int b = tid; b < kBins2; b += kSelThreads) loc3[b] = 0u;
    int64_t tot;
    block_exclusive_scan((int64_t)above, &tot, sm.scan);   // barrier: loc3 is zero
    if (tid < kC) peer_st32(peer(&sm.above2[rank], (uint32_t)tid), (uint32_t)tot);
    for (int i = g_lo + tid; i < g_hi; i += kSelThreads) {
      const uint4 v = group(i);
      const uint32_t ok = P.valid(i);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t x = comp(v, e);
        if (((ok >> e) & 1u) && (x >> 10) == pre2) atomicAdd(&loc3[x & (kBins2 - 1)], 1u);
      }
    }
    __syncthreads();
    for (int b = tid; b < kBins2; b += kSelThreads) {
      const uint32_t c = loc3[b];
      if (c) {
#pragma unroll
        for (int r = 0; r < kC; ++r) peer_st32(peer(&sm.h3[rank][b], (uint32_t)r), c);
      }
    }
  }
  cluster_sync();   // every CTA holds every slice's third-digit histogram; no remote
                    // shared-memory access follows
  // cluster histogram of the third digit (into loc2, no longer needed)
  for (int b = tid; b < kBins2; b += kSelThreads) {
    uint32_t c = 0;
#pragma unroll
    for (int r = 0; r < kC; ++r) c += sm.h3[r][b];
    loc2[b] = c;
  }
  __syncthreads();
  find_bin(sm, loc2, kBins2, need);
  const uint32_t d3 = sm.digit;
  need -= sm.above;
  const uint32_t tau = (pre2 << 10) | d3;   // need = ties of tau to keep, lowest index first
  // images above tau (high half) and equal to tau (low half) in the slices
  // before this one
  int64_t before = 0;
  for (uint32_t r = 0; r < rank; ++r) {
    if (tid == 0)
      before += ((int64_t)sm.above1[r] + sm.above2[r]) * (int64_t(1) << 32) + sm.h3[r][d3];
    for (int b = tid; b < kBins2; b += kSelThreads)
      before += (uint32_t)b > d3 ? (int64_t)sm.h3[r][b] << 32 : 0;
  }
  int64_t gt_base, eq_base;
  {
    int64_t tot;
    block_exclusive_scan(before, &tot, sm.scan);
    gt_base = tot >> 32;
    eq_base = tot & 0xFFFFFFFFll;
  }


  // ---- ascending positions: rounds of kOutGroups * kSelThreads consecutive
  // groups (kOutGroups per thread), one block scan of packed (above tau,
  // equal to tau) counts per round; the kept positions of a round fill a
  // contiguous range of slots
  for (int i0 = g_lo; i0 < g_hi; i0 += kOutGroups * kSelThreads) {
    const int ib = i0 + kOutGroups * tid;
    uint32_t gtm = 0, eqm = 0;     // bit 4j + e: position 4(ib + j) + e - off
#pragma unroll
    for (int j = 0; j < kOutGroups; ++j) {
      const int i = ib + j;
      if (i < g_hi) {
        const uint4 v = group(i);
        const uint32_t ok = P.valid(i);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t x = comp(v, e);
          gtm |= (uint32_t)(((ok >> e) & 1u) && x > tau) << (4 * j + e);
          eqm |= (uint32_t)(((ok >> e) & 1u) && x == tau) << (4 * j + e);
        }
      }
    }
    const int64_t mine = ((int64_t)__popc(gtm) << 32) | (int64_t)__popc(eqm);
    int64_t tot;
    const int64_t ex = block_exclusive_scan(mine, &tot, sm.scan);
    const int64_t gt_before = gt_base + (ex >> 32), eq_before = eq_base + (ex & 0xFFFFFFFFll);
    // this round's slots: [slot0, slot0 + kept)
    const int64_t slot0 = gt_base + (eq_base < need ? eq_base : (int64_t)need);
    const int p0 = 4 * ib - P.off;
    uint32_t any = gtm | eqm;
    while (any) {
      const int b = __ffs(any) - 1;
      any &= any - 1;
      const int64_t gb = gt_before + __popc(gtm & ((1u << b) - 1u));
      const int64_t eb = eq_before + __popc(eqm & ((1u << b) - 1u));
      const bool gt = (gtm >> b) & 1u;
      if (gt || eb < need) {
        const int64_t pos = gb + (eb < need ? eb : (int64_t)need);
        if (pos < want) {
          out[pos] = p0 + b;
          if (COPY) sm.src[pos - slot0] = p0 + b;
        }
      }
    }
    gt_base += tot >> 32;
    eq_base += tot & 0xFFFFFFFFll;
    if (COPY) {
      const int64_t slot1 = gt_base + (eq_base < need ? eq_base : (int64_t)need);
      __syncthreads();
      copy_rows(kv, Hkv, B, s, g, lo, (int)slot0, (int)(slot1 < want ? slot1 : want),
                [&](int j) { return sm.src[j - slot0]; });
      // the next round's scan (block barriers) orders these reads of sm.src
      // before its writes
    }
  }
}

}  // namespace

cudaError_t launch_select(const float* scores, const int32_t* cu, int nseq, int T, int Hkv,
                          int R, int B, int32_t* idx, int32_t* kept_len, uint32_t* status,
                          cudaStream_t s, const uint16_t* K, const uint16_t* V, int d,
                          uint16_t* Ko, uint16_t* Vo, int kv_row_heads) {
  const int64_t grid = (int64_t)nseq * Hkv * kC;
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  const int dyn = kStageGroups * (int)sizeof(uint4) + (int)sizeof(SelSmem);
  KVCopy kv{reinterpret_cast<const uint4*>(K), reinterpret_cast<const uint4*>(V),
            reinterpret_cast<uint4*>(Ko), reinterpret_cast<uint4*>(Vo), d == 128 ? 4 : 3,
            kv_row_heads > 0 ? kv_row_heads : Hkv};
  auto kernel = K ? select_kernel<true> : select_kernel<false>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
  if (err != cudaSuccess) return err;
  return launch_pdl_cluster(kernel, dim3((unsigned)grid), dim3(kSelThreads), kC, (size_t)dyn, s,
                            scores, cu, nseq, T, Hkv, R, B, idx, kept_len, status, kv);
}

}  // namespace waits
