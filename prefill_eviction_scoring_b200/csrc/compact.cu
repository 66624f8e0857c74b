// KV compaction ("retaining key-value pairs", WAITS README opening summary):
// K_out[s, g, j] = K[cu[s] + idx[s, g, j], g] for j < kept_len[s], zero after.
// Pure byte movement in 16-byte vectors: thread v moves vector v % (d/8) of
// output row v / (d/8) for both K and V, so a warp moves two or four whole
// 256/128-byte rows of each; 32-bit index arithmetic (the host checks the
// vector count fits), shifts instead of divisions where the sizes allow.
#include "waits_internal.cuh"

namespace waits {
namespace {

constexpr int kCompactThreads = 256;

template <int LOG_CPR>
__global__ void __launch_bounds__(kCompactThreads) compact_kernel(
    const uint4* __restrict__ K, const uint4* __restrict__ V, const int32_t* __restrict__ cu,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ kept_len, int Hkv, int B,
    int row_heads, uint32_t total, uint4* __restrict__ Ko, uint4* __restrict__ Vo,
    uint32_t* status) {
  constexpr int kCpr = 1 << LOG_CPR;                 // 16-byte vectors per row (d / 8)
  pdl_allow_next();
  pdl_wait();
  const uint32_t v = blockIdx.x * kCompactThreads + threadIdx.x;
  if (v >= total) return;
  const uint32_t row = v >> LOG_CPR;                 // (s, g, j) flattened
  const int c = (int)(v & (kCpr - 1));
  const uint32_t sg = row / (uint32_t)B;
  const int j = (int)(row - sg * (uint32_t)B);
  const int s = (int)(sg / (uint32_t)Hkv);
  const int g = (int)(sg - (uint32_t)s * (uint32_t)Hkv);
  uint4 kv = make_uint4(0, 0, 0, 0), vv = kv;
  // the four index loads are independent: issue them together, then the
  // row loads (two dependent levels instead of four)
  const int kl = __ldg(kept_len + s), lo = __ldg(cu + s), hi = __ldg(cu + s + 1);
  const int k = __ldg(idx + row);
  if (j < kl) {
    const int N = hi - lo;
    if (k >= 0 && k < N) {
      const size_t src = ((size_t)(lo + k) * row_heads + g) * kCpr + c;
      kv = __ldg(K + src);
      vv = __ldg(V + src);
    } else if (status && c == 0) {
      atomicOr(status, WAITS_DEV_BAD_INDEX);
    }
  }
  Ko[v] = kv;
  Vo[v] = vv;
}

}  // namespace

cudaError_t launch_compact(const uint16_t* K, const uint16_t* V, const int32_t* cu,
                           const int32_t* idx, const int32_t* kept_len, int nseq, int Hkv,
                           int d, int B, uint16_t* Ko, uint16_t* Vo, uint32_t* status,
                           cudaStream_t s, int kv_row_heads) {
  const int rh = kv_row_heads > 0 ? kv_row_heads : Hkv;
  const int64_t total = (int64_t)nseq * Hkv * B * (d / 8);
  if (total >= 0x7fffff00LL) return cudaErrorInvalidValue;
  const unsigned blocks = (unsigned)((total + kCompactThreads - 1) / kCompactThreads);
  const uint4* k4 = reinterpret_cast<const uint4*>(K);
  const uint4* v4 = reinterpret_cast<const uint4*>(V);
  uint4* ko = reinterpret_cast<uint4*>(Ko);
  uint4* vo = reinterpret_cast<uint4*>(Vo);
  if (d == 128)
    return launch_pdl(compact_kernel<4>, dim3(blocks), dim3(kCompactThreads), 0, s, k4, v4, cu,
                      idx, kept_len, Hkv, B, rh, (uint32_t)total, ko, vo, status);
  return launch_pdl(compact_kernel<3>, dim3(blocks), dim3(kCompactThreads), 0, s, k4, v4, cu, idx,
                    kept_len, Hkv, B, rh, (uint32_t)total, ko, vo, status);
}

}  // namespace waits
