// KV compaction ("retaining key-value pairs", WAITS README opening summary):
// K_out[s, g, j] = K[cu[s] + idx[s, g, j], g] for j < kept_len[s], zero after.
// Pure byte movement in 16-byte vectors; each thread moves one vector of K
// and the same vector of V; grid-stride over all output vectors.
#include "waits_internal.cuh"

namespace waits {
namespace {

__global__ void __launch_bounds__(256) compact_kernel(
    const uint4* __restrict__ K, const uint4* __restrict__ V, const int32_t* __restrict__ cu,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ kept_len, int nseq, int Hkv,
    int chunks /* d / 8 */, int B, uint4* __restrict__ Ko, uint4* __restrict__ Vo,
    uint32_t* status) {
  pdl_allow_next();
  pdl_wait();
  const int64_t total = (int64_t)nseq * Hkv * B * chunks;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < total;
       v += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = v / chunks;          // (s, g, j)
    const int c = (int)(v - row * chunks);
    const int j = (int)(row % B);
    const int64_t sg = row / B;
    const int g = (int)(sg % Hkv);
    const int s = (int)(sg / Hkv);
    uint4 kv = make_uint4(0, 0, 0, 0), vv = kv;
    if (j < kept_len[s]) {
      const int lo = cu[s], N = cu[s + 1] - lo;
      const int k = idx[row];
      if (k >= 0 && k < N) {
        const int64_t src = ((int64_t)(lo + k) * Hkv + g) * chunks + c;
        kv = K[src];
        vv = V[src];
      } else if (status && c == 0) {
        atomicOr(status, WAITS_DEV_BAD_INDEX);
      }
    }
    Ko[v] = kv;
    Vo[v] = vv;
  }
}

}  // namespace

cudaError_t launch_compact(const uint16_t* K, const uint16_t* V, const int32_t* cu,
                           const int32_t* idx, const int32_t* kept_len, int nseq, int Hkv,
                           int d, int B, uint16_t* Ko, uint16_t* Vo, uint32_t* status,
                           cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t total = (int64_t)nseq * Hkv * B * (d / 8);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = (int64_t)sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return launch_pdl(compact_kernel, dim3((unsigned)blocks), dim3(256), 0, s,
                    reinterpret_cast<const uint4*>(K), reinterpret_cast<const uint4*>(V), cu,
                    idx, kept_len, nseq, Hkv, d / 8, B, reinterpret_cast<uint4*>(Ko),
                    reinterpret_cast<uint4*>(Vo), status);
}

}  // namespace waits
