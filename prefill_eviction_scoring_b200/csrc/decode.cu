// One decode step of attention over the compacted cache.
//
// WAITS README (stig.sh/Dirac-Notation/A2SF), Quickstart: after init_cache
// turns the compression on, model.generate decodes from the cache the
// prefill left, i.e. from the kept rows K'[s, g, j], V'[s, g, j] of the
// compaction.  For sequence s and query head h (KV head g = h / G):
//   o[s, h] = sum_{j < len[s]} softmax_j(q[s, h] . K'[s, g, j] / sqrt(d)) V'[s, g, j]
//
// Split over the cache slots (flash-decoding): a CTA takes 256 slots of one
// (sequence, KV head) for all G query heads of the group, so every K and V
// row is read from memory once; one thread per slot forms the G logits, the
// CTA reduces them to a per-head maximum and sum and multiplies the weights
// into V (threads along the head dimension, coalesced V reads).  A second
// kernel merges the splits' (maximum, sum, weighted sum) in split order.
#include "waits_internal.cuh"

namespace waits {
namespace {

constexpr int kDecThreads = 256;   // cache slots per split
constexpr int kDecMaxG = 16;

__device__ inline float bf16_to_f32(uint16_t x) { return __uint_as_float((uint32_t)x << 16); }

template <int D>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ Kc,
    const uint16_t* __restrict__ Vc, const int32_t* __restrict__ cache_len, int Hq, int Hkv,
    int C, int nsplit, float scale_log2, float* __restrict__ part) {
  __shared__ float qs[kDecMaxG][D];
  __shared__ float pw[kDecMaxG][kDecThreads];   // weights 2^(logit - max) per head and slot
  __shared__ float red[kDecThreads / 32][kDecMaxG];
  __shared__ float hmax[kDecMaxG], hsum[kDecMaxG];
  pdl_allow_next();
  pdl_wait();
  const int split = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int G = Hq / Hkv;
  int n = cache_len[s];
  n = n < 0 ? 0 : (n > C ? C : n);
  const int j0 = split * kDecThreads;
  const int jn = n - j0 < kDecThreads ? n - j0 : kDecThreads;   // slots of this split
  float* out = part + (((size_t)s * Hq + (size_t)g * G) * nsplit + split) * (D + 2);
  const size_t hstride = (size_t)nsplit * (D + 2);
  if (jn <= 0) {
    // nothing to attend to in this split: an empty partial per head
    for (int i = t; i < G * (D + 2); i += kDecThreads) {
      const int h = i / (D + 2), c = i % (D + 2);
      out[h * hstride + c] = c == D ? -INFINITY : 0.f;
    }
    return;
  }
  for (int i = t; i < G * D; i += kDecThreads)
    qs[i / D][i % D] = bf16_to_f32(q[((size_t)s * Hq + (size_t)g * G + i / D) * D + i % D]);
  __syncthreads();
  // logits of this thread's slot for the G heads (log2 units)
  float lg[kDecMaxG];
  const size_t row0 = ((size_t)s * Hkv + g) * (size_t)C + j0;
  if (t < jn) {
    const uint4* kr = reinterpret_cast<const uint4*>(Kc + (row0 + t) * D);
    float acc[kDecMaxG];
#pragma unroll
    for (int h = 0; h < kDecMaxG; ++h) acc[h] = 0.f;
#pragma unroll 4
    for (int c8 = 0; c8 < D / 8; ++c8) {
      const uint4 v = __ldg(kr + c8);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      float k[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        k[2 * e] = __uint_as_float(w[e] << 16);
        k[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
      }
#pragma unroll
      for (int h = 0; h < kDecMaxG; ++h) {
        if (h < G) {
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[h] = fmaf(qs[h][c8 * 8 + e], k[e], acc[h]);
        }
      }
    }
#pragma unroll
    for (int h = 0; h < kDecMaxG; ++h) lg[h] = acc[h] * scale_log2;
  } else {
#pragma unroll
    for (int h = 0; h < kDecMaxG; ++h) lg[h] = -INFINITY;
  }
  // per-head maximum over the split, then the weights and their sum
#pragma unroll
  for (int h = 0; h < kDecMaxG; ++h) {
    if (h >= G) break;
    float m = lg[h];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[warp][h] = m;
  }
  __syncthreads();
  if (t < G) {
    float m = red[0][t];
    for (int w = 1; w < kDecThreads / 32; ++w) m = fmaxf(m, red[w][t]);
    hmax[t] = m;
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < kDecMaxG; ++h) {
    if (h >= G) break;
    const float e = t < jn ? exp2f(lg[h] - hmax[h]) : 0.f;
    pw[h][t] = e;
    float sum = e;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) red[warp][h] = sum;
  }
  __syncthreads();
  if (t < G) {
    float l = 0.f;
    for (int w = 0; w < kDecThreads / 32; ++w) l += red[w][t];
    hsum[t] = l;
  }
  __syncthreads();
  // weighted sum of V: thread (h, c) walks the split's slots along column c
  for (int i = t; i < G * D; i += kDecThreads) {
    const int h = i / D, c = i % D;
    const uint16_t* vcol = Vc + row0 * D + c;
    float acc = 0.f;
    for (int j = 0; j < jn; ++j) acc = fmaf(pw[h][j], bf16_to_f32(vcol[(size_t)j * D]), acc);
    out[h * hstride + c] = acc;
  }
  if (t < G) {
    out[t * hstride + D] = hmax[t];
    out[t * hstride + D + 1] = hsum[t];
  }
}

// Merge the splits of (sequence, head): o = sum_i o_i 2^(m_i - M) / L with
// M = max_i m_i, L = sum_i l_i 2^(m_i - M); lse = (M + log2 L) ln 2.
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const float* __restrict__ part,
                                                           int Hq, int nsplit,
                                                           float* __restrict__ out,
                                                           float* __restrict__ lse) {
  pdl_allow_next();
  pdl_wait();
  const int h = blockIdx.x, s = blockIdx.y, c = threadIdx.x;
  const float* p = part + ((size_t)s * Hq + h) * (size_t)nsplit * (D + 2);
  float M = -INFINITY;
  for (int i = 0; i < nsplit; ++i)
    if (p[i * (D + 2) + D + 1] > 0.f) M = fmaxf(M, p[i * (D + 2) + D]);
  float L = 0.f, acc = 0.f;
  for (int i = 0; i < nsplit; ++i) {
    const float l = p[i * (D + 2) + D + 1];
    if (!(l > 0.f)) continue;
    const float f = exp2f(p[i * (D + 2) + D] - M);
    L = fmaf(l, f, L);
    acc = fmaf(p[i * (D + 2) + c], f, acc);
  }
  const size_t o = ((size_t)s * Hq + h) * D + c;
  out[o] = L > 0.f ? acc / L : 0.f;
  if (lse && c == 0)
    lse[(size_t)s * Hq + h] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

template <int D>
cudaError_t launch_decode_d(int nseq, int Hq, int Hkv, int C, const uint16_t* q,
                            const uint16_t* Kc, const uint16_t* Vc, const int32_t* len,
                            float* out, float* lse, float* part, cudaStream_t st) {
  const int nsplit = (C + kDecThreads - 1) / kDecThreads;
  const float scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  cudaError_t err = launch_pdl(decode_split_kernel<D>, dim3(nsplit, Hkv, nseq), dim3(kDecThreads),
                               0, st, q, Kc, Vc, len, Hq, Hkv, C, nsplit, scale_log2, part);
  if (err != cudaSuccess) return err;
  return launch_pdl(decode_combine_kernel<D>, dim3(Hq, nseq), dim3(D), 0, st,
                    (const float*)part, Hq, nsplit, out, lse);
}

}  // namespace

size_t decode_workspace_bytes(int64_t nseq, int64_t Hq, int64_t d, int64_t C) {
  const int64_t nsplit = (C + kDecThreads - 1) / kDecThreads;
  return (size_t)(nseq * Hq * nsplit * (d + 2)) * sizeof(float);
}

int decode_max_group() { return kDecMaxG; }

cudaError_t launch_decode(int nseq, int Hq, int Hkv, int d, int C, const uint16_t* q,
                          const uint16_t* Kc, const uint16_t* Vc, const int32_t* len, float* out,
                          float* lse, float* part, cudaStream_t st) {
  return d == 64 ? launch_decode_d<64>(nseq, Hq, Hkv, C, q, Kc, Vc, len, out, lse, part, st)
                 : launch_decode_d<128>(nseq, Hq, Hkv, C, q, Kc, Vc, len, out, lse, part, st);
}

}  // namespace waits
