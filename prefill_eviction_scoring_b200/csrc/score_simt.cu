// Two-pass WAITS scorer on the CUDA cores (fp32 FMA dot products).
//
// Pass 1 computes, for every active query row, log2 of its causal softmax
// normaliser and folds it with log2 w[q] into one per-row bias.  Pass 2
// recomputes the logits and sums w[q] * P[q, k] = 2^(logit*log2e/sqrt(d) +
// bias[q]) over rows q >= k and over the query heads of the KV group (WAITS
// README, opening summary: accumulative attention score weighted by the
// forgetting curve).  Work follows the device plan: each unit holds up to
// four stationary tiles and streams the other operand's tiles.
#include "unit_iter.cuh"

namespace waits {
namespace {

constexpr int kThreads = 128;

__device__ inline float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ inline float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Copy Q tile j (tokq tokens x G heads) of (sequence, KV group g) into smem
// rows of stride RS elements; rows past the sequence or the tile are zero.
template <int D, int RS>
__device__ void load_qtile(uint16_t* dst, const PassArgs& p, const SeqInfo& si, int g, int j) {
  constexpr int CH = D / 8;
  for (int i = threadIdx.x; i < kTile * CH; i += kThreads) {
    const int r = i / CH, c = i % CH;
    const int tok = si.q0 + j * p.tokq + r / p.G;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < p.tokq * p.G && tok < si.len) {
      const size_t row = ((size_t)(si.start + tok) * p.Hq + (size_t)g * p.G + r % p.G) * D;
      v = *reinterpret_cast<const uint4*>(p.Q + row + c * 8);
    }
    *reinterpret_cast<uint4*>(dst + r * RS + c * 8) = v;
  }
}

template <int D, int RS>
__device__ void load_ktile(uint16_t* dst, const PassArgs& p, const SeqInfo& si, int g, int kt) {
  constexpr int CH = D / 8;
  for (int i = threadIdx.x; i < kTile * CH; i += kThreads) {
    const int r = i / CH, c = i % CH;
    const int key = kt * kTile + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (key < si.len) {
      const size_t row = ((size_t)(si.start + key) * p.Hkv + g) * D;
      v = *reinterpret_cast<const uint4*>(p.K + row + c * 8);
    }
    *reinterpret_cast<uint4*>(dst + r * RS + c * 8) = v;
  }
}

// Bias of the 128 packed rows of Q tile j; -inf where no row exists.
__device__ void load_qbias(float* dst, const PassArgs& p, const SeqInfo& si, int g, int j) {
  const int r = threadIdx.x;
  const int tok = si.q0 + j * p.tokq + r / p.G;
  float v = -INFINITY;
  if (r < p.tokq * p.G && tok < si.len)
    v = p.bias[((size_t)g * p.T + si.start + si.q0 + (size_t)j * p.tokq) * p.G + r];
  dst[r] = v;
}

// dots[c] = own . bcast[c] for the 128 rows of the broadcast tile.
template <int D, int RS>
__device__ void tile_dots(const uint16_t* own_row, const uint16_t* bcast, float* dots) {
  uint32_t own[D / 2];
#pragma unroll
  for (int k = 0; k < D / 8; ++k) {
    const uint4 v = *reinterpret_cast<const uint4*>(own_row + k * 8);
    own[4 * k + 0] = v.x; own[4 * k + 1] = v.y; own[4 * k + 2] = v.z; own[4 * k + 3] = v.w;
  }
#pragma unroll 4
  for (int c = 0; c < kTile; ++c) {
    const uint16_t* row = bcast + c * RS;
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int k = 0; k < D / 8; ++k) {
      const uint4 v = *reinterpret_cast<const uint4*>(row + k * 8);
      acc0 = fmaf(bf16_lo(own[4 * k + 0]), bf16_lo(v.x), acc0);
      acc1 = fmaf(bf16_hi(own[4 * k + 0]), bf16_hi(v.x), acc1);
      acc0 = fmaf(bf16_lo(own[4 * k + 1]), bf16_lo(v.y), acc0);
      acc1 = fmaf(bf16_hi(own[4 * k + 1]), bf16_hi(v.y), acc1);
      acc0 = fmaf(bf16_lo(own[4 * k + 2]), bf16_lo(v.z), acc0);
      acc1 = fmaf(bf16_hi(own[4 * k + 2]), bf16_hi(v.z), acc1);
      acc0 = fmaf(bf16_lo(own[4 * k + 3]), bf16_lo(v.w), acc0);
      acc1 = fmaf(bf16_hi(own[4 * k + 3]), bf16_hi(v.w), acc1);
    }
    dots[c] = acc0 + acc1;
  }
}

// Merge the per-unit (reference max, sum) partials of one row and write its
// bias = log2 w[q] - log2 sum_k 2^(x_k).
__device__ void finish_row(const PassArgs& p, const SeqInfo& si, int g, int j, int r,
                           const float2* parts, int nparts, int stride) {
  const int tok = si.q0 + j * p.tokq + r / p.G;
  if (r >= p.tokq * p.G || tok >= si.len) return;
  float M = -INFINITY;
  for (int u = 0; u < nparts; ++u) {
    const float2 v = __ldcg(parts + (size_t)u * stride);
    if (v.y > 0.f) M = fmaxf(M, v.x);
  }
  float L = 0.f;
  for (int u = 0; u < nparts; ++u) {
    const float2 v = __ldcg(parts + (size_t)u * stride);
    if (v.y > 0.f) L += v.y * ex2_approx(v.x - M);
  }
  const float lse2 = M + log2f(L);
  const float w = curve_weight(tok, si.len, p.a, p.b);
  const float bias = w > 0.f ? log2f(w) - lse2 : -INFINITY;
  p.bias[((size_t)g * p.T + si.start + tok) * p.G + r % p.G] = bias;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) pass_simt_kernel(PassArgs p, int pass) {
  constexpr int RS = D + 8;
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* stat = reinterpret_cast<uint16_t*>(smem);
  uint16_t* strm = stat + kMaxStat * kTile * RS;
  float* sbias = reinterpret_cast<float*>(strm + kTile * RS);   // [4][128]
  __shared__ int s_last;
  const int t = threadIdx.x;
  const PlanHeader* H = p.hdr;
  const bool p1 = pass == 1;
  const Entry* E = p1 ? p.e1 : p.e2;
  UnitIter it;
  if (!it.init(E, p1 ? H->n_e1 : H->n_e2, p1 ? H->s1 : H->s2, p1 ? H->p1 : H->p2, blockIdx.x))
    return;

  float dots[kTile];
  int ei, st0, st1, unit;
  while (it.next(ei, st0, st1, unit)) {
    const Entry e = E[ei];
    const SeqInfo si = p.seqs[e.seq];
    const int g = e.g;
    // stationary tiles
    for (int i = 0; i < e.n_stat; ++i) {
      if (e.mode == kModeP2K) load_ktile<D, RS>(stat + i * kTile * RS, p, si, g, e.stat0 + i);
      else load_qtile<D, RS>(stat + i * kTile * RS, p, si, g, e.stat0 + i);
      if (e.mode == kModeP2Q) load_qbias(sbias + i * kTile, p, si, g, e.stat0 + i);
    }
    float mref[kMaxStat], lsum[kMaxStat], acc[kMaxStat];
#pragma unroll
    for (int i = 0; i < kMaxStat; ++i) { mref[i] = -INFINITY; lsum[i] = 0.f; acc[i] = 0.f; }
    __syncthreads();

    for (int st = st0; st < st1; ++st) {
      const int o = e.step0 + st;   // streamed tile index
      if (e.mode == kModeP2K) {
        load_qtile<D, RS>(strm, p, si, g, o);
        load_qbias(sbias, p, si, g, o);
      } else {
        load_ktile<D, RS>(strm, p, si, g, o);
      }
      __syncthreads();
      float col = 0.f;   // P2Q: this key's sum over the stationary Q tiles
      for (int i = 0; i < e.n_stat; ++i) {
        const int j = e.mode == kModeP2K ? o : e.stat0 + i;
        const int kt = e.mode == kModeP2K ? e.stat0 + i : o;
        if (!pair_live(si, j, kt, p.tokq)) continue;
        if (e.mode == kModeP1) {
          // thread t = packed row t of Q tile j; columns = keys of tile kt
          tile_dots<D, RS>(stat + (i * kTile + t) * RS, strm, dots);
          const int tok = si.q0 + j * p.tokq + t / p.G;
          if (t < p.tokq * p.G && tok < si.len) {
            int nv = tok - kt * kTile + 1;
            nv = nv > kTile ? kTile : nv;
            if (nv > 0) {
              if (mref[i] == -INFINITY) {
                float mx = -INFINITY;
                for (int c = 0; c < nv; ++c) mx = fmaxf(mx, dots[c] * p.scale2);
                mref[i] = mx;
              }
              float s = 0.f;
              for (int c = 0; c < nv; ++c) s += ex2_approx(fmaf(dots[c], p.scale2, -mref[i]));
              const float ln = lsum[i] + s;
              if (ln <= kRebaseLimit) {
                lsum[i] = ln;
              } else {
                float mx = mref[i];
                for (int c = 0; c < nv; ++c) mx = fmaxf(mx, dots[c] * p.scale2);
                float s2 = 0.f;
                for (int c = 0; c < nv; ++c) s2 += ex2_approx(fmaf(dots[c], p.scale2, -mx));
                lsum[i] = lsum[i] * ex2_approx(mref[i] - mx) + s2;
                mref[i] = mx;
              }
            }
          }
        } else {
          // thread t = key t of tile kt; columns = packed rows of Q tile j
          const uint16_t* own = e.mode == kModeP2K ? stat + (i * kTile + t) * RS : strm + t * RS;
          const uint16_t* bc = e.mode == kModeP2K ? strm : stat + i * kTile * RS;
          const float* bias = e.mode == kModeP2K ? sbias : sbias + i * kTile;
          tile_dots<D, RS>(own, bc, dots);
          const int key = kt * kTile + t;
          const int f = si.q0 + j * p.tokq;
          float s = 0.f;
          for (int c = 0; c < kTile; ++c) {
            const bool ok = (f + c / p.G) >= key;   // bias is -inf past the rows
            const float v = ex2_approx(fmaf(dots[c], p.scale2, bias[c]));
            s += ok ? v : 0.f;
          }
          if (e.mode == kModeP2K) acc[i] += s; else col += s;
        }
      }
      if (e.mode == kModeP2Q) {
        const int key = o * kTile + t;
        if (key < si.len) p.scores[(size_t)g * p.T + si.start + key] = col;
      }
      __syncthreads();
    }

    // ---- unit results
    if (e.mode == kModeP1) {
      if (e.n_units == 1) {
        for (int i = 0; i < e.n_stat; ++i) {
          const float2 v = make_float2(mref[i], lsum[i]);
          // a single partial: finish directly from registers
          const int j = e.stat0 + i;
          const int tok = si.q0 + j * p.tokq + t / p.G;
          if (t < p.tokq * p.G && tok < si.len) {
            const float lse2 = v.x + log2f(v.y);
            const float w = curve_weight(tok, si.len, p.a, p.b);
            p.bias[((size_t)g * p.T + si.start + tok) * p.G + t % p.G] =
                w > 0.f ? log2f(w) - lse2 : -INFINITY;
          }
        }
      } else {
        for (int i = 0; i < e.n_stat; ++i)
          p.part1[((size_t)unit * kMaxStat + i) * kTile + t] = make_float2(mref[i], lsum[i]);
        __threadfence();
        __syncthreads();
        if (t == 0) s_last = atomicAdd(&p.c1[ei], 1u) == (uint32_t)(e.n_units - 1);
        __syncthreads();
        if (s_last) {
          __threadfence();
          for (int i = 0; i < e.n_stat; ++i)
            finish_row(p, si, g, e.stat0 + i, t,
                       p.part1 + ((size_t)e.unit_base * kMaxStat + i) * kTile + t,
                       e.n_units, kMaxStat * kTile);
        }
      }
    } else if (e.mode == kModeP2K) {
      if (e.n_units == 1) {
        for (int i = 0; i < e.n_stat; ++i) {
          const int key = (e.stat0 + i) * kTile + t;
          if (key < si.len) p.scores[(size_t)g * p.T + si.start + key] = acc[i];
        }
      } else {
        for (int i = 0; i < e.n_stat; ++i)
          p.part2[((size_t)unit * kMaxStat + i) * kTile + t] = acc[i];
        __threadfence();
        __syncthreads();
        if (t == 0) s_last = atomicAdd(&p.c2[ei], 1u) == (uint32_t)(e.n_units - 1);
        __syncthreads();
        if (s_last) {
          __threadfence();
          for (int i = 0; i < e.n_stat; ++i) {
            const int key = (e.stat0 + i) * kTile + t;
            float s = 0.f;
            for (int u = 0; u < e.n_units; ++u)
              s += __ldcg(p.part2 + ((size_t)(e.unit_base + u) * kMaxStat + i) * kTile + t);
            if (key < si.len) p.scores[(size_t)g * p.T + si.start + key] = s;
          }
        }
      }
    }
    __syncthreads();
  }
}

template <int D>
cudaError_t launch_d(const PassArgs& a, int grid, cudaStream_t s) {
  constexpr int RS = D + 8;
  const size_t smem = (size_t)(kMaxStat + 1) * kTile * RS * sizeof(uint16_t) +
                      kMaxStat * kTile * sizeof(float);
  cudaError_t err = cudaFuncSetAttribute(pass_simt_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  pass_simt_kernel<D><<<grid, kThreads, smem, s>>>(a, 1);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  pass_simt_kernel<D><<<grid, kThreads, smem, s>>>(a, 2);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_passes(const PassArgs& a, int grid, cudaStream_t s) {
  return a.d == 64 ? launch_d<64>(a, grid, s) : launch_d<128>(a, grid, s);
}

}  // namespace waits
