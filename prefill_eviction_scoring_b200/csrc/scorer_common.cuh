// Pieces shared by the WAITS scorer kernels (score_tc.cu: every plan;
// score_sparse.cu: the small plans of the sparse-weight regime): thread
// roles and register split, the epilogue arithmetic (exponential sums over
// a TMEM row of accumulators, the FMA-pipe 2^x), the merge of pass-1 row
// partials into pass-2 row biases, the in-CTA work plan, and the TMA tensor
// maps of the packed Q and K tensors.
#pragma once

#include "plan_core.cuh"
#include "sm100.cuh"
#include "unit_iter.cuh"

namespace waits {
namespace scorer {

using namespace sm100;

constexpr int kWGs = 2;                              // epilogue warpgroups
constexpr int kEpiThreads = kWGs * 128;
constexpr int kThreads = kEpiThreads + 128;          // + producer/MMA warpgroup
// Register split (setmaxnreg): launched at 168 per thread (3 warps per SM
// quadrant); the producer/MMA warpgroup drops to 104 and the two epilogue
// warpgroups rise to 200: 128*104 + 256*200 = 384*168 - 2048.  (56 for the
// copy and MMA warps made them spill in their loops; measured 1 % slower.)
constexpr int kRegsLaunch = 168;
constexpr int kRegsProducer = 104;
constexpr int kRegsEpilogue = 200;
static_assert(128 * kRegsProducer + kEpiThreads * kRegsEpilogue <= kThreads * kRegsLaunch,
              "register split exceeds the launch allocation");
constexpr int kProducerWarp = kWGs * 4;
constexpr int kMmaWarp = kProducerWarp + 1;
constexpr int kTmemCols = 512;
constexpr uint64_t kDoneLimitNs = 2000000000ull;   // 2 s for the MMAs a CTA issued
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 0.2 s after an abort
constexpr int kBarAll = 3;                           // named barrier of both epilogue WGs

__device__ inline float u2f(uint32_t v) { return __uint_as_float(v); }

// ------------------------------------------------------------ epilogue ---
// 128 accumulator columns of this thread's TMEM lane: the load and its wait
// in one statement, so no use of the registers can be scheduled before the
// data has arrived and the registers need no read-write operands (which can
// cost a copy of each).
struct Cols {
  uint32_t r[128];
  __device__ void load_wait(uint32_t taddr) {
#define W8(b) "=r"(r[b]), "=r"(r[b + 1]), "=r"(r[b + 2]), "=r"(r[b + 3]), "=r"(r[b + 4]), \
              "=r"(r[b + 5]), "=r"(r[b + 6]), "=r"(r[b + 7])
    asm volatile(
        "{\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x128.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, %96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, %112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%128];\n\t"
        "tcgen05.wait::ld.sync.aligned;\n\t"
        "}"
        : W8(0), W8(8), W8(16), W8(24), W8(32), W8(40), W8(48), W8(56),
          W8(64), W8(72), W8(80), W8(88), W8(96), W8(104), W8(112), W8(120)
        : "r"(taddr)
        : "memory");
#undef W8
  }
};

__device__ inline float2 f2(float x, float y) { return make_float2(x, y); }
__device__ inline float hsum8(const float2 (&a)[4]) {
  const float2 s = __fadd2_rn(__fadd2_rn(a[0], a[1]), __fadd2_rn(a[2], a[3]));
  return s.x + s.y;
}

// Column pairs whose exponential runs on the FMA pipe instead of the MUFU
// (which does 16 ex2 per clock per SM and bounds the unmasked passes): bit
// (pair index mod 8) of this mask.  Three in eight measured best with the
// shift-add exponential below (an epilogue-only loop over TMEM tiles, clocks
// per 128x128 tile: pass 1 885 against 1096 with the MUFU alone, 995 with two
// in eight, 951 with four; pass 2 865, 906 with four, 999 with five).
constexpr uint32_t kPolyPairs = 0x92u;
__device__ constexpr bool poly_col(int c) { return (kPolyPairs >> ((c >> 1) & 7)) & 1u; }

// acc + 2^x for a pair of fp32 values on the FMA/ALU pipes (Cody-Waite split
// plus a polynomial): x = n + f with n = rint(x) and f in [-1/2, 1/2];
// 2^f ~ 1 + f (c1 + f (c2 + f c3)), the relative-error minimax cubic with the
// constant term held at 1 (max relative error 1.013e-4; fitted by linear
// programming on a dense grid), so integer x gives exact powers of two.
// rint comes from adding 1.5 * 2^23 + 127: the sum's low mantissa bits are
// then n + 127, so shifting its bit pattern left by 23 leaves exactly the
// fp32 pattern of 2^n (the magic's own bits above bit 8 shift out); the
// product with the cubic is fused into the running sum.  x is raised to at
// least -127, whose pattern is +0, so x <= -126.5 adds nothing (as the MUFU's
// flush to zero does below 2^-126).  Valid for x <= 127: every argument the
// epilogue forms is at most 0 up to rounding (a logit minus the row maximum,
// or a bias that includes the row's log-sum-exp).
__device__ inline float2 exp2_poly_acc(float2 x, float2 acc) {
  constexpr float kMagic = 12582912.0f + 127.0f;     // exact in fp32
  constexpr float c1 = 0.69328290f, c2 = 0.24221097f, c3 = 0.05500906f;
  x = f2(fmaxf(x.x, -127.f), fmaxf(x.y, -127.f));
  const float2 t = __fadd2_rn(x, f2(kMagic, kMagic));
  const float2 n = __fadd2_rn(t, f2(-kMagic, -kMagic));
  const float2 fr = __ffma2_rn(n, f2(-1.f, -1.f), x);
  float2 q = __ffma2_rn(f2(c3, c3), fr, f2(c2, c2));
  q = __ffma2_rn(q, fr, f2(c1, c1));
  q = __ffma2_rn(q, fr, f2(1.f, 1.f));
  const float2 p = f2(__int_as_float(__float_as_int(t.x) << 23),
                      __int_as_float(__float_as_int(t.y) << 23));
  return __ffma2_rn(q, p, acc);
}

// acc + 2^x for a column pair: the polynomial for the pairs of kPolyPairs,
// else the MUFU.
__device__ inline float2 exp2_add(int c, float2 x, float2 acc) {
  return poly_col(c) ? exp2_poly_acc(x, acc)
                     : __fadd2_rn(acc, f2(ex2_approx(x.x), ex2_approx(x.y)));
}

// sum_c 2^(v_c * sc + off) over all 128 columns, packed fp32x2 arithmetic.
__device__ inline float exp_sum_full(const Cols& v, float sc, float off) {
  const float2 sc2 = f2(sc, sc), off2 = f2(off, off);
  float2 a[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) a[k] = f2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < kTile; c += 2) {
    const float2 x = __ffma2_rn(f2(u2f(v.r[c]), u2f(v.r[c + 1])), sc2, off2);
    a[(c >> 1) & 3] = exp2_add(c, x, a[(c >> 1) & 3]);
  }
  return hsum8(a);
}

// Largest of the tile's first nv values, scaled.
__device__ inline float tile_max(const Cols& v, int nv, float sc) {
  float mx = -INFINITY;
#pragma unroll
  for (int c = 0; c < kTile; ++c) mx = fmaxf(mx, c < nv ? u2f(v.r[c]) * sc : -INFINITY);
  return mx;
}

// sum over c < nv of 2^(v_c*sc + off) (masked tiles, MUFU only: exact zeros)
__device__ inline float exp_sum_masked(const Cols& v, int nv, float sc, float off) {
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = 0.f;
#pragma unroll
  for (int c = 0; c < kTile; ++c) {
    const float x = fmaf(u2f(v.r[c]), sc, off);
    a[c & 7] += ex2_approx(c < nv ? x : -INFINITY);
  }
  return ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
}

// max(a, b, c) in one instruction (the three-input form sm_100 has).
__device__ inline float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Largest raw value of the whole tile (8 independent chains of three-input
// maxima).
__device__ inline float tile_max_raw(const Cols& v) {
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = u2f(v.r[k]);
#pragma unroll
  for (int c = 8; c < kTile; c += 2) mx[(c >> 1) & 7] = fmax3(mx[(c >> 1) & 7], u2f(v.r[c]), u2f(v.r[c + 1]));
  return fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
}

// Pass 1, one 128-key tile of this thread's row (keys c < nv are causal):
// l += sum_c 2^(v_c*scale2 - m) after moving the reference m up to the
// tile's maximum when that is higher (rescaling l), so no term exceeds 1 and
// the sum cannot overflow.  A masked tile takes the maximum of its causal
// values only.
__device__ inline void p1_pair(const Cols& v, int nv, float sc, float& m, float& l) {
  // one path per warp: a warp whose rows are not all fully causal (or absent)
  // takes the masked path, which also serves its full rows
  const bool full_warp = __all_sync(0xffffffffu, nv == kTile || nv <= 0);
  if (nv <= 0) return;
  const float mx = full_warp ? tile_max_raw(v) * sc : tile_max(v, nv, sc);
  if (mx > m) {
    if (l > 0.f) l *= ex2_approx(m - mx);
    m = mx;
  }
  float t;
  if (full_warp) {
    t = exp_sum_full(v, sc, -m);
  } else {
    t = exp_sum_masked(v, nv, sc, -m);
  }
  l += t;
}

// Pass 2, one 128-row Q tile for this thread's key: sum over columns
// c in [c_lo, ncols) of 2^(v_c*scale2 + bias_c) (bias is -inf past the rows).
__device__ inline float p2_pair(const Cols& v, int c_lo, int ncols, float sc, const float* bias) {
  const float4* b4 = reinterpret_cast<const float4*>(bias);
  if (__all_sync(0xffffffffu, c_lo == 0)) {   // one path per warp
    const float2 sc2 = f2(sc, sc);
    float2 a[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) a[k] = f2(0.f, 0.f);
#pragma unroll
    for (int cb = 0; cb < kTile; cb += 32) {
      if (cb < ncols) {
#pragma unroll
        for (int c = cb; c < cb + 32; c += 4) {
          const float4 b = b4[c / 4];
          const float2 x0 = __ffma2_rn(f2(u2f(v.r[c]), u2f(v.r[c + 1])), sc2, f2(b.x, b.y));
          const float2 x1 = __ffma2_rn(f2(u2f(v.r[c + 2]), u2f(v.r[c + 3])), sc2, f2(b.z, b.w));
          a[(c >> 1) & 3] = exp2_add(c, x0, a[(c >> 1) & 3]);
          a[((c >> 1) + 1) & 3] = exp2_add(c + 2, x1, a[((c >> 1) + 1) & 3]);
        }
      }
    }
    return hsum8(a);
  }
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = 0.f;
#pragma unroll
  for (int cb = 0; cb < kTile; cb += 32) {
    if (cb < ncols) {
#pragma unroll
      for (int c = cb; c < cb + 32; c += 4) {
        const float4 b = b4[c / 4];
        const float x0 = fmaf(u2f(v.r[c + 0]), sc, b.x);
        const float x1 = fmaf(u2f(v.r[c + 1]), sc, b.y);
        const float x2 = fmaf(u2f(v.r[c + 2]), sc, b.z);
        const float x3 = fmaf(u2f(v.r[c + 3]), sc, b.w);
        a[(c + 0) & 7] += ex2_approx(c + 0 >= c_lo ? x0 : -INFINITY);
        a[(c + 1) & 7] += ex2_approx(c + 1 >= c_lo ? x1 : -INFINITY);
        a[(c + 2) & 7] += ex2_approx(c + 2 >= c_lo ? x2 : -INFINITY);
        a[(c + 3) & 7] += ex2_approx(c + 3 >= c_lo ? x3 : -INFINITY);
      }
    }
  }
  return ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
}

__device__ inline void bar_sync(int id, int n) {
  __syncwarp();
  named_bar_sync(id, n);
}
// Named barrier that also ORs `v` over its threads (a uniform answer).
__device__ inline bool bar_vote_or(int id, int n, bool v) {
  __syncwarp();
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// Merge two (reference max, sum) pairs of the same row.
__device__ inline float2 lse_merge(float2 x, float2 y) {
  if (!(y.y > 0.f)) return x;
  if (!(x.y > 0.f)) return y;
  const float M = fmaxf(x.x, y.x);
  return make_float2(M, x.y * ex2_approx(x.x - M) + y.y * ex2_approx(y.x - M));
}

// Bias of packed row r of the Q tiles j[k] (j[k] < 0: none; -inf where no
// row exists): log2 of the row's curve weight minus its log2-sum-exp over
// the keys, from the pass-1 partials of the row's units.  The partials of
// all NR rows are loaded together (kMergeBatch units per row in flight) and
// merged in unit order as a maximum, then a sum of the rescaled partial sums.
// Row r's bias of Q tile j, already merged by row_bias_kernel: one load.
__device__ inline float merged_bias(const PassArgs& p, const Entry* e1, const SeqInfo& si, int g,
                                    int j, int r) {
  const int ngrp = (si.nqt + kMaxStat1 - 1) / kMaxStat1;
  const Entry& e = e1[si.e1 + g * ngrp + j / kMaxStat1];
  return __ldcg(&p.part1[((size_t)e.unit_base * kMaxStat1 + j % kMaxStat1) * kTile + r].x);
}

template <int NR>
__device__ inline void qrow_bias(const PassArgs& p, const Entry* e1, const SeqInfo& si, int g,
                                 const int (&j)[NR], int r, float (&out)[NR]) {
  if (p.bias_ready) {
#pragma unroll
    for (int k = 0; k < NR; ++k) out[k] = j[k] >= 0 ? merged_bias(p, e1, si, g, j[k], r) : -INFINITY;
    return;
  }
  if (p.lse) {
    // the caller's natural-log row LSE replaces pass 1: log2 w - lse * log2(e)
    constexpr float kLog2e = 1.4426950408889634f;
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      const int tok = si.q0 + j[k] * p.tokq + r / p.G;
      const bool row = j[k] >= 0 && r < p.tokq * p.G && tok < si.len;
      const float w = row ? curve_weight(tok, si.len, si.a, si.b) : 0.f;
      const size_t h = (size_t)g * p.G + r % p.G;
      out[k] = w > 0.f ? log2f(w) - p.lse[h * p.T + si.start + tok] * kLog2e : -INFINITY;
    }
    return;
  }
  constexpr size_t kStride = (size_t)kMaxStat1 * kTile;
  constexpr int kMergeBatch = 16;
  const int ngrp = (si.nqt + kMaxStat1 - 1) / kMaxStat1;     // pass-1 groups per head
  const float2* src[NR];
  int nu[NR], tok[NR], numax = 0;
#pragma unroll
  for (int k = 0; k < NR; ++k) {
    tok[k] = si.q0 + j[k] * p.tokq + r / p.G;
    nu[k] = 0;
    src[k] = p.part1;
    if (j[k] >= 0 && r < p.tokq * p.G && tok[k] < si.len) {
      const Entry& e = e1[si.e1 + g * ngrp + j[k] / kMaxStat1];
      src[k] = p.part1 + ((size_t)e.unit_base * kMaxStat1 + j[k] % kMaxStat1) * kTile + r;
      nu[k] = e.n_units;
    }
    numax = max(numax, nu[k]);
  }
  float2 acc[NR];
#pragma unroll
  for (int k = 0; k < NR; ++k) acc[k] = make_float2(-INFINITY, 0.f);
  for (int u0 = 0; u0 < numax; u0 += kMergeBatch) {
    float2 x[NR][kMergeBatch];
#pragma unroll
    for (int k = 0; k < NR; ++k)
#pragma unroll
      for (int b = 0; b < kMergeBatch; ++b)
        x[k][b] = u0 + b < nu[k] ? __ldcg(src[k] + (size_t)(u0 + b) * kStride)
                                 : make_float2(-INFINITY, 0.f);
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      float M = acc[k].x;
#pragma unroll
      for (int b = 0; b < kMergeBatch; ++b)
        if (x[k][b].y > 0.f) M = fmaxf(M, x[k][b].x);
      float L = acc[k].y > 0.f ? acc[k].y * ex2_approx(acc[k].x - M) : 0.f;
#pragma unroll
      for (int b = 0; b < kMergeBatch; ++b)
        if (x[k][b].y > 0.f) L += x[k][b].y * ex2_approx(x[k][b].x - M);
      acc[k] = make_float2(M, L);
    }
  }
#pragma unroll
  for (int k = 0; k < NR; ++k) {
    const float w = nu[k] > 0 ? curve_weight(tok[k], si.len, si.a, si.b) : 0.f;
    out[k] = w > 0.f ? log2f(w) - (acc[k].x + log2f(acc[k].y)) : -INFINITY;
  }
}

// The same, with the pass-1 entries of the plan `p` points at.
template <int NR>
__device__ inline void qrow_bias(const PassArgs& p, const SeqInfo& si, int g, const int (&j)[NR],
                                 int r, float (&out)[NR]) {
  qrow_bias<NR>(p, p.e1, si, g, j, r, out);
}

// The host's one-sequence plan into this CTA's shared memory.  It is a
// kernel parameter, so this runs before the wait for the previous kernel;
// plan_prologue then only checks cu_seqlens and writes the header.
__device__ inline void stage_host_plan(const PassArgs& pa, const HostPlan& hp, LocalPlan* lp) {
  if (!pa.local_plan || !pa.host_plan) return;
  constexpr int kVecs = (int)(sizeof(Entry) / sizeof(uint4));
  const int n1 = hp.hdr.n_e1, n2 = hp.hdr.n_e2;
  const uint4* h1 = reinterpret_cast<const uint4*>(hp.e1);
  const uint4* h2 = reinterpret_cast<const uint4*>(hp.e2);
  uint4* d1 = reinterpret_cast<uint4*>(lp->e1);
  uint4* d2 = reinterpret_cast<uint4*>(lp->e2);
  for (int i = threadIdx.x; i < (n1 + n2) * kVecs; i += blockDim.x) {
    if (i < n1 * kVecs) d1[i] = h1[i];
    else d2[i - n1 * kVecs] = h2[i - n1 * kVecs];
  }
  if (threadIdx.x == 0) lp->seqs[0] = hp.seq;
}

// Every CTA's share of the plan: with a local plan each CTA builds it in
// shared memory (or takes the host's one-sequence plan, staged before the
// wait) and points `p` at it; pass 1 also resets the call's status word and
// zeroes the scores of sequences without an active row.  Called by all
// threads of the CTA.
__device__ inline void plan_prologue(PassArgs& p, const PassArgs& pa, const HostPlan& hp,
                                     LocalPlan* lp, bool p1, int warp) {
  if (p.local_plan) {
    // every CTA plans for itself (cu_seqlens is complete: pass 1 has waited
    // above, and pass 2 starts only after pass 1 has), or copies the plan
    // the host built for the batch {0, T} once cu_seqlens reads so
    if (p.host_plan) {
      // the entries are already in shared memory (stage_host_plan, before
      // the wait); a plan is only used if cu_seqlens reads {0, T}
      const bool valid = p.cu[0] == 0 && p.cu[1] == p.T;   // the same two words in every thread
      if (threadIdx.x == 0) {
        PlanHeader h = hp.hdr;
        if (!valid) {
          h = PlanHeader{};
          h.status = WAITS_DEV_BAD_SEQLENS;
        }
        lp->hdr = h;
      }
    } else if (warp == 0) {
      warp_plan(p.cu, p.nseq, p.T, p.max_seqlen, p.Hkv, p.tokq, p.a, p.b, (int)gridDim.x, !p1,
                *lp);
    }
    __syncthreads();
    p.hdr = &lp->hdr;
    p.seqs = lp->seqs;
    p.e1 = lp->e1;
    p.e2 = lp->e2;
    if (p1 || pa.lse) {
      // this call's device status word, and zero scores for sequences
      // without an active row (the planner kernel's duties), in the first
      // pass the call runs
      if (blockIdx.x == 0 && threadIdx.x == 0) *pa.status = lp->hdr.status;
      if (lp->hdr.status == 0) {
        const int64_t stride = (int64_t)gridDim.x * blockDim.x;
        for (int q = 0; q < p.nseq; ++q) {
          const SeqInfo si = lp->seqs[q];
          if (si.len == 0 || si.q0 < si.len) continue;
          for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
               i < (int64_t)si.len * p.Hkv; i += stride)
            p.scores[(i / si.len) * p.T + si.start + i % si.len] = 0.0f;
        }
      }
    }
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 3-D view [T][heads][d] of a packed bf16 tensor; box = 64 x box_h x box_t.
inline bool make_map(CUtensorMap* m, const void* base, int T, int heads, int row_heads, int d,
                     int box_h, int box_t) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  // `heads` heads of each token row are addressed; a row holds `row_heads`
  // (more when the call covers a range of the layer's heads)
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)row_heads * d * 2};
  const cuuint32_t box[3] = {64u, (cuuint32_t)box_h, (cuuint32_t)box_t};
  const cuuint32_t elem[3] = {1u, 1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}


}  // namespace scorer
}  // namespace waits
