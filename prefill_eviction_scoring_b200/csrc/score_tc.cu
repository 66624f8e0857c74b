// Two-pass WAITS scorer on the sm_100a tensor cores.
//
// WAITS README (stig.sh/Dirac-Notation/A2SF), opening summary: the score of
// key k is the accumulative attention it receives, each query row q weighted
// by the forgetting curve w[q].  Read as causal softmax(QK^T / sqrt(d)) summed
// over the query heads of a KV group:
//   pass 1  per row (q, h): sum_{k<=q} 2^(x[q,k]), x = (Q.K) * log2(e) / sqrt(d),
//           as (reference max, sum) partials of the CTAs sharing the row
//   pass 2  bias[q,h] = log2 w[q] - log2 of the merged sum, then
//           s[g,k]    = sum_{h in g} sum_{q>=k} 2^(x[q,k] + bias[q,h])
// Rows whose fp32 weight is exactly 0 are never visited (the planner starts
// each sequence at its first non-zero row).
//
// Per CTA (persistent, one per SM): warp 4 streams tiles with TMA into
// 128-byte-swizzled shared memory, warp 5 issues tcgen05.mma (bf16 in, fp32
// accumulators in tensor memory, 128x128 per tile pair, four TMEM buffers),
// warps 0-3 read the accumulators with tcgen05.ld and do the exp / reduction
// work, one TMEM lane per thread.  Pass 1 puts query rows in the lanes (row
// statistics stay in a thread); pass 2 puts keys in the lanes (column sums
// stay in a thread), so neither pass needs a cross-thread reduction.
// Every wait is bounded; a timeout sets WAITS_DEV_TIMEOUT and the CTA exits
// after its copies and MMAs in flight have landed.
#include "plan_core.cuh"
#include "sm100.cuh"
#include "unit_iter.cuh"

namespace waits {
namespace {

using namespace sm100;

constexpr int kWGs = 2;                              // epilogue warpgroups
constexpr int kEpiThreads = kWGs * 128;
constexpr int kThreads = kEpiThreads + 128;          // + producer/MMA warpgroup
// Register split (setmaxnreg): launched at 168 per thread (3 warps per SM
// quadrant); the producer/MMA warpgroup drops to 56 and the two epilogue
// warpgroups rise to 224: 128*56 + 256*224 = 384*168.
constexpr int kRegsLaunch = 168;
constexpr int kRegsProducer = 56;
constexpr int kRegsEpilogue = 224;
static_assert(128 * kRegsProducer + kEpiThreads * kRegsEpilogue <= kThreads * kRegsLaunch,
              "register split exceeds the launch allocation");
constexpr int kProducerWarp = kWGs * 4;
constexpr int kMmaWarp = kProducerWarp + 1;
constexpr int kTmemBufs = 2 * kWGs;                  // two 128-column buffers per WG
constexpr int kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 0.2 s after an abort
constexpr int kBarWG0 = 1;                           // named barriers: 1, 2 per WG,
constexpr int kBarAll = 3;                           // 3 for both WGs

// Shared-memory plan per head dim and pass: pass 1 holds 2 stationary Q
// tiles and streams K through 4 stages (d = 128); pass 2 holds up to 4
// stationary tiles with 2 stages.
template <int D, int PASS>
struct Cfg {
  static constexpr int kSub = D / 64;                    // 128-byte column blocks
  static constexpr int kSubBytes = kTile * 128;          // 16 KB
  static constexpr int kTileBytes = kSub * kSubBytes;
  static constexpr int kStat = PASS == 1 ? kMaxStat1 : kMaxStat;
  static constexpr int kStages = (D == 128 ? 2 : 4) * (PASS == 1 ? 2 : 1);
  static constexpr int kKSteps = D / 16;
  static constexpr size_t kFloats = kMaxStat * kTile            // stationary Q biases
                                    + kWGs * 2 * kTile           // streamed Q biases
                                    + 2 * kWGs * kMaxStat * kTile;  // per-WG state
  static constexpr size_t kSmem = 1024 + (size_t)(kStat + kStages) * kTileBytes +
                                  kFloats * sizeof(float) + sizeof(LocalPlan) + 256;
};

struct Smem {
  uint8_t* stat;
  uint8_t* strm;
  float* bias_stat;  // [4][128]
  float* bias_strm;  // [WG][2][128]
  float* st_m;       // [WG][4][128] reference max (pass 1)
  float* st_l;       // [WG][4][128] running sum (pass 1) / column sum (pass 2)
  uint64_t* full;
  uint64_t* empty;
  uint64_t* stat_full;
  uint64_t* stat_empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* done;
  LocalPlan* lp;          // the plan, when each CTA builds it
  uint32_t* tmem_slot;
  volatile int* abort;
  int* last;
};

template <int D, int PASS>
__device__ Smem carve(uint8_t* raw) {
  using C = Cfg<D, PASS>;
  Smem s;
  const uint32_t a = smem_addr(raw);
  uint8_t* base = raw + ((1024u - (a & 1023u)) & 1023u);
  s.stat = base;
  s.strm = s.stat + C::kStat * C::kTileBytes;
  s.bias_stat = reinterpret_cast<float*>(s.strm + C::kStages * C::kTileBytes);
  s.bias_strm = s.bias_stat + kMaxStat * kTile;
  s.st_m = s.bias_strm + kWGs * 2 * kTile;
  s.st_l = s.st_m + kWGs * kMaxStat * kTile;
  s.lp = reinterpret_cast<LocalPlan*>(s.st_l + kWGs * kMaxStat * kTile);
  uint64_t* bars = reinterpret_cast<uint64_t*>(s.lp + 1);
  s.full = bars;
  s.empty = s.full + C::kStages;
  s.stat_full = s.empty + C::kStages;
  s.stat_empty = s.stat_full + 1;
  s.tfull = s.stat_empty + 1;
  s.tempty = s.tfull + kTmemBufs;
  s.done = s.tempty + kTmemBufs;
  s.tmem_slot = reinterpret_cast<uint32_t*>(s.done + 1);
  s.abort = reinterpret_cast<volatile int*>(s.tmem_slot + 1);
  s.last = const_cast<int*>(s.abort) + 1;
  return s;
}

__device__ inline float u2f(uint32_t v) { return __uint_as_float(v); }

// Streamed / stationary operand kinds per mode.
__device__ inline bool stat_is_q(int mode) { return mode != kModeP2K; }

// (Q tile, K tile) of the pair (streamed tile o, stationary slot i).
__device__ inline void pair_tiles(const Entry& e, int o, int i, int& j, int& kt) {
  j = e.mode == kModeP2K ? o : e.stat0 + i;
  kt = e.mode == kModeP2K ? e.stat0 + i : o;
}

// ------------------------------------------------------------ producer ---
template <int D, int PASS>
__device__ void load_tile(const CUtensorMap* tmQ, const CUtensorMap* tmK, uint8_t* dst,
                          uint64_t* bar, const PassArgs& p, const SeqInfo& si, int g, bool is_q,
                          int idx, uint64_t k_policy) {
  using C = Cfg<D, PASS>;
#pragma unroll
  for (int sb = 0; sb < C::kSub; ++sb) {
    if (is_q)
      tma_load_3d(dst + sb * C::kSubBytes, tmQ, bar, sb * 64, g * p.G,
                  si.start + si.q0 + idx * p.tokq);
    else
      tma_load_3d_hint(dst + sb * C::kSubBytes, tmK, bar, sb * 64, g, si.start + idx * kTile,
                       k_policy);
  }
}

template <int D, int PASS>
__device__ void producer(const CUtensorMap* tmQ, const CUtensorMap* tmK, const PassArgs& p,
                         const Smem& s, const Entry* E, UnitIter it) {
  using C = Cfg<D, PASS>;
  const uint32_t q_bytes = (uint32_t)(D * 2 * p.G * p.tokq);
  const uint32_t k_bytes = (uint32_t)(D * 2 * kTile);
  // K tiles stream through L2 once per pass (each CTA reads its own keys):
  // evict them first, so that they do not push out the lines every layer
  // reuses (Q tiles shared by CTAs, row partials, the kernels' code)
  const uint64_t k_policy = l2_policy_evict_first();
  int stage = 0;
  uint32_t sph = 0, uph = 0;
  int issued[C::kStages];
  uint32_t issued_ph[C::kStages];
  for (int i = 0; i < C::kStages; ++i) issued[i] = 0;
  int stat_issued = 0;
  uint32_t stat_ph = 0;
  int ei, st0, st1, unit;
  while (it.next(ei, st0, st1, unit)) {
    const Entry e = E[ei];
    const SeqInfo si = p.seqs[e.seq];
    const bool sq = stat_is_q(e.mode);
    if (!mbar_wait(s.stat_empty, uph ^ 1u, s.abort, p.status, kWaitLimitNs)) goto out;
    mbar_arrive_expect_tx(s.stat_full, (sq ? q_bytes : k_bytes) * (uint32_t)e.n_stat);
    for (int i = 0; i < e.n_stat; ++i)
      load_tile<D, PASS>(tmQ, tmK, s.stat + i * C::kTileBytes, s.stat_full, p, si, e.g, sq,
                         e.stat0 + i, k_policy);
    stat_issued = 1;
    stat_ph = uph;
    uph ^= 1u;
    for (int st = st0; st < st1; ++st) {
      if (!mbar_wait(&s.empty[stage], sph ^ 1u, s.abort, p.status, kWaitLimitNs)) goto out;
      mbar_arrive_expect_tx(&s.full[stage], sq ? k_bytes : q_bytes);
      load_tile<D, PASS>(tmQ, tmK, s.strm + stage * C::kTileBytes, &s.full[stage], p, si, e.g,
                         !sq, e.step0 + st, k_policy);
      issued[stage] = 1;
      issued_ph[stage] = sph;
      if (++stage == C::kStages) { stage = 0; sph ^= 1u; }
    }
  }
out:
  if (*s.abort) {
    // let every copy already issued land before the CTA exits
    int zero = 0;
    for (int i = 0; i < C::kStages; ++i)
      if (issued[i]) mbar_wait(&s.full[i], issued_ph[i], &zero, p.status, kDrainLimitNs);
    if (stat_issued) mbar_wait(s.stat_full, stat_ph, &zero, p.status, kDrainLimitNs);
  }
}

// ---------------------------------------------------------- MMA issuer ---
// Pairs of stationary slot i go to epilogue warpgroup i % 2, so both groups
// work on the same streamed tile and the next one is prefetched meanwhile.
// Each group owns two TMEM buffers.
template <int D, int PASS>
__device__ void mma_issuer(const PassArgs& p, const Smem& s, const Entry* E, UnitIter it,
                           uint32_t tmem) {
  using C = Cfg<D, PASS>;
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128);
  int stage = 0;
  uint32_t sph = 0, uph = 0;
  uint32_t kpair[kWGs] = {0, 0};
  const uint32_t stat0 = smem_addr(s.stat), strm0 = smem_addr(s.strm);
  int ei, st0, st1, unit;
  while (it.next(ei, st0, st1, unit)) {
    const Entry e = E[ei];
    const SeqInfo si = p.seqs[e.seq];
    if (!mbar_wait(s.stat_full, uph, s.abort, p.status, kWaitLimitNs)) goto out;
    uph ^= 1u;
    tc_fence_after();
    for (int st = st0; st < st1; ++st) {
      const int o = e.step0 + st;
      if (!mbar_wait(&s.full[stage], sph, s.abort, p.status, kWaitLimitNs)) goto out;
      tc_fence_after();
      const uint32_t sa = strm0 + stage * C::kTileBytes;
      for (int i = 0; i < e.n_stat; ++i) {
        int j, kt;
        pair_tiles(e, o, i, j, kt);
        if (!pair_live(si, j, kt, p.tokq)) continue;
        const int w = i & 1;
        const int buf = 2 * w + (int)(kpair[w] & 1u);
        const uint32_t ph = (kpair[w] >> 1) & 1u;
        if (!mbar_wait(&s.tempty[buf], ph ^ 1u, s.abort, p.status, kWaitLimitNs)) goto out;
        tc_fence_after();
        const uint32_t ta = stat0 + i * C::kTileBytes;
        // P1: A = Q (stationary), B = K (streamed); P2Q: A = K (streamed),
        // B = Q (stationary); P2K: A = K (stationary), B = Q (streamed).
        const uint32_t a_base = e.mode == kModeP2Q ? sa : ta;
        const uint32_t b_base = e.mode == kModeP2Q ? ta : sa;
        const uint32_t d_tmem = tmem + (uint32_t)(buf * kTile);
#pragma unroll
        for (int k = 0; k < C::kKSteps; ++k) {
          const uint32_t off = (uint32_t)((k >> 2) * C::kSubBytes + (k & 3) * 32);
          mma_bf16(d_tmem, sdesc_kmajor_sw128(a_base + off), sdesc_kmajor_sw128(b_base + off),
                   idesc, k > 0 ? 1u : 0u);
        }
        mma_commit(&s.tfull[buf]);
        ++kpair[w];
      }
      mma_commit(&s.empty[stage]);
      if (++stage == C::kStages) { stage = 0; sph ^= 1u; }
    }
    mma_commit(s.stat_empty);
  }
out:
  // every MMA issued so far must finish before TMEM is released
  mma_commit(s.done);
  int zero = 0;
  mbar_wait(s.done, 0, &zero, p.status, kWaitLimitNs);
}

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
// (pair index mod 8) of this mask.  One in eight measured best here (the
// epilogue is latency-bound rather than MUFU-bound in this kernel; two in
// eight was within 1.5%, three in eight 6% slower).
constexpr uint32_t kPolyPairs = 0x80u;
__device__ constexpr bool poly_col(int c) { return (kPolyPairs >> ((c >> 1) & 7)) & 1u; }

// 2^x for a pair of fp32 values on the FMA/ALU pipes (Cody-Waite split plus
// a polynomial): x = n + f with n = rint(x) and f in [-1/2, 1/2];
// 2^f ~ 1 + f (c1 + f (c2 + f c3)), the relative-error minimax cubic with the
// constant term held at 1 (max relative error 1.0e-4; fitted by linear
// programming on a dense grid), so integer x gives exact powers of two; 2^n
// is added to the exponent bits.  x is clamped to [-125, 127] so the result
// stays a normal fp32 number.
__device__ inline float2 exp2_poly2(float2 x) {
  constexpr float kMagic = 12582912.0f;              // 1.5 * 2^23: rint via fadd
  constexpr float c1 = 0.69328290f, c2 = 0.24221097f, c3 = 0.05500906f;
  x = f2(fminf(fmaxf(x.x, -125.f), 127.f), fminf(fmaxf(x.y, -125.f), 127.f));
  const float2 t = __fadd2_rn(x, f2(kMagic, kMagic));
  const float2 n = __fadd2_rn(t, f2(-kMagic, -kMagic));
  const float2 fr = __ffma2_rn(n, f2(-1.f, -1.f), x);
  float2 q = __ffma2_rn(f2(c3, c3), fr, f2(c2, c2));
  q = __ffma2_rn(q, fr, f2(c1, c1));
  q = __ffma2_rn(q, fr, f2(1.f, 1.f));
  // the magic's low 9 bits are zero, so (bits(t) << 23) == n << 23
  const int ex = __float_as_int(t.x) << 23, ey = __float_as_int(t.y) << 23;
  return f2(__int_as_float(__float_as_int(q.x) + ex), __int_as_float(__float_as_int(q.y) + ey));
}

// sum_c 2^(v_c * sc + off) over all 128 columns, packed fp32x2 arithmetic;
// the column pairs picked by kPolyPairs use the polynomial, the rest the MUFU.
__device__ inline float exp_sum_full(const Cols& v, float sc, float off) {
  const float2 sc2 = f2(sc, sc), off2 = f2(off, off);
  float2 a[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) a[k] = f2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < kTile; c += 2) {
    const float2 x = __ffma2_rn(f2(u2f(v.r[c]), u2f(v.r[c + 1])), sc2, off2);
    const float2 e = poly_col(c) ? exp2_poly2(x) : f2(ex2_approx(x.x), ex2_approx(x.y));
    a[(c >> 1) & 3] = __fadd2_rn(a[(c >> 1) & 3], e);
  }
  return hsum8(a);
}

// Pass 1, one 128-key tile of this thread's row (keys c < nv are causal):
// l += sum_c 2^(v_c*scale2 - m), m = first maximum seen, moved up only when
// the running sum would leave the safe fp32 range.
__device__ inline void p1_pair(const Cols& v, int nv, float sc, float& m, float& l) {
  // one path per warp: a warp whose rows are not all fully causal (or absent)
  // takes the masked path, which also serves its full rows
  const bool full_warp = __all_sync(0xffffffffu, nv == kTile || nv <= 0);
  if (nv <= 0) return;
  if (m == -INFINITY) {
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < kTile; ++c) mx = fmaxf(mx, c < nv ? u2f(v.r[c]) * sc : -INFINITY);
    m = mx;
  }
  float t;
  if (full_warp) {
    t = exp_sum_full(v, sc, -m);
  } else {
    const float nm = -m;
    float a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = 0.f;
#pragma unroll
    for (int c = 0; c < kTile; ++c) {
      const float x = fmaf(u2f(v.r[c]), sc, nm);
      a[c & 7] += ex2_approx(c < nv ? x : -INFINITY);
    }
    t = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
  }
  if (l + t <= kRebaseLimit) {
    l += t;
    return;
  }
  // a value far above the reference: rebase on this tile's maximum
  float mx = m;
#pragma unroll
  for (int c = 0; c < kTile; ++c) mx = fmaxf(mx, c < nv ? u2f(v.r[c]) * sc : -INFINITY);
  float t2 = 0.f;
#pragma unroll
  for (int c = 0; c < kTile; ++c) {
    const float x = fmaf(u2f(v.r[c]), sc, -mx);
    t2 += ex2_approx(c < nv ? x : -INFINITY);
  }
  l = l * ex2_approx(m - mx) + t2;
  m = mx;
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
          const float2 e0 = poly_col(c) ? exp2_poly2(x0) : f2(ex2_approx(x0.x), ex2_approx(x0.y));
          const float2 e1 =
              poly_col(c + 2) ? exp2_poly2(x1) : f2(ex2_approx(x1.x), ex2_approx(x1.y));
          a[(c >> 1) & 3] = __fadd2_rn(a[(c >> 1) & 3], e0);
          a[((c >> 1) + 1) & 3] = __fadd2_rn(a[((c >> 1) + 1) & 3], e1);
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
template <int NR>
__device__ inline void qrow_bias(const PassArgs& p, const SeqInfo& si, int g, const int (&j)[NR],
                                 int r, float (&out)[NR]) {
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
      const Entry& e = p.e1[si.e1 + g * ngrp + j[k] / kMaxStat1];
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
    const float w = nu[k] > 0 ? curve_weight(tok[k], si.len, p.a, p.b) : 0.f;
    out[k] = w > 0.f ? log2f(w) - (acc[k].x + log2f(acc[k].y)) : -INFINITY;
  }
}

template <int D, int PASS>
__device__ void epilogue(const PassArgs& p, const Smem& s, const Entry* E, UnitIter it,
                         uint32_t tmem) {
  const int tid = threadIdx.x;               // 0..255
  const int wg = tid >> 7;                    // warpgroup: owns stationary slots wg, wg + 2
  const int t = tid & 127;                    // TMEM lane == row (pass 1) / key (pass 2)
  const int lane = tid & 31;
  const uint32_t lane_addr = tmem + ((uint32_t)((t >> 5) * 32) << 16);
  // pass 1: this lane's packed row is token t / G of its Q tile (none past
  // the tile's tokq * G rows); the division is done once here
  const int t_tok = t / p.G;
  const bool t_row = t < p.tokq * p.G;
  uint32_t kp = 0;          // pairs consumed by this warpgroup
  int sstep = 0;            // streamed steps seen (double-buffered shared data)
  bool ok = true;           // false after a timeout: keep every barrier, skip the work
  int ei, st0, st1, unit;
  while (it.next(ei, st0, st1, unit)) {
    const Entry e = E[ei];
    const SeqInfo si = p.seqs[e.seq];
    const int g = e.g;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};   // P1 row state / P2K sums
    // pass 1: this lane's token in each of its stationary Q tiles (-1: no row)
    int row_tok[2] = {-1, -1};
    if (PASS == 1) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int tok = si.q0 + (e.stat0 + wg + 2 * k) * p.tokq + t_tok;
        row_tok[k] = t_row && tok < si.len ? tok : -1;
      }
    }
    bar_sync(kBarAll, kEpiThreads);   // the previous unit's shared data is no longer read
    if (PASS == 2 && e.mode == kModeP2Q) {
      static_assert(kMaxStat == 2 * kWGs, "two stationary slots per warpgroup");
      int js[2];
      float bs[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) js[k] = wg + kWGs * k < e.n_stat ? e.stat0 + wg + kWGs * k : -1;
      qrow_bias<2>(p, si, g, js, t, bs);
#pragma unroll
      for (int k = 0; k < 2; ++k)
        if (js[k] >= 0) s.bias_stat[(wg + kWGs * k) * kTile + t] = bs[k];
      bar_sync(kBarAll, kEpiThreads);
    }
    for (int st = st0; st < st1; ++st) {
      const int o = e.step0 + st;
      const int sb = sstep & 1;
      ++sstep;
      float* bias_o = s.bias_strm + sb * kTile;
      if (PASS == 2 && e.mode == kModeP2K) {
        if (wg == 0) {
          const int js[1] = {o};
          float bs[1];
          qrow_bias<1>(p, si, g, js, t, bs);
          bias_o[t] = bs[0];
        }
        bar_sync(kBarAll, kEpiThreads);
      }
      float col = 0.f;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int i = wg + 2 * k;
        if (i >= e.n_stat) break;
        int j, kt;
        pair_tiles(e, o, i, j, kt);
        if (!pair_live(si, j, kt, p.tokq)) continue;
        const int buf = 2 * wg + (int)(kp & 1u);
        const uint32_t ph = (kp >> 1) & 1u;
        ++kp;
        if (ok && !mbar_wait(&s.tfull[buf], ph, s.abort, p.status, kWaitLimitNs)) ok = false;
        if (!ok) continue;
        tc_fence_after();
        Cols v;
        v.load_wait(lane_addr + (uint32_t)(buf * kTile));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.tempty[buf]);
        if (PASS == 1) {
          // in pass 1, j == e.stat0 + i: the token was found at the unit's start
          int nv = row_tok[k] >= 0 ? row_tok[k] - kt * kTile + 1 : 0;
          nv = nv > kTile ? kTile : nv;
          p1_pair(v, nv, p.scale2, m[k], l[k]);
        } else {
          const int key = kt * kTile + t;
          const int f = si.q0 + j * p.tokq;
          const int c_lo = key > f ? min((key - f) * p.G, kTile) : 0;
          const int ncols = min(p.tokq, si.len - f) * p.G;   // valid columns (uniform)
          const float* bias = e.mode == kModeP2K ? bias_o : s.bias_stat + i * kTile;
          const float a2 = p2_pair(v, c_lo, ncols, p.scale2, bias);
          if (e.mode == kModeP2K) l[k] += a2; else col += a2;
        }
      }
      if (PASS == 2 && e.mode == kModeP2Q) {
        // the two warpgroups' halves of this key's column sum
        float* part = s.st_l + (sb * kWGs + wg) * kTile;
        part[t] = col;
        bar_sync(kBarAll, kEpiThreads);
        if (wg == 0 && ok) {
          const int key = o * kTile + t;
          if (key < si.len)
            p.scores[(size_t)g * p.T + si.start + key] = part[t] + part[kTile + t];
        }
      }
    }

    // ---- unit results: each warpgroup writes the slots it owns
    const bool fail = bar_vote_or(kBarAll, kEpiThreads, !ok || *s.abort);
    if (fail) { ok = false; continue; }
    if (PASS == 2 && e.mode == kModeP2Q) continue;
    if (PASS == 1) {
      // the row partials; pass 2 merges them where it reads the rows
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int i = wg + 2 * k;
        if (i >= e.n_stat) break;
        p.part1[((size_t)unit * kMaxStat1 + i) * kTile + t] = make_float2(m[k], l[k]);
      }
      continue;
    }
    if (e.n_units == 1) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int i = wg + 2 * k;
        if (i >= e.n_stat) break;
        const int key = (e.stat0 + i) * kTile + t;
        if (key < si.len) p.scores[(size_t)g * p.T + si.start + key] = l[k];
      }
      continue;
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int i = wg + 2 * k;
      if (i >= e.n_stat) break;
      p.part2[((size_t)unit * kMaxStat + i) * kTile + t] = l[k];
    }
    __threadfence();
    bar_sync(kBarAll, kEpiThreads);
    if (tid == 0) *s.last = atomicAdd(&p.c2[ei], 1u) == (uint32_t)(e.n_units - 1);
    bar_sync(kBarAll, kEpiThreads);
    if (!*s.last) continue;
    __threadfence();
    // each thread merges key t of the slots wg and wg + 2: the partials of all
    // units, in unit order, up to 40 loads in flight
    constexpr size_t kStride = (size_t)kMaxStat * kTile;
    constexpr int kBatch = 20;
    const int nu = e.n_units;
    {
      float acc[2] = {0.f, 0.f};
      for (int u0 = 0; u0 < nu; u0 += kBatch) {
        float x[2][kBatch];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int i = wg + 2 * k;
          const size_t base = ((size_t)e.unit_base * kMaxStat + i) * kTile + t;
#pragma unroll
          for (int b = 0; b < kBatch; ++b)
            x[k][b] = i < e.n_stat && u0 + b < nu
                          ? __ldcg(p.part2 + base + (size_t)(u0 + b) * kStride) : 0.f;
        }
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
          for (int b = 0; b < kBatch; ++b) acc[k] += x[k][b];
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int i = wg + 2 * k;
        const int key = (e.stat0 + i) * kTile + t;
        if (i < e.n_stat && key < si.len) p.scores[(size_t)g * p.T + si.start + key] = acc[k];
      }
    }
  }
}

template <int D, int PASS>
__global__ void __launch_bounds__(kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK, const PassArgs pa,
                    const __grid_constant__ HostPlan hp) {
  using C = Cfg<D, PASS>;
  extern __shared__ uint8_t smem_raw[];
  const Smem s = carve<D, PASS>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr bool p1 = PASS == 1;
  PassArgs p = pa;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], 1); }
    mbar_init(s.stat_full, 1);
    mbar_init(s.stat_empty, 1);
    for (int i = 0; i < kTmemBufs; ++i) { mbar_init(&s.tfull[i], 1); mbar_init(&s.tempty[i], 4); }
    mbar_init(s.done, 1);
    *s.abort = 0;
    fence_mbar_init();
  }
  // padded rows of Q tiles are never written by TMA: keep them finite (zero)
  {
    uint4* z = reinterpret_cast<uint4*>(s.stat);
    const int n = (C::kStat + C::kStages) * C::kTileBytes / 16;
    for (int i = threadIdx.x; i < n; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  if (warp == kMmaWarp) tmem_alloc(s.tmem_slot, kTmemCols);
  if (warp == kProducerWarp && lane == 0) { prefetch_tensormap(&tmQ); prefetch_tensormap(&tmK); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s.tmem_slot;
  // Pass 1 waits for the planner (and whatever wrote Q, K) before anything,
  // then lets pass 2 launch: from then on the plan, Q and K are complete, so
  // pass 2's copy and MMA warps start on them at once; only its epilogue
  // waits (below) for pass 1's row biases.
  if (p1) {
    pdl_wait();
    pdl_allow_next();
  }
  if (p.local_plan) {
    // every CTA plans for itself (cu_seqlens is complete: pass 1 has waited
    // above, and pass 2 starts only after pass 1 has), or copies the plan
    // the host built for the batch {0, T} once cu_seqlens reads so
    if (p.host_plan) {
      const bool valid = p.cu[0] == 0 && p.cu[1] == p.T;   // the same two words in every thread
      const int n1 = valid ? hp.hdr.n_e1 : 0, n2 = valid ? hp.hdr.n_e2 : 0;
      constexpr int kVecs = (int)(sizeof(Entry) / sizeof(uint4));
      const uint4* h1 = reinterpret_cast<const uint4*>(hp.e1);
      const uint4* h2 = reinterpret_cast<const uint4*>(hp.e2);
      uint4* d1 = reinterpret_cast<uint4*>(s.lp->e1);
      uint4* d2 = reinterpret_cast<uint4*>(s.lp->e2);
      for (int i = threadIdx.x; i < (n1 + n2) * kVecs; i += blockDim.x) {
        if (i < n1 * kVecs) d1[i] = h1[i];
        else d2[i - n1 * kVecs] = h2[i - n1 * kVecs];
      }
      if (threadIdx.x == 0) {
        s.lp->seqs[0] = hp.seq;
        PlanHeader h = hp.hdr;
        if (!valid) {
          h = PlanHeader{};
          h.status = WAITS_DEV_BAD_SEQLENS;
        }
        s.lp->hdr = h;
      }
    } else if (warp == 0) {
      warp_plan(p.cu, p.nseq, p.T, p.max_seqlen, p.Hkv, p.tokq, p.a, p.b, (int)gridDim.x, !p1,
                *s.lp);
    }
    __syncthreads();
    p.hdr = &s.lp->hdr;
    p.seqs = s.lp->seqs;
    p.e1 = s.lp->e1;
    p.e2 = s.lp->e2;
    if (p1) {
      // this call's device status word, and zero scores for sequences
      // without an active row (the planner kernel's duties)
      if (blockIdx.x == 0 && threadIdx.x == 0) *pa.status = s.lp->hdr.status;
      if (s.lp->hdr.status == 0) {
        const int64_t stride = (int64_t)gridDim.x * blockDim.x;
        for (int q = 0; q < p.nseq; ++q) {
          const SeqInfo si = s.lp->seqs[q];
          if (si.len == 0 || si.q0 < si.len) continue;
          for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
               i < (int64_t)si.len * p.Hkv; i += stride)
            p.scores[(i / si.len) * p.T + si.start + i % si.len] = 0.0f;
        }
      }
    }
  }
  const PlanHeader* H = p.hdr;
  const Entry* E = p1 ? p.e1 : p.e2;

  UnitIter it;
  const bool have = it.init(E, p1 ? H->n_e1 : H->n_e2, p1 ? H->s1 : H->s2,
                            p1 ? H->p1 : H->p2, blockIdx.x,
                            (p1 ? H->aligned1 : H->aligned2) != 0);
  if (warp >= kProducerWarp) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProducer));
    if (have && warp == kProducerWarp) {
      if (lane == 0) producer<D, PASS>(&tmQ, &tmK, p, s, E, it);
      __syncwarp();
    } else if (have && warp == kMmaWarp) {
      if (lane == 0) mma_issuer<D, PASS>(p, s, E, it, tmem);
      __syncwarp();
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpilogue));
    if (!p1) {
      pdl_wait();
      pdl_allow_next();
    }
    if (have) epilogue<D, PASS>(p, s, E, it, tmem);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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
bool make_map(CUtensorMap* m, const void* base, int T, int heads, int d, int box_h, int box_t) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2};
  const cuuint32_t box[3] = {64u, (cuuint32_t)box_h, (cuuint32_t)box_t};
  const cuuint32_t elem[3] = {1u, 1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

static_assert(sizeof(HostPlan) + 2 * sizeof(CUtensorMap) + sizeof(PassArgs) + 64 <= 4096,
              "scorer parameters must stay within 4 KB");

template <int D>
cudaError_t launch_d(const PassArgs& a, const HostPlan& hp, int grid, cudaStream_t st) {
  CUtensorMap mq, mk;
  if (!make_map(&mq, a.Q, a.T, a.Hq, D, a.G, a.tokq) ||
      !make_map(&mk, a.K, a.T, a.Hkv, D, 1, kTile))
    return cudaErrorInvalidValue;
  const size_t smem1 = Cfg<D, 1>::kSmem, smem2 = Cfg<D, 2>::kSmem;
  cudaError_t err;
  if ((err = cudaFuncSetAttribute(score_tc_kernel<D, 1>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1)) !=
          cudaSuccess ||
      (err = cudaFuncSetAttribute(score_tc_kernel<D, 2>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2)) !=
          cudaSuccess)
    return err;
  if ((err = launch_pdl(score_tc_kernel<D, 1>, dim3(grid), dim3(kThreads), smem1, st, mq, mk,
                        a, hp)) != cudaSuccess) {
    cudaFuncAttributes fa{};
    cudaFuncGetAttributes(&fa, score_tc_kernel<D, 1>);
    int dev = 0, optin = 0, regs = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaDeviceGetAttribute(&regs, cudaDevAttrMaxRegistersPerBlock, dev);
    set_error_detail("scorer: regs %d, max threads %d, local %zu B, static smem %zu B, "
                     "dynamic %zu of opt-in %d B, block regs %d, threads %d",
                     fa.numRegs, fa.maxThreadsPerBlock, fa.localSizeBytes, fa.sharedSizeBytes,
                     smem1, optin, regs, kThreads);
    return err;
  }
  return launch_pdl(score_tc_kernel<D, 2>, dim3(grid), dim3(kThreads), smem2, st, mq, mk, a,
                    hp);
}

}  // namespace

cudaError_t launch_score_passes(const PassArgs& a, const HostPlan* hp, int grid, cudaStream_t s) {
  static const HostPlan kNone{};
  const HostPlan& h = hp ? *hp : kNone;
  return a.d == 64 ? launch_d<64>(a, h, grid, s) : launch_d<128>(a, h, grid, s);
}

}  // namespace waits
