// Two-pass WAITS scorer on the sm_100a tensor cores.
//
// WAITS README (stig.sh/Dirac-Notation/A2SF), opening summary: the score of
// key k is the accumulative attention it receives, each query row q weighted
// by the forgetting curve w[q].  Read as causal softmax(QK^T / sqrt(d)) summed
// over the query heads of a KV group:
//   pass 1  bias[q,h] = log2 w[q] - log2 sum_{k<=q} 2^(x[q,k]),
//           x = (Q.K) * log2(e) / sqrt(d)
//   pass 2  s[g,k]    = sum_{h in g} sum_{q>=k} 2^(x[q,k] + bias[q,h])
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
#include "sm100.cuh"
#include "unit_iter.cuh"

namespace waits {
namespace {

using namespace sm100;

constexpr int kEpiWarps = 4;
constexpr int kThreads = (kEpiWarps + 2) * 32;
constexpr int kProducerWarp = kEpiWarps;
constexpr int kMmaWarp = kEpiWarps + 1;
constexpr int kTmemBufs = 4;
constexpr int kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 0.2 s after an abort
constexpr int kEpiBar = 1;                          // named barrier of warps 0-3

template <int D>
struct Cfg {
  static constexpr int kSub = D / 64;                    // 128-byte column blocks
  static constexpr int kSubBytes = kTile * 128;          // 16 KB
  static constexpr int kTileBytes = kSub * kSubBytes;
  static constexpr int kStages = D == 128 ? 2 : 4;
  static constexpr int kKSteps = D / 16;
  static constexpr size_t kSmem = 1024 + (size_t)(kMaxStat + kStages) * kTileBytes +
                                  (kMaxStat + 2) * kTile * sizeof(float) + 256;
};

struct Smem {
  uint8_t* stat;
  uint8_t* strm;
  float* bias_stat;  // [4][128]
  float* bias_strm;  // [2][128]
  uint64_t* full;
  uint64_t* empty;
  uint64_t* stat_full;
  uint64_t* stat_empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* done;
  uint32_t* tmem_slot;
  volatile int* abort;
  int* last;
};

template <int D>
__device__ Smem carve(uint8_t* raw) {
  using C = Cfg<D>;
  Smem s;
  const uint32_t a = smem_addr(raw);
  uint8_t* base = raw + ((1024u - (a & 1023u)) & 1023u);
  s.stat = base;
  s.strm = s.stat + kMaxStat * C::kTileBytes;
  s.bias_stat = reinterpret_cast<float*>(s.strm + C::kStages * C::kTileBytes);
  s.bias_strm = s.bias_stat + kMaxStat * kTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s.bias_strm + 2 * kTile);
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

// ------------------------------------------------------------ producer ---
template <int D>
__device__ void load_tile(const CUtensorMap* tmQ, const CUtensorMap* tmK, uint8_t* dst,
                          uint64_t* bar, const PassArgs& p, const SeqInfo& si, int g, bool is_q,
                          int idx) {
  using C = Cfg<D>;
#pragma unroll
  for (int sb = 0; sb < C::kSub; ++sb) {
    if (is_q)
      tma_load_3d(dst + sb * C::kSubBytes, tmQ, bar, sb * 64, g * p.G,
                  si.start + si.q0 + idx * p.tokq);
    else
      tma_load_3d(dst + sb * C::kSubBytes, tmK, bar, sb * 64, g, si.start + idx * kTile);
  }
}

template <int D>
__device__ void producer(const CUtensorMap* tmQ, const CUtensorMap* tmK, const PassArgs& p,
                         const Smem& s, const Entry* E, UnitIter it) {
  using C = Cfg<D>;
  const uint32_t q_bytes = (uint32_t)(D * 2 * p.G * p.tokq);
  const uint32_t k_bytes = (uint32_t)(D * 2 * kTile);
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
      load_tile<D>(tmQ, tmK, s.stat + i * C::kTileBytes, s.stat_full, p, si, e.g, sq,
                   e.stat0 + i);
    stat_issued = 1;
    stat_ph = uph;
    uph ^= 1u;
    for (int st = st0; st < st1; ++st) {
      if (!mbar_wait(&s.empty[stage], sph ^ 1u, s.abort, p.status, kWaitLimitNs)) goto out;
      mbar_arrive_expect_tx(&s.full[stage], sq ? k_bytes : q_bytes);
      load_tile<D>(tmQ, tmK, s.strm + stage * C::kTileBytes, &s.full[stage], p, si, e.g, !sq,
                   e.step0 + st);
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
template <int D>
__device__ void mma_issuer(const PassArgs& p, const Smem& s, const Entry* E, UnitIter it,
                           uint32_t tmem) {
  using C = Cfg<D>;
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128);
  int stage = 0, buf = 0;
  uint32_t sph = 0, uph = 0, bph = 0;
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
        const int j = e.mode == kModeP2K ? o : e.stat0 + i;
        const int kt = e.mode == kModeP2K ? e.stat0 + i : o;
        if (!pair_live(si, j, kt, p.tokq)) continue;
        if (!mbar_wait(&s.tempty[buf], bph ^ 1u, s.abort, p.status, kWaitLimitNs)) goto out;
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
        if (++buf == kTmemBufs) { buf = 0; bph ^= 1u; }
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
// Load 32 TMEM columns of this warp's lanes; the wait names the registers so
// no use of them can be scheduled before the data has arrived.
struct Chunk {
  uint32_t r[32];
  __device__ void load(uint32_t taddr) { tmem_ld32(taddr, r); }
  __device__ void wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]),
                   "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                   "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]),
                   "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
  }
};

// Pass 1, one chunk of 32 keys for this thread's row: adds
// sum 2^(v*scale2 - mref) over the valid keys (c < nv) to *acc (relative to
// mref), moving mref up when the running sum would leave the safe range.
__device__ inline void p1_chunk(const Chunk& ch, int cbase, int nv, float scale2, float& mref,
                                float& lsum, float& acc) {
  if (cbase >= nv) return;
  const bool masked = cbase + 32 > nv;
  if (mref == -INFINITY) {
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (!masked || cbase + j < nv) mx = fmaxf(mx, u2f(ch.r[j]) * scale2);
    mref = mx;
  }
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
  if (!masked) {
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      s0 += ex2_approx(fmaf(u2f(ch.r[j + 0]), scale2, -mref));
      s1 += ex2_approx(fmaf(u2f(ch.r[j + 1]), scale2, -mref));
      s2 += ex2_approx(fmaf(u2f(ch.r[j + 2]), scale2, -mref));
      s3 += ex2_approx(fmaf(u2f(ch.r[j + 3]), scale2, -mref));
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      s0 += cbase + j + 0 < nv ? ex2_approx(fmaf(u2f(ch.r[j + 0]), scale2, -mref)) : 0.f;
      s1 += cbase + j + 1 < nv ? ex2_approx(fmaf(u2f(ch.r[j + 1]), scale2, -mref)) : 0.f;
      s2 += cbase + j + 2 < nv ? ex2_approx(fmaf(u2f(ch.r[j + 2]), scale2, -mref)) : 0.f;
      s3 += cbase + j + 3 < nv ? ex2_approx(fmaf(u2f(ch.r[j + 3]), scale2, -mref)) : 0.f;
    }
  }
  const float cs = (s0 + s1) + (s2 + s3);
  if (lsum + acc + cs <= kRebaseLimit) {
    acc += cs;
    return;
  }
  // a value far above the reference: rebase on this chunk's maximum
  float mx = mref;
#pragma unroll
  for (int j = 0; j < 32; ++j)
    if (!masked || cbase + j < nv) mx = fmaxf(mx, u2f(ch.r[j]) * scale2);
  const float f = ex2_approx(mref - mx);
  lsum *= f;
  acc *= f;
  float t = 0.f;
#pragma unroll
  for (int j = 0; j < 32; ++j)
    if (!masked || cbase + j < nv) t += ex2_approx(fmaf(u2f(ch.r[j]), scale2, -mx));
  acc += t;
  mref = mx;
}

// Pass 2, one chunk of 32 query columns for this thread's key: adds
// sum 2^(v*scale2 + bias[c]) over columns c in [c0, 128).
__device__ inline float p2_chunk(const Chunk& ch, int cbase, int c0, float scale2,
                                 const float* bias) {
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
  const float4* b4 = reinterpret_cast<const float4*>(bias + cbase);
  if (c0 <= cbase) {
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      const float4 b = b4[j / 4];
      s0 += ex2_approx(fmaf(u2f(ch.r[j + 0]), scale2, b.x));
      s1 += ex2_approx(fmaf(u2f(ch.r[j + 1]), scale2, b.y));
      s2 += ex2_approx(fmaf(u2f(ch.r[j + 2]), scale2, b.z));
      s3 += ex2_approx(fmaf(u2f(ch.r[j + 3]), scale2, b.w));
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      const float4 b = b4[j / 4];
      s0 += cbase + j + 0 >= c0 ? ex2_approx(fmaf(u2f(ch.r[j + 0]), scale2, b.x)) : 0.f;
      s1 += cbase + j + 1 >= c0 ? ex2_approx(fmaf(u2f(ch.r[j + 1]), scale2, b.y)) : 0.f;
      s2 += cbase + j + 2 >= c0 ? ex2_approx(fmaf(u2f(ch.r[j + 2]), scale2, b.z)) : 0.f;
      s3 += cbase + j + 3 >= c0 ? ex2_approx(fmaf(u2f(ch.r[j + 3]), scale2, b.w)) : 0.f;
    }
  }
  return (s0 + s1) + (s2 + s3);
}

__device__ inline void epi_sync() {
  __syncwarp();
  named_bar_sync(kEpiBar, kEpiWarps * 32);
}
// Barrier of warps 0-3 that also ORs `v` over them (a uniform answer).
__device__ inline bool epi_vote_or(bool v) {
  __syncwarp();
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(kEpiBar), "r"(kEpiWarps * 32)
      : "memory");
  return r != 0;
}

// Bias of the 128 packed rows of Q tile j (-inf where no row exists).
__device__ inline float qrow_bias(const PassArgs& p, const SeqInfo& si, int g, int j, int r) {
  const int tok = si.q0 + j * p.tokq + r / p.G;
  if (r < p.tokq * p.G && tok < si.len)
    return p.bias[((size_t)g * p.T + si.start + si.q0 + (size_t)j * p.tokq) * p.G + r];
  return -INFINITY;
}

__device__ void write_row_bias(const PassArgs& p, const SeqInfo& si, int g, int tok, int hg,
                               float lse2) {
  const float w = curve_weight(tok, si.len, p.a, p.b);
  p.bias[((size_t)g * p.T + si.start + tok) * p.G + hg] = w > 0.f ? log2f(w) - lse2 : -INFINITY;
}

template <int D>
__device__ void epilogue(const PassArgs& p, const Smem& s, const Entry* E, UnitIter it,
                         uint32_t tmem, bool pass1) {
  const int t = threadIdx.x;                 // TMEM lane == row (pass 1) / key (pass 2)
  const int warp = t >> 5, lane = t & 31;
  const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
  int buf = 0, sstep = 0;
  uint32_t bph = 0;
  bool ok = true;   // false after a timeout: keep every barrier, skip the work
  int ei, st0, st1, unit;
  while (it.next(ei, st0, st1, unit)) {
    const Entry e = E[ei];
    const SeqInfo si = p.seqs[e.seq];
    const int g = e.g;
    float mref[kMaxStat], lsum[kMaxStat], acc[kMaxStat];
#pragma unroll
    for (int i = 0; i < kMaxStat; ++i) { mref[i] = -INFINITY; lsum[i] = 0.f; acc[i] = 0.f; }
    if (e.mode == kModeP2Q) {
      epi_sync();
      for (int i = 0; i < e.n_stat; ++i) s.bias_stat[i * kTile + t] = qrow_bias(p, si, g, e.stat0 + i, t);
      epi_sync();
    }
    for (int st = st0; st < st1; ++st) {
      const int o = e.step0 + st;
      float* bias_o = s.bias_strm + (sstep & 1) * kTile;
      if (e.mode == kModeP2K) {
        bias_o[t] = qrow_bias(p, si, g, o, t);
        epi_sync();
      }
      ++sstep;
      float col = 0.f;
#pragma unroll
      for (int i = 0; i < kMaxStat; ++i) {
        if (i >= e.n_stat) break;
        const int j = e.mode == kModeP2K ? o : e.stat0 + i;
        const int kt = e.mode == kModeP2K ? e.stat0 + i : o;
        if (!pair_live(si, j, kt, p.tokq)) continue;
        if (ok && !mbar_wait(&s.tfull[buf], bph, s.abort, p.status, kWaitLimitNs)) ok = false;
        if (!ok) { if (++buf == kTmemBufs) { buf = 0; bph ^= 1u; } continue; }
        tc_fence_after();
        const uint32_t ta = lane_addr + (uint32_t)(buf * kTile);
        Chunk c0, c1;
        if (e.mode == kModeP1) {
          const int tok = si.q0 + j * p.tokq + t / p.G;
          const bool row_ok = t < p.tokq * p.G && tok < si.len;
          int nv = row_ok ? tok - kt * kTile + 1 : 0;
          nv = nv > kTile ? kTile : (nv < 0 ? 0 : nv);
          float a2 = 0.f;
          c0.load(ta); c0.wait();
          c1.load(ta + 32);
          p1_chunk(c0, 0, nv, p.scale2, mref[i], lsum[i], a2);
          __syncwarp(); c1.wait();
          c0.load(ta + 64);
          p1_chunk(c1, 32, nv, p.scale2, mref[i], lsum[i], a2);
          __syncwarp(); c0.wait();
          c1.load(ta + 96);
          p1_chunk(c0, 64, nv, p.scale2, mref[i], lsum[i], a2);
          __syncwarp(); c1.wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s.tempty[buf]);
          p1_chunk(c1, 96, nv, p.scale2, mref[i], lsum[i], a2);
          lsum[i] += a2;
        } else {
          const int key = kt * kTile + t;
          const int f = si.q0 + j * p.tokq;
          const int cmin = key > f ? (key - f) * p.G : 0;
          const int c_lo = cmin > kTile ? kTile : cmin;
          const int ncols = min(p.tokq, si.len - f) * p.G;   // valid columns (uniform)
          const float* bias = e.mode == kModeP2K ? bias_o : s.bias_stat + i * kTile;
          float a2 = 0.f;
          c0.load(ta); c0.wait();
          c1.load(ta + 32);
          if (0 < ncols) a2 += p2_chunk(c0, 0, c_lo, p.scale2, bias);
          __syncwarp(); c1.wait();
          c0.load(ta + 64);
          if (32 < ncols) a2 += p2_chunk(c1, 32, c_lo, p.scale2, bias);
          __syncwarp(); c0.wait();
          c1.load(ta + 96);
          if (64 < ncols) a2 += p2_chunk(c0, 64, c_lo, p.scale2, bias);
          __syncwarp(); c1.wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s.tempty[buf]);
          if (96 < ncols) a2 += p2_chunk(c1, 96, c_lo, p.scale2, bias);
          if (e.mode == kModeP2K) acc[i] += a2; else col += a2;
        }
        if (++buf == kTmemBufs) { buf = 0; bph ^= 1u; }
      }
      if (e.mode == kModeP2Q && ok) {
        const int key = o * kTile + t;
        if (key < si.len) p.scores[(size_t)g * p.T + si.start + key] = col;
      }
    }

    // ---- unit results (skipped by all epilogue threads together after a timeout)
    if (epi_vote_or(!ok || *s.abort)) { ok = false; continue; }
    if (e.mode == kModeP1) {
      if (e.n_units == 1) {
#pragma unroll
        for (int i = 0; i < kMaxStat; ++i) {
          if (i >= e.n_stat) break;
          const int tok = si.q0 + (e.stat0 + i) * p.tokq + t / p.G;
          if (t < p.tokq * p.G && tok < si.len)
            write_row_bias(p, si, g, tok, t % p.G, mref[i] + log2f(lsum[i]));
        }
      } else {
#pragma unroll
        for (int i = 0; i < kMaxStat; ++i)
          if (i < e.n_stat)
            p.part1[((size_t)unit * kMaxStat + i) * kTile + t] = make_float2(mref[i], lsum[i]);
        __threadfence();
        epi_sync();
        if (t == 0) *s.last = atomicAdd(&p.c1[ei], 1u) == (uint32_t)(e.n_units - 1);
        epi_sync();
        if (*s.last) {
          __threadfence();
          for (int i = 0; i < e.n_stat; ++i) {
            const int tok = si.q0 + (e.stat0 + i) * p.tokq + t / p.G;
            if (t >= p.tokq * p.G || tok >= si.len) continue;
            const float2* parts = p.part1 + ((size_t)e.unit_base * kMaxStat + i) * kTile + t;
            float M = -INFINITY;
            for (int u = 0; u < e.n_units; ++u) {
              const float2 v = __ldcg(parts + (size_t)u * kMaxStat * kTile);
              if (v.y > 0.f) M = fmaxf(M, v.x);
            }
            float L = 0.f;
            for (int u = 0; u < e.n_units; ++u) {
              const float2 v = __ldcg(parts + (size_t)u * kMaxStat * kTile);
              if (v.y > 0.f) L += v.y * ex2_approx(v.x - M);
            }
            write_row_bias(p, si, g, tok, t % p.G, M + log2f(L));
          }
        }
      }
    } else if (e.mode == kModeP2K) {
      if (e.n_units == 1) {
#pragma unroll
        for (int i = 0; i < kMaxStat; ++i) {
          const int key = (e.stat0 + i) * kTile + t;
          if (i < e.n_stat && key < si.len) p.scores[(size_t)g * p.T + si.start + key] = acc[i];
        }
      } else {
#pragma unroll
        for (int i = 0; i < kMaxStat; ++i)
          if (i < e.n_stat) p.part2[((size_t)unit * kMaxStat + i) * kTile + t] = acc[i];
        __threadfence();
        epi_sync();
        if (t == 0) *s.last = atomicAdd(&p.c2[ei], 1u) == (uint32_t)(e.n_units - 1);
        epi_sync();
        if (*s.last) {
          __threadfence();
          for (int i = 0; i < e.n_stat; ++i) {
            const int key = (e.stat0 + i) * kTile + t;
            float sum = 0.f;
            for (int u = 0; u < e.n_units; ++u)
              sum += __ldcg(p.part2 + ((size_t)(e.unit_base + u) * kMaxStat + i) * kTile + t);
            if (key < si.len) p.scores[(size_t)g * p.T + si.start + key] = sum;
          }
        }
      }
    }
  }
  (void)pass1;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK, PassArgs p, int pass) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const Smem s = carve<D>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool p1 = pass == 1;
  const PlanHeader* H = p.hdr;
  const Entry* E = p1 ? p.e1 : p.e2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], 1); }
    mbar_init(s.stat_full, 1);
    mbar_init(s.stat_empty, 1);
    for (int i = 0; i < kTmemBufs; ++i) { mbar_init(&s.tfull[i], 1); mbar_init(&s.tempty[i], kEpiWarps); }
    mbar_init(s.done, 1);
    *s.abort = 0;
    fence_mbar_init();
  }
  // padded rows of Q tiles are never written by TMA: keep them finite (zero)
  {
    uint4* z = reinterpret_cast<uint4*>(s.stat);
    const int n = (kMaxStat + C::kStages) * C::kTileBytes / 16;
    for (int i = threadIdx.x; i < n; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  if (warp == kMmaWarp) tmem_alloc(s.tmem_slot, kTmemCols);
  if (warp == kProducerWarp && lane == 0) { prefetch_tensormap(&tmQ); prefetch_tensormap(&tmK); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s.tmem_slot;

  UnitIter it;
  const bool have = it.init(E, p1 ? H->n_e1 : H->n_e2, p1 ? H->s1 : H->s2,
                            p1 ? H->p1 : H->p2, blockIdx.x);
  if (have) {
    if (warp == kProducerWarp) {
      if (lane == 0) producer<D>(&tmQ, &tmK, p, s, E, it);
      __syncwarp();
    } else if (warp == kMmaWarp) {
      if (lane == 0) mma_issuer<D>(p, s, E, it, tmem);
      __syncwarp();
    } else {
      epilogue<D>(p, s, E, it, tmem, p1);
    }
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

template <int D>
cudaError_t launch_d(const PassArgs& a, int grid, cudaStream_t st) {
  CUtensorMap mq, mk;
  if (!make_map(&mq, a.Q, a.T, a.Hq, D, a.G, a.tokq) ||
      !make_map(&mk, a.K, a.T, a.Hkv, D, 1, kTile))
    return cudaErrorInvalidValue;
  const size_t smem = Cfg<D>::kSmem;
  cudaError_t err = cudaFuncSetAttribute(score_tc_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  score_tc_kernel<D><<<grid, kThreads, smem, st>>>(mq, mk, a, 1);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  score_tc_kernel<D><<<grid, kThreads, smem, st>>>(mq, mk, a, 2);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_passes(const PassArgs& a, int grid, cudaStream_t s) {
  return a.d == 64 ? launch_d<64>(a, grid, s) : launch_d<128>(a, grid, s);
}

}  // namespace waits
