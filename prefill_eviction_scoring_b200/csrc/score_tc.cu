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
#include "scorer_common.cuh"

namespace waits {
namespace {

using namespace scorer;
constexpr int kTmemBufs = 2 * kWGs;                  // two 128-column buffers per WG

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
    if (!mbar_wait(s.stat_empty, uph ^ 1u, s.abort, p.status, p.wait_ns)) goto out;
    mbar_arrive_expect_tx(s.stat_full, (sq ? q_bytes : k_bytes) * (uint32_t)e.n_stat);
    for (int i = 0; i < e.n_stat; ++i)
      load_tile<D, PASS>(tmQ, tmK, s.stat + i * C::kTileBytes, s.stat_full, p, si, e.g, sq,
                         e.stat0 + i, k_policy);
    stat_issued = 1;
    stat_ph = uph;
    uph ^= 1u;
    for (int st = st0; st < st1; ++st) {
      if (!mbar_wait(&s.empty[stage], sph ^ 1u, s.abort, p.status, p.wait_ns)) goto out;
      mbar_arrive_expect_tx(&s.full[stage], sq ? k_bytes : q_bytes);
      load_tile<D, PASS>(tmQ, tmK, s.strm + stage * C::kTileBytes, &s.full[stage], p, si, e.g,
                         !sq, e.step0 + st, k_policy);
      issued[stage] = 1;
      issued_ph[stage] = sph;
      if (++stage == C::kStages) { stage = 0; sph ^= 1u; }
    }
  }
out:
  {
    // let every copy issued land before the CTA exits (after a normal run
    // the MMA warp has consumed them all and these return at once)
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
  if (p.withhold_mma) goto out;   // testing aid: every accumulator wait runs out
  while (it.next(ei, st0, st1, unit)) {
    const Entry e = E[ei];
    const SeqInfo si = p.seqs[e.seq];
    if (!mbar_wait(s.stat_full, uph, s.abort, p.status, p.wait_ns)) goto out;
    uph ^= 1u;
    tc_fence_after();
    for (int st = st0; st < st1; ++st) {
      const int o = e.step0 + st;
      if (!mbar_wait(&s.full[stage], sph, s.abort, p.status, p.wait_ns)) goto out;
      tc_fence_after();
      const uint32_t sa = strm0 + stage * C::kTileBytes;
      for (int i = 0; i < e.n_stat; ++i) {
        int j, kt;
        pair_tiles(e, o, i, j, kt);
        if (!pair_live(si, j, kt, p.tokq)) continue;
        const int w = i & 1;
        const int buf = 2 * w + (int)(kpair[w] & 1u);
        const uint32_t ph = (kpair[w] >> 1) & 1u;
        if (!mbar_wait(&s.tempty[buf], ph ^ 1u, s.abort, p.status, p.wait_ns)) goto out;
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
  mbar_wait(s.done, 0, &zero, p.status, kDoneLimitNs);
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
    // P2K with merged biases: each warpgroup loads each streamed Q tile's
    // row biases itself, one step ahead (the latency overlaps the previous
    // step's arithmetic), into its own buffers, so the groups do not wait
    // for each other at every step
    const bool ahead = PASS == 2 && e.mode == kModeP2K && p.bias_ready;
    float nb = ahead && st0 < st1 ? merged_bias(p, p.e1, si, g, e.step0 + st0, t) : 0.f;
    for (int st = st0; st < st1; ++st) {
      const int o = e.step0 + st;
      const int sb = sstep & 1;
      ++sstep;
      float* bias_o = s.bias_strm + (ahead ? wg * 2 + sb : sb) * kTile;
      if (PASS == 2 && e.mode == kModeP2K) {
        if (ahead) {
          bias_o[t] = nb;
          if (st + 1 < st1) nb = merged_bias(p, p.e1, si, g, o + 1, t);
          bar_sync(1 + wg, 128);
        } else {
          if (wg == 0) {
            const int js[1] = {o};
            float bs[1];
            qrow_bias<1>(p, si, g, js, t, bs);
            bias_o[t] = bs[0];
          }
          bar_sync(kBarAll, kEpiThreads);
        }
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
        if (ok && !mbar_wait(&s.tfull[buf], ph, s.abort, p.status, p.wait_ns)) ok = false;
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
  stage_host_plan(pa, hp, s.lp);
  if (p1 || pa.lse) {
    pdl_wait();
    pdl_allow_next();
  }
  plan_prologue(p, pa, hp, s.lp, p1, warp);
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

static_assert(sizeof(HostPlan) + 2 * sizeof(CUtensorMap) + sizeof(PassArgs) + 64 <= 4096,
              "scorer parameters must stay within 4 KB");

template <int D>
cudaError_t launch_d(const PassArgs& a, const HostPlan& hp, int grid, cudaStream_t st,
                     bool pass1 = true) {
  CUtensorMap mq, mk;
  if (!make_map(&mq, a.Q, a.T, a.Hq, a.q_row_heads, D, a.G, a.tokq) ||
      !make_map(&mk, a.K, a.T, a.Hkv, a.kv_row_heads, D, 1, kTile))
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
  if (pass1 && !a.lse &&
      (err = launch_pdl(score_tc_kernel<D, 1>, dim3(grid), dim3(kThreads), smem1, st, mq, mk, a,
                        hp)) != cudaSuccess) {
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

// The scorer's FMA-pipe 2^x on n values (a testing aid: the same function
// the epilogue runs, added to zero, so its error can be measured against
// exact powers).
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  const float2 zero = make_float2(0.f, 0.f);
  if (i + 1 < n) {
    const float2 r = exp2_poly_acc(make_float2(x[i], x[i + 1]), zero);
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_poly_acc(make_float2(x[i], 0.f), zero).x;
  }
}

cudaError_t launch_exp2_poly(const float* x, float* y, int64_t n, cudaStream_t s) {
  const int64_t pairs = (n + 1) / 2;
  const int64_t blocks = (pairs + 255) / 256;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  exp2_poly_kernel<<<(unsigned)blocks, 256, 0, s>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_score_passes(const PassArgs& a, const HostPlan* hp, int grid, cudaStream_t s) {
  static const HostPlan kNone{};
  const HostPlan& h = hp ? *hp : kNone;
  return a.d == 64 ? launch_d<64>(a, h, grid, s) : launch_d<128>(a, h, grid, s);
}

// Each row's bias (log2 of its curve weight minus its log2-sum-exp) from its
// pass-1 partials, merged once for pass 2 instead of once per stationary
// K-tile group that streams the row: thread (entry, slot, row) runs the
// merge pass 2 would run and writes the result over the entry's first
// partial (it alone reads or writes those slots).
__global__ void __launch_bounds__(256) row_bias_kernel(const __grid_constant__ PassArgs p) {
  pdl_allow_next();
  pdl_wait();
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t e = idx / (kMaxStat1 * kTile);
  const int i = (int)((idx / kTile) % kMaxStat1), r = (int)(idx % kTile);
  if (e >= p.hdr->n_e1) return;
  const Entry en = p.e1[e];
  if (i >= en.n_stat || en.n_units <= 0) return;
  const SeqInfo si = p.seqs[en.seq];
  const int js[1] = {en.stat0 + i};
  float b[1];
  qrow_bias<1>(p, p.e1, si, en.g, js, r, b);
  p.part1[((size_t)en.unit_base * kMaxStat1 + i) * kTile + r] = make_float2(b[0], 0.f);
}

cudaError_t launch_row_bias(const PassArgs& a, int64_t max_e1, cudaStream_t s) {
  const int64_t threads = max_e1 * kMaxStat1 * kTile;
  const int64_t blocks = (threads + 255) / 256;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
  PassArgs b = a;
  b.bias_ready = 0;
  return launch_pdl(row_bias_kernel, dim3((unsigned)blocks), dim3(256), 0, s, b);
}

cudaError_t launch_score_pass2(const PassArgs& a, int grid, cudaStream_t s) {
  static const HostPlan kNone{};
  return a.d == 64 ? launch_d<64>(a, kNone, grid, s, false)
                   : launch_d<128>(a, kNone, grid, s, false);
}

}  // namespace waits
