// WAITS scorer for the small plans of the sparse-weight regime: every
// sequence's active query rows fit in 4 Q tiles, so pass 2 holds all of them
// stationary and finishes a key's score in one step (mode P2Q), and the plan
// is small enough for every CTA to build it (or for the host to pass it).
//
// WAITS README (stig.sh/Dirac-Notation/A2SF), opening summary: the score of
// key k is the attention it receives, each query row q weighted by the
// forgetting curve w[q]; read as causal softmax(QK^T / sqrt(d)) summed over
// the query heads of a KV group.  The two passes compute what score_tc.cu's
// passes compute, with the same arithmetic in the same order, so the scores
// are bit-identical to it:
//   pass 1  per row (q, h): sum_{k<=q} 2^(x[q,k]), x = (Q.K) * log2(e) / sqrt(d),
//           as (reference max, sum) partials of the CTAs sharing the row
//   pass 2  bias[q,h] = log2 w[q] - log2 of the merged sum, then
//           s[g,k]    = sum_{h in g} sum_{q>=k} 2^(x[q,k] + bias[q,h])
//
// What differs is the shape of the tensor-core work: each MMA covers 256
// columns instead of 128 (pass 1: two K tiles of 128 keys against one Q
// tile; pass 2: one K tile against two Q tiles), so tensor memory holds two
// 256-column accumulators, one per epilogue warpgroup, and every handshake
// between the MMA warp and the epilogue (barrier waits, fences, commits)
// moves twice the work.  The epilogue reads an accumulator in two halves of
// 128 columns and frees it after the second read, so the next MMA into it
// overlaps the arithmetic on the second half.
//
// Per CTA (persistent, one per SM): warp 8 streams tiles with TMA into
// 128-byte-swizzled shared memory, warp 9 issues tcgen05.mma, warpgroups 0-1
// read the accumulators (one TMEM lane per thread) and do the exponentials.
// In pass 2 the two warpgroups own different query tiles of the same keys;
// warpgroup 1 hands its half of each key's column sum to warpgroup 0 through
// shared memory and a pair of mbarriers, so the groups are not held in step
// by a barrier of both.  Every wait is bounded; a timeout sets
// WAITS_DEV_TIMEOUT and the CTA exits after its copies and MMAs have landed.
#include "scorer_common.cuh"

namespace waits {
namespace {

using namespace scorer;

constexpr int kAccCols = 256;   // columns of one accumulator (one per epilogue warpgroup)
constexpr int kSubBytes = kTile * 128;   // one 128-row x 64-column bf16 block (16 KB)

// Shared memory per head dim and pass.  Tiles are stored as 64-column blocks
// of 128 rows, block-major across the tiles of a region ([block][tile][row]),
// so consecutive tiles form one operand of 256 rows for the MMA.
//   pass 1: 2 stationary Q tiles; stages of 2 K tiles (256 keys)
//   pass 2: 4 stationary Q tiles; stages of 1 K tile (128 keys)
template <int D, int PASS>
struct SCfg {
  static constexpr int kSub = D / 64;
  static constexpr int kTileBytes = kSub * kSubBytes;
  static constexpr int kStat = PASS == 1 ? 2 : 4;
  static constexpr int kStageTiles = PASS == 1 ? 2 : 1;
  static constexpr int kStages = (D == 128 ? 2 : 4);
  static constexpr int kStageBytes = kStageTiles * kTileBytes;
  static constexpr int kKSteps = D / 16;
};

// Byte offsets of everything in shared memory, from the 1024-byte-aligned
// base: compile-time constants, so the roles hold one base pointer instead
// of a register per buffer.
template <int D, int PASS>
struct SL {
  using C = SCfg<D, PASS>;
  static constexpr uint32_t stat = 0;
  static constexpr uint32_t strm = stat + C::kStat * C::kTileBytes;
  static constexpr uint32_t bias = strm + C::kStages * C::kStageBytes;   // float [4][128]
  static constexpr uint32_t part = bias + 4 * kTile * 4;                  // float [2][128]
  static constexpr uint32_t lp = part + 2 * kTile * 4;                    // LocalPlan
  static constexpr uint32_t bars = lp + (uint32_t)((sizeof(LocalPlan) + 7) / 8 * 8);
  static constexpr uint32_t full = bars;                                  // [kStages]
  static constexpr uint32_t empty = full + 8 * C::kStages;                // [kStages]
  static constexpr uint32_t stat_full = empty + 8 * C::kStages;
  static constexpr uint32_t stat_empty = stat_full + 8;
  static constexpr uint32_t tfull = stat_empty + 8;                       // [2]
  static constexpr uint32_t tempty = tfull + 16;                          // [2]
  static constexpr uint32_t pfull = tempty + 16;                          // [2]
  static constexpr uint32_t pfree = pfull + 16;                           // [2]
  static constexpr uint32_t done = pfree + 16;
  static constexpr uint32_t tmem_slot = done + 8;
  static constexpr uint32_t abort = tmem_slot + 4;
  static constexpr uint32_t end = abort + 4;
};

// Accessors on the aligned base.
struct SB {
  uint8_t* b;
  template <typename T>
  __device__ T* at(uint32_t off) const { return reinterpret_cast<T*>(b + off); }
  __device__ uint64_t* bar(uint32_t off, int i = 0) const { return at<uint64_t>(off) + i; }
  __device__ volatile int* abort_flag(uint32_t off) const { return at<volatile int>(off); }
};

// Slot of stationary Q tile i in pass 2: warpgroup w owns tiles w and w + 2
// (as score_tc.cu's epilogue does, so the column sums add in the same
// order), stored next to each other as one 256-row operand.
__device__ inline int p2_slot(int i) { return (i & 1) * 2 + (i >> 1); }

// Pass 1: K tiles [o, o + nt) against stationary Q tile j: how many of them
// some row of the tile sees (the later tile first drops out).
__device__ inline int p1_live_tiles(const SeqInfo& si, int j, int o, int nt, int tokq) {
  if (!pair_live(si, j, o, tokq)) return 0;
  return nt == 2 && pair_live(si, j, o + 1, tokq) ? 2 : 1;
}

// ------------------------------------------------------------ producer ---
template <int D, int PASS>
__device__ void s_producer(const CUtensorMap* tmQ, const CUtensorMap* tmK, const PassArgs& p,
                           SB sm, const SeqInfo* seqs, const Entry* E, UnitIter it) {
  using C = SCfg<D, PASS>;
  using L = SL<D, PASS>;
  const uint32_t q_bytes = (uint32_t)(D * 2 * p.G * p.tokq);
  const uint32_t k_bytes = (uint32_t)(D * 2 * kTile);
  volatile int* abort = sm.abort_flag(L::abort);
  // K tiles stream through L2 once per pass: evict them first (they would
  // otherwise push out the lines every layer reuses)
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
    const SeqInfo si = seqs[e.seq];
    if (!mbar_wait(sm.bar(L::stat_empty), uph ^ 1u, abort, p.status, p.wait_ns)) goto out;
    mbar_arrive_expect_tx(sm.bar(L::stat_full), q_bytes * (uint32_t)e.n_stat);
    for (int i = 0; i < e.n_stat; ++i) {
      const int slot = PASS == 1 ? i : p2_slot(i);
#pragma unroll
      for (int sb = 0; sb < C::kSub; ++sb)
        tma_load_3d(sm.b + L::stat + (sb * C::kStat + slot) * kSubBytes, tmQ,
                    sm.bar(L::stat_full), sb * 64, e.g * p.G,
                    si.start + si.q0 + (e.stat0 + i) * p.tokq);
    }
    stat_issued = 1;
    stat_ph = uph;
    uph ^= 1u;
    for (int st = st0; st < st1; st += C::kStageTiles) {
      const int nt = min(C::kStageTiles, st1 - st);
      if (!mbar_wait(sm.bar(L::empty, stage), sph ^ 1u, abort, p.status, p.wait_ns)) goto out;
      mbar_arrive_expect_tx(sm.bar(L::full, stage), k_bytes * (uint32_t)nt);
      uint8_t* dst = sm.b + L::strm + stage * C::kStageBytes;
      for (int t = 0; t < nt; ++t) {
#pragma unroll
        for (int sb = 0; sb < C::kSub; ++sb)
          tma_load_3d_hint(dst + (sb * C::kStageTiles + t) * kSubBytes, tmK,
                           sm.bar(L::full, stage), sb * 64, e.g,
                           si.start + (e.step0 + st + t) * kTile, k_policy);
      }
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
      if (issued[i]) mbar_wait(sm.bar(L::full, i), issued_ph[i], &zero, p.status, kDrainLimitNs);
    if (stat_issued) mbar_wait(sm.bar(L::stat_full), stat_ph, &zero, p.status, kDrainLimitNs);
  }
}

// ---------------------------------------------------------- MMA issuer ---
// Pass 1: warpgroup w's accumulator = Q tile (stat0 + w) x the stage's K
// tiles (128 or 256 keys).  Pass 2: warpgroup w's accumulator = the stage's
// K tile x Q tiles w and w + 2 (128 or 256 query rows).  Descriptors are
// built once per accumulator and advanced by the k-step's byte offset.
template <int D, int PASS>
__device__ void s_mma(const PassArgs& p, SB sm, const SeqInfo* seqs, const Entry* E, UnitIter it,
                      uint32_t tmem) {
  using C = SCfg<D, PASS>;
  using L = SL<D, PASS>;
  constexpr uint32_t idesc128 = idesc_bf16_f32(128, 128);
  constexpr uint32_t idesc256 = idesc_bf16_f32(128, 256);
  volatile int* abort = sm.abort_flag(L::abort);
  int stage = 0;
  uint32_t sph = 0, uph = 0;
  uint32_t cnt[2] = {0, 0};
  const uint32_t base = smem_addr(sm.b);
  int ei, st0, st1, unit;
  if (p.withhold_mma) goto out;   // testing aid: every accumulator wait runs out
  while (it.next(ei, st0, st1, unit)) {
    const Entry e = E[ei];
    const SeqInfo si = seqs[e.seq];
    if (!mbar_wait(sm.bar(L::stat_full), uph, abort, p.status, p.wait_ns)) goto out;
    uph ^= 1u;
    tc_fence_after();
    for (int st = st0; st < st1; st += C::kStageTiles) {
      const int nt = min(C::kStageTiles, st1 - st);
      const int o = e.step0 + st;
      if (!mbar_wait(sm.bar(L::full, stage), sph, abort, p.status, p.wait_ns)) goto out;
      tc_fence_after();
      const uint32_t sa = base + L::strm + stage * C::kStageBytes;
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        int ncols;
        uint32_t a_base, b_base, a_blk, b_blk;
        if (PASS == 1) {
          ncols = w < e.n_stat ? kTile * p1_live_tiles(si, e.stat0 + w, o, nt, p.tokq) : 0;
          a_base = base + L::stat + w * kSubBytes;         // Q tile w
          a_blk = C::kStat * kSubBytes;
          b_base = sa;                                     // the stage's K tiles
          b_blk = C::kStageTiles * kSubBytes;
        } else {
          const bool ex0 = w < e.n_stat, ex1 = w + 2 < e.n_stat;
          const bool live = (ex0 && pair_live(si, w, o, p.tokq)) ||
                            (ex1 && pair_live(si, w + 2, o, p.tokq));
          ncols = live ? (ex1 ? 2 * kTile : kTile) : 0;
          a_base = sa;                                     // the K tile
          a_blk = kSubBytes;
          b_base = base + L::stat + 2 * w * kSubBytes;     // Q tiles w, w + 2
          b_blk = C::kStat * kSubBytes;
        }
        if (ncols == 0) continue;
        const uint32_t ph = cnt[w] & 1u;
        if (!mbar_wait(sm.bar(L::tempty, w), ph ^ 1u, abort, p.status, p.wait_ns)) goto out;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(w * kAccCols);
        const uint32_t idesc = ncols == kTile ? idesc128 : idesc256;
        const uint64_t da = sdesc_kmajor_sw128(a_base), db = sdesc_kmajor_sw128(b_base);
#pragma unroll
        for (int k = 0; k < C::kKSteps; ++k) {
          // byte offsets within the swizzled blocks, in units of 16 bytes
          const uint32_t oa = ((k >> 2) * a_blk + (k & 3) * 32) >> 4;
          const uint32_t ob = ((k >> 2) * b_blk + (k & 3) * 32) >> 4;
          mma_bf16(d_tmem, da + oa, db + ob, idesc, k > 0 ? 1u : 0u);
        }
        mma_commit(sm.bar(L::tfull, w));
        ++cnt[w];
      }
      mma_commit(sm.bar(L::empty, stage));
      if (++stage == C::kStages) { stage = 0; sph ^= 1u; }
    }
    mma_commit(sm.bar(L::stat_empty));
  }
out:
  // every MMA issued so far must finish before TMEM is released
  mma_commit(sm.bar(L::done));
  int zero = 0;
  mbar_wait(sm.bar(L::done), 0, &zero, p.status, kDoneLimitNs);
}

// ------------------------------------------------------------ epilogue ---
__device__ inline void release_acc(uint64_t* bar, int lane) {
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

template <int D>
__device__ void s_epilogue_p1(const PassArgs& p, SB sm, const SeqInfo* seqs, const Entry* E,
                              UnitIter it, uint32_t tmem) {
  using L = SL<D, 1>;
  const int tid = threadIdx.x;               // 0..255
  const int w = tid >> 7;                     // warpgroup: stationary slot w
  const int t = tid & 127;                    // TMEM lane == packed query row
  const int lane = tid & 31;
  const uint32_t lane_addr = tmem + (uint32_t)(w * kAccCols) + ((uint32_t)((t >> 5) * 32) << 16);
  const int t_tok = t / p.G;                  // token of row t within its Q tile
  const bool t_row = t < p.tokq * p.G;
  volatile int* abort = sm.abort_flag(L::abort);
  uint32_t kp = 0;   // accumulators consumed by this warpgroup
  bool ok = true;    // false after a timeout: skip the work, keep the loop
  int ei, st0, st1, unit;
  while (it.next(ei, st0, st1, unit)) {
    const Entry e = E[ei];
    if (w >= e.n_stat) continue;
    const SeqInfo si = seqs[e.seq];
    const int j = e.stat0 + w;
    const int tok = si.q0 + j * p.tokq + t_tok;
    const int row_tok = t_row && tok < si.len ? tok : -1;
    float m = -INFINITY, l = 0.f;
    for (int st = st0; st < st1; st += 2) {
      const int nt = min(2, st1 - st);
      const int o = e.step0 + st;
      const int n = p1_live_tiles(si, j, o, nt, p.tokq);
      if (n == 0) continue;
      const uint32_t ph = kp & 1u;
      ++kp;
      if (ok && !mbar_wait(sm.bar(L::tfull, w), ph, abort, p.status, p.wait_ns)) ok = false;
      if (!ok) continue;
      tc_fence_after();
      // the accumulator's halves in one loop: one copy of the unrolled
      // arithmetic in the instruction stream
#pragma unroll 1
      for (int h = 0; h < n; ++h) {
        Cols v;
        v.load_wait(lane_addr + (uint32_t)(h * kTile));
        if (h == n - 1) release_acc(sm.bar(L::tempty, w), lane);
        const int nv = row_tok >= 0 ? row_tok - (o + h) * kTile + 1 : 0;
        p1_pair(v, nv > kTile ? kTile : nv, p.scale2, m, l);
      }
    }
    // this unit's row partial; pass 2 merges the partials where it reads the rows
    if (ok && !*abort) p.part1[((size_t)unit * kMaxStat1 + w) * kTile + t] = make_float2(m, l);
  }
}

template <int D>
__device__ void s_epilogue_p2(const PassArgs& p, SB sm, const SeqInfo* seqs, const Entry* E1,
                              const Entry* E, UnitIter it, uint32_t tmem) {
  using L = SL<D, 2>;
  const int tid = threadIdx.x;               // 0..255
  const int w = tid >> 7;                     // warpgroup: Q tiles w and w + 2
  const int t = tid & 127;                    // TMEM lane == key of the K tile
  const int lane = tid & 31;
  const uint32_t lane_addr = tmem + (uint32_t)(w * kAccCols) + ((uint32_t)((t >> 5) * 32) << 16);
  const int bar_wg = 1 + w;                   // named barrier of this warpgroup
  volatile int* abort = sm.abort_flag(L::abort);
  float* bias0 = sm.at<float>(L::bias) + w * kTile;         // Q tile w
  float* bias1 = sm.at<float>(L::bias) + (w + 2) * kTile;   // Q tile w + 2
  uint32_t kp = 0;   // accumulators consumed by this warpgroup
  uint32_t hs = 0;   // column-sum handoffs between the warpgroups
  bool ok = true;
  int ei, st0, st1, unit;
  while (it.next(ei, st0, st1, unit)) {
    const Entry e = E[ei];
    const SeqInfo si = seqs[e.seq];
    const bool ex0 = w < e.n_stat, ex1 = w + 2 < e.n_stat;
    const bool both = e.n_stat > 1;           // warpgroup 1 has tiles: hand its sums over
    // row biases of this warpgroup's tiles (the previous unit's reads are done)
    bar_sync(bar_wg, 128);
    if (ex0) {
      const int js[2] = {w, ex1 ? w + 2 : -1};
      float bs[2];
      qrow_bias<2>(p, E1, si, e.g, js, t, bs);
      bias0[t] = bs[0];
      if (ex1) bias1[t] = bs[1];
    }
    bar_sync(bar_wg, 128);
    const int f0 = si.q0 + w * p.tokq, f1 = si.q0 + (w + 2) * p.tokq;   // first tokens
    const int nc0 = min(p.tokq, si.len - f0) * p.G, nc1 = min(p.tokq, si.len - f1) * p.G;
    float* out = p.scores + (size_t)e.g * p.T + si.start;
    for (int st = st0; st < st1; ++st) {
      const int o = e.step0 + st;
      const int key = o * kTile + t;
      const bool live0 = ex0 && pair_live(si, w, o, p.tokq);
      const bool live1 = ex1 && pair_live(si, w + 2, o, p.tokq);
      float col = 0.f;
      if (live0 || live1) {
        const uint32_t ph = kp & 1u;
        ++kp;
        if (ok && !mbar_wait(sm.bar(L::tfull, w), ph, abort, p.status, p.wait_ns)) ok = false;
        if (ok) {
          tc_fence_after();
          // both Q tiles in one loop: one copy of the unrolled arithmetic
          const int nh = ex1 ? 2 : 1;
#pragma unroll 1
          for (int h = 0; h < nh; ++h) {
            Cols v;
            v.load_wait(lane_addr + (uint32_t)(h * kTile));
            if (h == nh - 1) release_acc(sm.bar(L::tempty, w), lane);
            const bool live = h == 0 ? live0 : live1;
            const int f = h == 0 ? f0 : f1;
            if (live) col += p2_pair(v, key > f ? min((key - f) * p.G, kTile) : 0,
                                     h == 0 ? nc0 : nc1, p.scale2, h == 0 ? bias0 : bias1);
          }
        }
      }
      float score = col;
      if (both) {
        const int sb = (int)(hs & 1u);
        const uint32_t hph = (hs >> 1) & 1u;
        ++hs;
        float* part = sm.at<float>(L::part) + sb * kTile;
        if (w == 1) {
          if (ok && !mbar_wait(sm.bar(L::pfree, sb), hph ^ 1u, abort, p.status, p.wait_ns))
            ok = false;
          part[t] = col;
          __syncwarp();
          if (lane == 0) mbar_arrive(sm.bar(L::pfull, sb));
          continue;
        }
        if (ok && !mbar_wait(sm.bar(L::pfull, sb), hph, abort, p.status, p.wait_ns)) ok = false;
        score = col + part[t];
        __syncwarp();
        if (lane == 0) mbar_arrive(sm.bar(L::pfree, sb));
      } else if (w == 1) {
        continue;
      }
      if (ok && key < si.len) out[key] = score;
    }
  }
}

template <int D, int PASS>
__global__ void __launch_bounds__(kThreads, 1)
    score_sparse_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ PassArgs pa,
                        const __grid_constant__ HostPlan hp) {
  using C = SCfg<D, PASS>;
  using L = SL<D, PASS>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t a0 = smem_addr(smem_raw);
  const SB sm{smem_raw + ((1024u - (a0 & 1023u)) & 1023u)};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr bool p1 = PASS == 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(sm.bar(L::full, i), 1);
      mbar_init(sm.bar(L::empty, i), 1);
    }
    mbar_init(sm.bar(L::stat_full), 1);
    mbar_init(sm.bar(L::stat_empty), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(sm.bar(L::tfull, i), 1);
      mbar_init(sm.bar(L::tempty, i), 4);
      mbar_init(sm.bar(L::pfull, i), 4);
      mbar_init(sm.bar(L::pfree, i), 4);
    }
    mbar_init(sm.bar(L::done), 1);
    *sm.abort_flag(L::abort) = 0;
    fence_mbar_init();
  }
  // rows of Q tiles that TMA never writes (tokq * G < 128) must stay finite
  {
    uint4* z = sm.at<uint4>(L::stat);
    const int n = (int)(L::bias / 16);
    for (int i = threadIdx.x; i < n; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  if (warp == kMmaWarp) tmem_alloc(sm.at<uint32_t>(L::tmem_slot), kTmemCols);
  if (warp == kProducerWarp && lane == 0) { prefetch_tensormap(&tmQ); prefetch_tensormap(&tmK); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.at<uint32_t>(L::tmem_slot);
  // Pass 1 waits for whatever wrote Q, K and cu_seqlens before anything,
  // then lets pass 2 launch; pass 2's copy and MMA warps start at once, only
  // its epilogue waits (below) for pass 1's row partials.
  stage_host_plan(pa, hp, sm.at<LocalPlan>(L::lp));
  if (p1 || pa.lse) {
    pdl_wait();
    pdl_allow_next();
  }
  // the plan: this CTA's own (local plans) or the planner kernel's, in the
  // workspace (pass 1 of a large plan, whose pass 2 the general kernel runs)
  PassArgs q = pa;
  plan_prologue(q, pa, hp, sm.at<LocalPlan>(L::lp), p1, warp);
  const Entry* E = p1 ? q.e1 : q.e2;
  const SeqInfo* seqs = q.seqs;

  UnitIter it;
  const PlanHeader& H = *q.hdr;
  const bool have = it.init(E, p1 ? H.n_e1 : H.n_e2, p1 ? H.s1 : H.s2, p1 ? H.p1 : H.p2,
                            blockIdx.x, (p1 ? H.aligned1 : H.aligned2) != 0);
  if (warp >= kProducerWarp) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProducer));
    if (have && warp == kProducerWarp) {
      if (lane == 0) s_producer<D, PASS>(&tmQ, &tmK, pa, sm, seqs, E, it);
      __syncwarp();
    } else if (have && warp == kMmaWarp) {
      if (lane == 0) s_mma<D, PASS>(pa, sm, seqs, E, it, tmem);
      __syncwarp();
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpilogue));
    if (!p1) {
      pdl_wait();
      pdl_allow_next();
    }
    if (have) {
      if (p1) s_epilogue_p1<D>(pa, sm, seqs, E, it, tmem);
      else s_epilogue_p2<D>(pa, sm, seqs, q.e1, E, it, tmem);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int PASS>
constexpr size_t sparse_smem() { return 1024 + SL<D, PASS>::end; }

static_assert(sparse_smem<128, 1>() <= 227 * 1024 && sparse_smem<128, 2>() <= 227 * 1024,
              "shared memory plan exceeds the opt-in limit");
static_assert(sizeof(HostPlan) + 2 * sizeof(CUtensorMap) + sizeof(PassArgs) + 64 <= 4096,
              "scorer parameters must stay within 4 KB");

template <int D>
cudaError_t launch_sparse_d(const PassArgs& a, const HostPlan& hp, int grid, cudaStream_t st,
                            bool pass2 = true) {
  CUtensorMap mq, mk;
  if (!make_map(&mq, a.Q, a.T, a.Hq, a.q_row_heads, D, a.G, a.tokq) ||
      !make_map(&mk, a.K, a.T, a.Hkv, a.kv_row_heads, D, 1, kTile))
    return cudaErrorInvalidValue;
  const size_t smem1 = sparse_smem<D, 1>(), smem2 = sparse_smem<D, 2>();
  cudaError_t err;
  if ((err = cudaFuncSetAttribute(score_sparse_kernel<D, 1>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1)) !=
          cudaSuccess ||
      (err = cudaFuncSetAttribute(score_sparse_kernel<D, 2>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2)) !=
          cudaSuccess)
    return err;
  if (!a.lse && (err = launch_pdl(score_sparse_kernel<D, 1>, dim3(grid), dim3(kThreads), smem1,
                                  st, mq, mk, a, hp)) != cudaSuccess)
    return err;
  if (!pass2) return cudaSuccess;
  return launch_pdl(score_sparse_kernel<D, 2>, dim3(grid), dim3(kThreads), smem2, st, mq, mk, a,
                    hp);
}

}  // namespace

cudaError_t launch_sparse_passes(const PassArgs& a, const HostPlan* hp, int grid,
                                 cudaStream_t s) {
  static const HostPlan kNone{};
  const HostPlan& h = hp ? *hp : kNone;
  return a.d == 64 ? launch_sparse_d<64>(a, h, grid, s) : launch_sparse_d<128>(a, h, grid, s);
}

cudaError_t launch_sparse_pass1(const PassArgs& a, int grid, cudaStream_t s) {
  static const HostPlan kNone{};
  return a.d == 64 ? launch_sparse_d<64>(a, kNone, grid, s, false)
                   : launch_sparse_d<128>(a, kNone, grid, s, false);
}

}  // namespace waits
