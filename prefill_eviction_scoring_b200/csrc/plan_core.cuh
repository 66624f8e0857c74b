// Work-plan rules shared by the planner kernel and the scorer's local plan:
// per-sequence bounds and first active row, the stationary groups of each
// pass, the fields of an entry, and the split of an entry's steps over the
// persistent CTAs.  The local plan (`warp_plan`) is the same computation by
// one warp, for plans small enough to be rebuilt by every CTA in shared
// memory (no planner kernel, no global plan).
#pragma once

#include "waits_internal.cuh"

namespace waits {

__host__ __device__ inline int ceil_div(int x, int y) { return (x + y - 1) / y; }

// Number of stationary groups per (sequence, KV head) for each pass.
__host__ __device__ inline int groups_p1(const SeqInfo& si) {
  return si.len > si.q0 ? ceil_div(si.nqt, kMaxStat1) : 0;
}
__host__ __device__ inline int groups_p2(const SeqInfo& si) {
  if (si.len <= si.q0) return 0;
  return si.nqt <= kMaxStat ? 1 : ceil_div(si.nkt, kMaxStat);
}

// Last position covered by Q tile j (sequence-local).
__host__ __device__ inline int qtile_last_token(const SeqInfo& si, int j, int tokq) {
  const int e = si.q0 + (j + 1) * tokq;
  return (e < si.len ? e : si.len) - 1;
}

// Sequence s with offsets [lo, hi): validity, first row with non-zero fp32
// weight and tile counts (entry offsets e1 / e2 are left to the caller).
// Invalid offsets give an empty sequence and set `bad`.
__host__ __device__ inline SeqInfo seq_info(int lo, int hi, int s, int nseq, int T,
                                            int max_seqlen, int tokq, float a, int b, bool& bad) {
  SeqInfo si{};
  bad = (s == 0 && lo != 0) || hi < lo || hi > T || (hi - lo) > max_seqlen ||
        (s == nseq - 1 && hi != T);
  // an invalid curve (only routed calls can pass one) leaves the sequence
  // without active rows: its scores are zero
  const bool curve_ok = a >= 0.0f && a <= 3.4e38f && b >= 0;
  si.start = lo;
  si.len = bad ? 0 : hi - lo;
  si.a = curve_ok ? a : 0.0f;
  si.b = curve_ok ? b : 0;
  si.q0 = curve_ok ? first_active_row(si.len, a, b) : si.len;
  si.nqt = (si.len - si.q0 + tokq - 1) / tokq;
  si.nkt = (si.len + kTile - 1) / kTile;
  return si;
}

// The same, reading the offsets of sequence s from cu_seqlens.
__device__ inline SeqInfo seq_info(const int32_t* cu, int s, int nseq, int T, int max_seqlen,
                                   int tokq, float a, int b, bool& bad) {
  return seq_info(cu[s], cu[s + 1], s, nseq, T, max_seqlen, tokq, a, b, bad);
}

__host__ __device__ inline void fill_entry_p1(int tokq, const SeqInfo& si, int s, int local, Entry& e) {
  const int ng = groups_p1(si);
  e.seq = s;
  e.g = local / ng;
  e.grp = local % ng;
  e.mode = kModeP1;
  e.stat0 = e.grp * kMaxStat1;
  e.n_stat = min(kMaxStat1, si.nqt - e.stat0);
  const int last = qtile_last_token(si, e.stat0 + e.n_stat - 1, tokq);
  e.step0 = 0;
  e.n_steps = last / kTile + 1;
  // K tiles from the one holding the group's first row on cross the diagonal
  e.n_masked = e.n_steps - (si.q0 + e.stat0 * tokq) / kTile;
}

__host__ __device__ inline void fill_entry_p2(int tokq, const SeqInfo& si, int s, int local, Entry& e) {
  const int ng = groups_p2(si);
  e.seq = s;
  e.g = local / ng;
  e.grp = local % ng;
  if (si.nqt <= kMaxStat) {
    e.mode = kModeP2Q;
    e.stat0 = 0;
    e.n_stat = si.nqt;
    e.step0 = 0;
    e.n_steps = si.nkt;
    // K tiles from the one holding the first active row on cross the diagonal
    e.n_masked = e.n_steps - si.q0 / kTile;
  } else {
    e.mode = kModeP2K;
    e.stat0 = e.grp * kMaxStat;
    e.n_stat = min(kMaxStat, si.nkt - e.stat0);
    // first Q tile whose last position reaches the group's first key
    const int x = e.stat0 * kTile - si.q0;
    const int j0 = x > 0 ? x / tokq : 0;
    e.step0 = j0;
    e.n_steps = si.nqt - j0;
  }
}

// CTA boundary nearest to global step c when P CTAs share S steps (32-bit
// arithmetic when c * P + S / 2 fits it, c <= S).
__host__ __device__ inline int64_t cta_at(int64_t c, int64_t P, int64_t S) {
  if (S * P + S / 2 <= 0xFFFFFFFFll)
    return (int64_t)(((uint32_t)c * (uint32_t)P + (uint32_t)(S / 2)) / (uint32_t)S);
  return (c * P + S / 2) / S;
}

// ------------------------------------------------------------ local plan ---
constexpr int kLocalMax = 32;   // sequences, and entries per pass, of a local plan

struct LocalPlan {
  SeqInfo seqs[kLocalMax];
  Entry e1[kLocalMax];
  Entry e2[kLocalMax];
  PlanHeader hdr;
};

// ------------------------------------------------------------- host plan ---
// A batch of one sequence can only be valid as cu_seqlens = {0, T}, so its
// plan follows from the call's scalars: the host builds it (the same rules
// as warp_plan with both passes) and hands it to the scorer as a kernel
// parameter; each CTA copies it and checks cu_seqlens instead of planning.
constexpr int kHostPlanMax = 24;   // entries per pass (keeps the parameter under 4 KB)

struct __align__(16) HostPlan {
  PlanHeader hdr;
  SeqInfo seq;
  Entry e1[kHostPlanMax];
  Entry e2[kHostPlanMax];
};

// Builds the plan of the batch {0, T}; false (nothing built) when the
// device must plan instead: an invalid or empty batch, more entries than
// kHostPlanMax, or a pass-2 entry with stationary K tiles.
bool host_plan_single(int T, int max_seqlen, int Hkv, int tokq, float a, int b, int grid,
                      HostPlan* hp);

__device__ inline int64_t warp_exclusive_scan(int64_t v, int64_t* total) {
  const int lane = threadIdx.x & 31;
  int64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  *total = __shfl_sync(0xffffffffu, x, 31);
  return x - v;
}

// One pass's entries, one per lane (n <= 32), split over `grid` CTAs by the
// planner kernel's rule: when every entry can own whole CTAs, each gets the
// CTAs nearest to its share of the steps ("aligned", unit = CTA); otherwise
// CTAs split the global step range and an entry's units are numbered in
// entry order.
template <bool P1>
__device__ inline void warp_plan_pass(const SeqInfo* seqs, int nseq, int tokq, int n, int grid,
                                      Entry* out, int64_t* steps, int* units, int* ctas,
                                      int* aligned_out) {
  const int i = threadIdx.x & 31;
  Entry e{};
  if (i < n) {
    int s = 0;
    for (int k = 1; k < nseq; ++k)
      if ((P1 ? seqs[k].e1 : seqs[k].e2) <= i) s = k;
    const SeqInfo& si = seqs[s];
    if (P1) fill_entry_p1(tokq, si, s, i - si.e1, e);
    else fill_entry_p2(tokq, si, s, i - si.e2, e);
  }
  const int64_t v = i < n ? (int64_t)e.n_steps : 0;
  int64_t Stot;
  const int64_t c = warp_exclusive_scan(v, &Stot);
  const int64_t P = Stot < (int64_t)grid ? Stot : (int64_t)grid;
  bool aligned = n <= P && Stot > 0;
  int64_t f0 = 0, f1 = 0;   // the entry's CTA boundaries under the aligned split
  if (aligned) {
    bool ok = true;
    if (i < n) {
      f0 = cta_at(c, P, Stot);
      f1 = cta_at(c + v, P, Stot);
      ok = f1 - f0 >= 1 && f1 - f0 <= v;
    }
    aligned = __all_sync(0xffffffffu, ok);
  }
  int64_t nu = 0;
  if (i < n) {
    e.sbase = c;
    if (aligned) {
      e.first_cta = (int)f0;
      nu = f1 - f0;
    } else {
      const int64_t f = c * P / Stot, l = (c + v - 1) * P / Stot;
      e.first_cta = (int)f;
      nu = l - f + 1;
    }
    e.n_units = (int)nu;
  }
  int64_t U;
  const int64_t ux = warp_exclusive_scan(nu, &U);
  e.unit_base = aligned ? e.first_cta : (int)ux;
  if (i < n) out[i] = e;
  *steps = Stot;
  *units = (int)U;
  *ctas = (int)P;
  *aligned_out = aligned ? 1 : 0;
}

// The whole plan for nseq <= kLocalMax sequences by one warp (all 32 lanes):
// sequence table, pass-1 entries and (with_p2) pass-2 entries into `lp`.
// Either pass having more than kLocalMax entries, or a pass-2 entry that
// would need stationary K tiles, sets WAITS_DEV_PLAN_OVERFLOW; invalid
// offsets set WAITS_DEV_BAD_SEQLENS; either way no entries are planned (both
// passes check both, so each sees the same status).
__device__ inline void warp_plan(const int32_t* cu, int nseq, int T, int max_seqlen, int Hkv,
                                 int tokq, float a, int b, int grid, bool with_p2,
                                 LocalPlan& lp) {
  const int lane = threadIdx.x & 31;
  SeqInfo si{};
  bool bad = false, p2k = false;
  int64_t v1 = 0, v2 = 0;
  if (lane < nseq && nseq <= kLocalMax) {
    si = seq_info(cu, lane, nseq, T, max_seqlen, tokq, a, b, bad);
    v1 = (int64_t)Hkv * groups_p1(si);
    v2 = (int64_t)Hkv * groups_p2(si);
    p2k = si.len > si.q0 && si.nqt > kMaxStat;
  }
  int64_t n1, n2;
  si.e1 = (int)warp_exclusive_scan(v1, &n1);
  si.e2 = (int)warp_exclusive_scan(v2, &n2);
  if (lane < nseq && nseq <= kLocalMax) lp.seqs[lane] = si;
  const bool any_bad = __any_sync(0xffffffffu, bad);
  const bool overflow = nseq > kLocalMax || n1 > kLocalMax || n2 > kLocalMax ||
                        __any_sync(0xffffffffu, p2k);
  __syncwarp();
  PlanHeader& H = lp.hdr;
  int64_t S1 = 0, S2 = 0;
  int U1 = 0, U2 = 0, P1 = 0, P2 = 0, A1 = 0, A2 = 0;
  if (!any_bad && !overflow) {
    warp_plan_pass<true>(lp.seqs, nseq, tokq, (int)n1, grid, lp.e1, &S1, &U1, &P1, &A1);
    if (with_p2)
      warp_plan_pass<false>(lp.seqs, nseq, tokq, (int)n2, grid, lp.e2, &S2, &U2, &P2, &A2);
  }
  if (lane == 0) {
    const bool ok = !any_bad && !overflow;
    H.status = any_bad ? WAITS_DEV_BAD_SEQLENS : (overflow ? WAITS_DEV_PLAN_OVERFLOW : 0u);
    H.n_e1 = ok ? (int)n1 : 0;
    H.n_e2 = ok && with_p2 ? (int)n2 : 0;
    H.n_u1 = U1;
    H.n_u2 = U2;
    H.p1 = ok ? P1 : 0;
    H.p2 = ok ? P2 : 0;
    H.s1 = S1;
    H.s2 = S2;
    H.aligned1 = A1;
    H.aligned2 = A2;
  }
  __syncwarp();
}

}  // namespace waits
