// Walking the work plan: which steps (streamed tiles) of which entries a
// persistent CTA owns, and the per-tile geometry both scorer passes share.
#pragma once

#include "waits_internal.cuh"

namespace waits {

// Two ways to split a pass's steps over its P CTAs, chosen by the planner:
//  * by global step: CTA `cta` owns global steps [ceil(cta*S/P),
//    ceil((cta+1)*S/P)); a maximal run of them inside one entry is a unit,
//    so a CTA may hold pieces of several entries;
//  * entry by entry ("aligned"): entry e owns CTAs [first_cta, first_cta +
//    n_units), which split its steps evenly; every CTA has exactly one unit,
//    so none pays for a second set of stationary tiles.
struct UnitIter {
  const Entry* E;
  int nE;
  int64_t hi;     // end of this CTA's step range
  int e;          // current entry
  int64_t pos;    // next global step
  int cta;

  __device__ bool init(const Entry* E_, int nE_, int64_t S, int P, int cta_, bool aligned) {
    E = E_; nE = nE_; cta = cta_;
    if (cta >= P || nE <= 0 || S <= 0) return false;
    if (aligned) {
      int a = 0, b = nE - 1;
      while (a < b) {
        const int m = (a + b + 1) / 2;
        if (E[m].first_cta <= cta) a = m; else b = m - 1;
      }
      const Entry& en = E[a];
      const int64_t u = cta - en.first_cta, nu = en.n_units, n = en.n_steps;
      if (u < 0 || u >= nu) return false;
      // split the entry's cost evenly: its last n_masked steps (on the
      // causal diagonal) cost kMaskedCost each, the others 1.  Every unit
      // must keep a step (pass 2 reads every unit's partials), which holds
      // when a unit's share of the cost is at least one masked step; else
      // the steps are split evenly.
      int64_t m = en.n_masked < 0 ? 0 : (en.n_masked > n ? n : en.n_masked);
      if (n - m + m * kMaskedCost < nu * kMaskedCost) m = 0;
      const int64_t plain = n - m, cost = plain + m * kMaskedCost;
      auto step_at = [&](int64_t c) {
        return c <= plain ? c : plain + (c - plain + kMaskedCost - 1) / kMaskedCost;
      };
      e = a;
      pos = en.sbase + step_at(u * cost / nu);
      hi = en.sbase + step_at((u + 1) * cost / nu);
      return pos < hi;
    }
    const int64_t lo = ((int64_t)cta * S + P - 1) / P;
    hi = ((int64_t)(cta + 1) * S + P - 1) / P;
    if (lo >= hi) return false;
    int a = 0, b = nE - 1;
    while (a < b) {
      const int m = (a + b + 1) / 2;
      if (E[m].sbase <= lo) a = m; else b = m - 1;
    }
    e = a;
    pos = lo;
    return true;
  }
  // Next unit: entry index, local step range [st0, st1) and unit slot.
  __device__ bool next(int& ei, int& st0, int& st1, int& unit) {
    if (pos >= hi || e >= nE) return false;
    const Entry& en = E[e];
    const int64_t end = en.sbase + en.n_steps;
    const int64_t stop = end < hi ? end : hi;
    ei = e;
    st0 = (int)(pos - en.sbase);
    st1 = (int)(stop - en.sbase);
    unit = en.unit_base + (cta - en.first_cta);
    pos = stop;
    if (stop == end) ++e;
    return true;
  }
};

// Geometry of Q tile j of a sequence (packed rows r = token * G + head).
__device__ inline int qtile_first_tok(const SeqInfo& si, int j, int tokq) {
  return si.q0 + j * tokq;
}
__device__ inline int qtile_last_tok(const SeqInfo& si, int j, int tokq) {
  const int e = si.q0 + (j + 1) * tokq;
  return (e < si.len ? e : si.len) - 1;
}
// Some row of Q tile j sees some key of K tile kt (causal).
__device__ inline bool pair_live(const SeqInfo& si, int j, int kt, int tokq) {
  return qtile_last_tok(si, j, tokq) >= kt * kTile;
}
// Every row of Q tile j sees every key of K tile kt.
__device__ inline bool pair_full(const SeqInfo& si, int j, int kt, int tokq) {
  return qtile_first_tok(si, j, tokq) >= kt * kTile + kTile - 1;
}

__device__ inline float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Largest partial sum kept before the reference maximum of a row is moved
// up (2^64: far from fp32 overflow even after adding a whole tile).
constexpr float kRebaseLimit = 1.8446744073709552e19f;

}  // namespace waits
