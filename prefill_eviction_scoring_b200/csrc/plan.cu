// Device-side planner: one CTA reads cu_seqlens, finds each sequence's first
// row with non-zero fp32 forgetting-curve weight, and writes the work entries
// of both scorer passes plus their split over the persistent CTAs.  Running
// on the device keeps the whole path asynchronous (no host round trip for
// sequence lengths).  Intermediate values stay in shared memory / registers;
// global memory is only written.
#include "plan_core.cuh"

namespace waits {
namespace {

constexpr int kSmemSeqs = 512;     // sequences kept in shared memory

struct Seqs {
  SeqInfo* sm;   // shared copy (nseq <= kSmemSeqs) or null
  SeqInfo* gm;   // global copy (always written)
  __device__ const SeqInfo& operator[](int i) const { return sm ? sm[i] : gm[i]; }
};

// Entry i of a pass: find its sequence by binary search over the per-
// sequence entry offsets and fill it.
template <bool P1>
__device__ Entry make_entry(const Seqs& S, int nseq, int tokq, int i) {
  int lo = 0, hi = nseq - 1;
  while (lo < hi) {
    const int m = (lo + hi + 1) / 2;
    if ((P1 ? S[m].e1 : S[m].e2) <= i) lo = m; else hi = m - 1;
  }
  Entry e{};
  const SeqInfo& si = S[lo];
  if (P1) fill_entry_p1(tokq, si, lo, i - si.e1, e);
  else fill_entry_p2(tokq, si, lo, i - si.e2, e);
  return e;
}

// Fill, scan and split the entries of one pass over the CTAs; entries are
// regenerated from the sequence table in each sweep rather than re-read.
// When every entry can have at least one CTA of its own (CTA boundaries at
// the rounded positions C_e * P / S of the entries' first steps, every entry
// with at least as many steps as CTAs), each entry gets its own CTAs
// ("aligned"); otherwise CTAs split the global step range.
template <bool P1>
__device__ void plan_pass(const Seqs& S, int nseq, int tokq, int n, int grid, Entry* out,
                          uint32_t* counters, int64_t max_units, int64_t* sh, int64_t* steps,
                          int* units, int* ctas, int* aligned_out, bool* overflow) {
  int64_t carry = 0;
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const int64_t v = i < n ? (int64_t)make_entry<P1>(S, nseq, tokq, i).n_steps : 0;
    int64_t tot;
    block_exclusive_scan(v, &tot, sh);
    carry += tot;
  }
  const int64_t Stot = carry;
  const int64_t P = Stot < (int64_t)grid ? Stot : (int64_t)grid;
  auto cta_at = [&](int64_t c) { return waits::cta_at(c, P, Stot); };
  // can every entry own whole CTAs?
  bool aligned = n <= P && Stot > 0;
  {
    int64_t sb = 0;
    int bad = 0;
    for (int base = 0; base < n && aligned; base += blockDim.x) {
      const int i = base + threadIdx.x;
      const int64_t v = i < n ? (int64_t)make_entry<P1>(S, nseq, tokq, i).n_steps : 0;
      int64_t tot;
      const int64_t c = sb + block_exclusive_scan(v, &tot, sh);
      sb += tot;
      if (i < n) {
        const int64_t nu = cta_at(c + v) - cta_at(c);
        if (nu < 1 || nu > v) bad = 1;
      }
      if (__syncthreads_or(bad)) aligned = false;
    }
  }
  int64_t sb = 0, ub = 0;
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + threadIdx.x;
    Entry e{};
    if (i < n) e = make_entry<P1>(S, nseq, tokq, i);
    int64_t tot;
    const int64_t ex = block_exclusive_scan(i < n ? (int64_t)e.n_steps : 0, &tot, sh);
    e.sbase = sb + ex;
    sb += tot;
    int64_t nu = 0;
    if (i < n) {
      if (aligned) {
        e.first_cta = (int)cta_at(e.sbase);
        nu = cta_at(e.sbase + e.n_steps) - e.first_cta;
      } else {
        const int64_t f = e.sbase * P / Stot;
        const int64_t l = (e.sbase + e.n_steps - 1) * P / Stot;
        e.first_cta = (int)f;
        nu = l - f + 1;
      }
      e.n_units = (int)nu;
    }
    const int64_t ux = block_exclusive_scan(nu, &tot, sh);
    e.unit_base = aligned ? e.first_cta : (int)(ub + ux);   // aligned: unit = CTA
    ub += tot;
    if (i < n) {
      out[i] = e;
      if (counters) counters[i] = 0u;
    }
  }
  *steps = Stot;
  *units = (int)ub;
  *ctas = (int)P;
  *aligned_out = aligned ? 1 : 0;
  if (ub > max_units) *overflow = true;
}

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(PlanArgs p) {
  __shared__ int64_t sh[32];
  __shared__ int s_bad, s_bad_curve;
  __shared__ SeqInfo s_seqs[kSmemSeqs];
  const int tid = threadIdx.x;
  if (tid == 0) s_bad = s_bad_curve = 0;
  pdl_allow_next();
  pdl_wait();
  __syncthreads();
  Seqs S{p.nseq <= kSmemSeqs ? s_seqs : nullptr, p.seqs};

  // 1) per-sequence bounds, first active row, tile counts, entry offsets.
  int64_t c1 = 0, c2 = 0;
  for (int base = 0; base < p.nseq; base += blockDim.x) {
    const int s = base + tid;
    SeqInfo si{};
    int64_t v1 = 0, v2 = 0;
    if (s < p.nseq) {
      bool bad;
      const float a = p.seq_a ? p.seq_a[s] : p.a;
      const int b = p.seq_b ? p.seq_b[s] : p.b;
      si = seq_info(p.cu, s, p.nseq, p.T, p.max_seqlen, p.tokq, a, b, bad);
      if (bad) atomicOr(&s_bad, 1);
      if (!(a >= 0.0f && a <= 3.4e38f && b >= 0)) atomicOr(&s_bad_curve, 1);
      v1 = (int64_t)p.Hkv * groups_p1(si);
      v2 = (int64_t)p.Hkv * groups_p2(si);
    }
    int64_t t1, t2;
    const int64_t x1 = block_exclusive_scan(v1, &t1, sh);
    const int64_t x2 = block_exclusive_scan(v2, &t2, sh);
    if (s < p.nseq) {
      si.e1 = (int)(c1 + x1);
      si.e2 = (int)(c2 + x2);
      if (S.sm) S.sm[s] = si;
      p.seqs[s] = si;
    }
    c1 += t1;
    c2 += t2;
  }
  __syncthreads();
  PlanHeader* H = p.hdr;
  if (s_bad) {
    if (tid == 0) {
      H->status = WAITS_DEV_BAD_SEQLENS;
      H->n_e1 = H->n_e2 = H->n_u1 = H->n_u2 = H->p1 = H->p2 = 0;
      H->s1 = H->s2 = 0;
      H->aligned1 = H->aligned2 = 0;
    }
    return;
  }
  bool overflow = c1 > p.max_e1 || c2 > p.max_e2;
  int64_t S1 = 0, S2 = 0;
  int U1 = 0, U2 = 0, P1 = 0, P2 = 0, A1 = 0, A2 = 0;
  if (!overflow) {
    plan_pass<true>(S, p.nseq, p.tokq, (int)c1, p.grid, p.e1, nullptr, p.max_u1, sh, &S1, &U1,
                    &P1, &A1, &overflow);
    plan_pass<false>(S, p.nseq, p.tokq, (int)c2, p.grid, p.e2, p.c2, p.max_u2, sh, &S2, &U2,
                     &P2, &A2, &overflow);
  }
  if (tid == 0) {
    H->status = (overflow ? WAITS_DEV_PLAN_OVERFLOW : 0u) | (s_bad_curve ? WAITS_DEV_BAD_CURVE : 0u);
    H->n_e1 = overflow ? 0 : (int)c1;
    H->n_e2 = overflow ? 0 : (int)c2;
    H->n_u1 = U1;
    H->n_u2 = U2;
    H->p1 = overflow ? 0 : P1;
    H->p2 = overflow ? 0 : P2;
    H->s1 = S1;
    H->s2 = S2;
    H->aligned1 = A1;
    H->aligned2 = A2;
  }

  // 2) sequences without any active row score 0 everywhere.
  for (int s = 0; s < p.nseq; ++s) {
    const SeqInfo& si = S[s];
    if (si.len > 0 && si.q0 >= si.len) {
      for (int64_t i = tid; i < (int64_t)si.len * p.Hkv; i += blockDim.x) {
        const int g = (int)(i / si.len), k = (int)(i % si.len);
        p.scores[(int64_t)g * p.T + si.start + k] = 0.0f;
      }
    }
  }
}

}  // namespace

cudaError_t launch_plan(const PlanArgs& a, cudaStream_t s) {
  // few sequences: one warp plans alone (shuffle scans, no block barriers)
  const int threads = a.nseq <= 64 ? 32 : kPlanThreads;
  return launch_pdl(plan_kernel, dim3(1), dim3(threads), 0, s, a);
}

namespace {

// One pass of the one-sequence plan: warp_plan_pass's rule, entry by entry.
template <bool P1>
void host_plan_pass(const SeqInfo& si, int tokq, int n, int grid, Entry* out, int64_t* steps,
                    int* units, int* ctas, int* aligned_out) {
  int64_t c[kHostPlanMax], v[kHostPlanMax], f0[kHostPlanMax], f1[kHostPlanMax];
  int64_t S = 0;
  for (int i = 0; i < n; ++i) {
    out[i] = Entry{};
    if (P1) fill_entry_p1(tokq, si, 0, i, out[i]);
    else fill_entry_p2(tokq, si, 0, i, out[i]);
    v[i] = out[i].n_steps;
    c[i] = S;
    S += v[i];
  }
  const int64_t P = S < (int64_t)grid ? S : (int64_t)grid;
  bool aligned = n <= P && S > 0;
  for (int i = 0; aligned && i < n; ++i) {
    f0[i] = cta_at(c[i], P, S);
    f1[i] = cta_at(c[i] + v[i], P, S);
    aligned = f1[i] - f0[i] >= 1 && f1[i] - f0[i] <= v[i];
  }
  int64_t U = 0;
  for (int i = 0; i < n; ++i) {
    Entry& e = out[i];
    int64_t nu;
    e.sbase = c[i];
    if (aligned) {
      e.first_cta = (int)f0[i];
      nu = f1[i] - f0[i];
    } else {
      const int64_t f = c[i] * P / S, l = (c[i] + v[i] - 1) * P / S;
      e.first_cta = (int)f;
      nu = l - f + 1;
    }
    e.n_units = (int)nu;
    e.unit_base = aligned ? e.first_cta : (int)U;
    U += nu;
  }
  *steps = S;
  *units = (int)U;
  *ctas = (int)P;
  *aligned_out = aligned ? 1 : 0;
}

}  // namespace

bool host_plan_single(int T, int max_seqlen, int Hkv, int tokq, float a, int b, int grid,
                      HostPlan* hp) {
  bool bad = false;
  SeqInfo si = seq_info(0, T, 0, 1, T, max_seqlen, tokq, a, b, bad);
  if (bad) return false;
  const int64_t n1 = (int64_t)Hkv * groups_p1(si), n2 = (int64_t)Hkv * groups_p2(si);
  if (n1 > kHostPlanMax || n2 > kHostPlanMax) return false;
  if (si.len > si.q0 && si.nqt > kMaxStat) return false;   // would need stationary K tiles
  si.e1 = 0;
  si.e2 = 0;
  *hp = HostPlan{};
  hp->seq = si;
  PlanHeader& H = hp->hdr;
  H.status = 0u;
  H.n_e1 = (int)n1;
  H.n_e2 = (int)n2;
  host_plan_pass<true>(si, tokq, (int)n1, grid, hp->e1, &H.s1, &H.n_u1, &H.p1, &H.aligned1);
  host_plan_pass<false>(si, tokq, (int)n2, grid, hp->e2, &H.s2, &H.n_u2, &H.p2, &H.aligned2);
  return true;
}

}  // namespace waits
