// Device-side planner: one CTA reads cu_seqlens, finds each sequence's first
// row with non-zero fp32 forgetting-curve weight, and writes the work entries
// of both scorer passes plus their split over the persistent CTAs.  Running
// on the device keeps the whole path asynchronous (no host round trip for
// sequence lengths).
#include "waits_internal.cuh"

namespace waits {
namespace {

__device__ inline int ceil_div(int x, int y) { return (x + y - 1) / y; }

// Number of stationary groups per (sequence, KV head) for each pass.
__device__ inline int groups_p1(const SeqInfo& si) {
  return si.len > si.q0 ? ceil_div(si.nqt, kMaxStat) : 0;
}
__device__ inline int groups_p2(const SeqInfo& si) {
  if (si.len <= si.q0) return 0;
  return si.nqt <= kMaxStat ? 1 : ceil_div(si.nkt, kMaxStat);
}

// Last packed-token position covered by Q tile j (sequence-local).
__device__ inline int qtile_last_token(const SeqInfo& si, int j, int tokq) {
  const int e = si.q0 + (j + 1) * tokq;
  return (e < si.len ? e : si.len) - 1;
}

__device__ void fill_entry_p1(const PlanArgs& p, const SeqInfo& si, int s, int local, Entry& e) {
  const int ng = groups_p1(si);
  e.seq = s;
  e.g = local / ng;
  e.grp = local % ng;
  e.mode = kModeP1;
  e.stat0 = e.grp * kMaxStat;
  e.n_stat = min(kMaxStat, si.nqt - e.stat0);
  const int last = qtile_last_token(si, e.stat0 + e.n_stat - 1, p.tokq);
  e.step0 = 0;
  e.n_steps = last / kTile + 1;
}

__device__ void fill_entry_p2(const PlanArgs& p, const SeqInfo& si, int s, int local, Entry& e) {
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
  } else {
    e.mode = kModeP2K;
    e.stat0 = e.grp * kMaxStat;
    e.n_stat = min(kMaxStat, si.nkt - e.stat0);
    // first Q tile whose last position reaches the group's first key
    const int x = e.stat0 * kTile - si.q0;
    const int j0 = x > 0 ? x / p.tokq : 0;
    e.step0 = j0;
    e.n_steps = si.nqt - j0;
  }
}

// Scan entry step counts, then assign consecutive steps to CTAs.
__device__ void split_steps(Entry* E, int n, int grid, int64_t max_units, int64_t* sh,
                            int64_t* out_steps, int* out_units, int* out_ctas, bool* overflow) {
  int64_t carry = 0;
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const int64_t v = i < n ? (int64_t)E[i].n_steps : 0;
    int64_t tot;
    const int64_t ex = block_exclusive_scan(v, &tot, sh);
    if (i < n) E[i].sbase = carry + ex;
    carry += tot;
  }
  __syncthreads();
  const int64_t S = carry;
  const int64_t P = S < (int64_t)grid ? S : (int64_t)grid;
  carry = 0;
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + threadIdx.x;
    int64_t nu = 0;
    if (i < n) {
      const int64_t f = E[i].sbase * P / S;
      const int64_t l = (E[i].sbase + E[i].n_steps - 1) * P / S;
      E[i].first_cta = (int)f;
      nu = l - f + 1;
      E[i].n_units = (int)nu;
    }
    int64_t tot;
    const int64_t ex = block_exclusive_scan(nu, &tot, sh);
    if (i < n) E[i].unit_base = (int)(carry + ex);
    carry += tot;
  }
  *out_steps = S;
  *out_units = (int)carry;
  *out_ctas = (int)P;
  if (carry > max_units) *overflow = true;
}

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(PlanArgs p) {
  __shared__ int64_t sh[32];
  __shared__ int s_bad;
  __shared__ int64_t s_n1, s_n2;
  const int tid = threadIdx.x;
  if (tid == 0) { s_bad = 0; p.hdr->status = 0u; }
  __syncthreads();

  // 1) per-sequence bounds, first active row, tile counts.
  for (int s = tid; s < p.nseq; s += blockDim.x) {
    const int lo = p.cu[s], hi = p.cu[s + 1];
    bool bad = (s == 0 && lo != 0) || hi < lo || hi > p.T || (hi - lo) > p.max_seqlen ||
               (s == p.nseq - 1 && hi != p.T);
    SeqInfo si{};
    si.start = lo;
    si.len = bad ? 0 : hi - lo;
    si.q0 = first_active_row(si.len, p.a, p.b);
    si.nqt = (si.len - si.q0 + p.tokq - 1) / p.tokq;
    si.nkt = (si.len + kTile - 1) / kTile;
    p.seqs[s] = si;
    if (bad) atomicOr(&s_bad, 1);
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) {
      p.hdr->status = WAITS_DEV_BAD_SEQLENS;
      p.hdr->n_e1 = p.hdr->n_e2 = 0;
      p.hdr->n_u1 = p.hdr->n_u2 = 0;
      p.hdr->p1 = p.hdr->p2 = 0;
      p.hdr->s1 = p.hdr->s2 = 0;
    }
    return;
  }

  // 2) entry offsets per sequence.
  int64_t c1 = 0, c2 = 0;
  for (int base = 0; base < p.nseq; base += blockDim.x) {
    const int s = base + tid;
    int64_t v1 = 0, v2 = 0;
    if (s < p.nseq) {
      v1 = (int64_t)p.Hkv * groups_p1(p.seqs[s]);
      v2 = (int64_t)p.Hkv * groups_p2(p.seqs[s]);
    }
    int64_t t1, t2;
    const int64_t x1 = block_exclusive_scan(v1, &t1, sh);
    const int64_t x2 = block_exclusive_scan(v2, &t2, sh);
    if (s < p.nseq) { p.seqs[s].e1 = (int)(c1 + x1); p.seqs[s].e2 = (int)(c2 + x2); }
    c1 += t1;
    c2 += t2;
  }
  if (tid == 0) { s_n1 = c1; s_n2 = c2; }
  __syncthreads();
  const int64_t n1 = s_n1, n2 = s_n2;
  bool overflow = n1 > p.max_e1 || n2 > p.max_e2;

  if (!overflow) {
    // 3) entries (sequence found by binary search over the offsets).
    for (int64_t i = tid; i < n1; i += blockDim.x) {
      int lo = 0, hi = p.nseq - 1;
      while (lo < hi) { const int m = (lo + hi + 1) / 2; if (p.seqs[m].e1 <= i) lo = m; else hi = m - 1; }
      Entry e{};
      fill_entry_p1(p, p.seqs[lo], lo, (int)(i - p.seqs[lo].e1), e);
      p.e1[i] = e;
      p.c1[i] = 0u;
    }
    for (int64_t i = tid; i < n2; i += blockDim.x) {
      int lo = 0, hi = p.nseq - 1;
      while (lo < hi) { const int m = (lo + hi + 1) / 2; if (p.seqs[m].e2 <= i) lo = m; else hi = m - 1; }
      Entry e{};
      fill_entry_p2(p, p.seqs[lo], lo, (int)(i - p.seqs[lo].e2), e);
      p.e2[i] = e;
      p.c2[i] = 0u;
    }
    __syncthreads();
    // 4) split steps over CTAs.
    int64_t S1, S2;
    int U1, U2, P1, P2;
    bool ov = false;
    split_steps(p.e1, (int)n1, p.grid, p.max_u1, sh, &S1, &U1, &P1, &ov);
    __syncthreads();
    split_steps(p.e2, (int)n2, p.grid, p.max_u2, sh, &S2, &U2, &P2, &ov);
    overflow = overflow || ov;
    if (tid == 0) {
      p.hdr->n_e1 = overflow ? 0 : (int)n1;
      p.hdr->n_e2 = overflow ? 0 : (int)n2;
      p.hdr->n_u1 = U1; p.hdr->n_u2 = U2;
      p.hdr->p1 = overflow ? 0 : P1;
      p.hdr->p2 = overflow ? 0 : P2;
      p.hdr->s1 = S1; p.hdr->s2 = S2;
    }
  } else if (tid == 0) {
    p.hdr->n_e1 = p.hdr->n_e2 = 0;
    p.hdr->p1 = p.hdr->p2 = 0;
  }
  if (overflow && tid == 0) atomicOr(&p.hdr->status, WAITS_DEV_PLAN_OVERFLOW);

  // 5) sequences without any active row score 0 everywhere.
  for (int s = 0; s < p.nseq; ++s) {
    const SeqInfo si = p.seqs[s];
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
  plan_kernel<<<1, kPlanThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace waits
