"""fp64 restatement of WAITS prefill scoring, selection and compaction.

Test infrastructure (see the package docstring): never imported by the
product path.

Source: the WAITS README (stig.sh/Dirac-Notation/A2SF).

* Opening summary: keys are retained by an accumulative attention score in
  which every query row q is weighted by the sigmoid forgetting curve
  ``w[q] = 1 / (1 + exp(-a * (q - (N - b - 0.5))))``; a=0 gives H2O,
  a->inf with b=1 gives TOVA, a->inf with b=window gives SnapKV.
* Quickstart: ``recent_budget`` (R) and ``select_budget`` (B) parameters of
  ``init_cache``.

Readings where the page is silent (each one is listed in the design notes):

* q is the 0-based position inside its own sequence and N is that
  sequence's prompt length (only this makes b=1 keep exactly the last row in
  the a->inf limit).
* The attention is causal softmax over the prompt, scaled by 1/sqrt(d).
* The score of a KV head is the sum over the query heads that share it
  (grouped-query attention, head h uses KV head h // G).
* B is the total budget: the last R positions are always kept and the B-R
  best of the rest by score are added; ties go to the lower index; N <= B
  keeps everything.
* Kept indices are reported in ascending order, padded with -1; the
  compacted cache is zero beyond the kept length.

Inputs are numpy arrays: Q ``[T, Hq, d]``, K and V ``[T, Hkv, d]`` holding
bf16-representable values (any float dtype; upcast to fp64 is exact), packed
"THD" with int ``cu_seqlens`` ``[nseq + 1]``.
"""

from __future__ import annotations

import numpy as np


def forgetting_curve(q, N, a, b):
    """w[q] of the WAITS opening summary, in fp64.

    ``q`` may be any real array (the curve is also evaluated between integer
    rows by the tests); ``N`` is the sequence length, ``a`` the slope and
    ``b`` the window.  exp overflow to +inf yields w = 0 exactly, which is
    the correct limit.
    """
    q = np.asarray(q, dtype=np.float64)
    centre = float(N) - float(b) - 0.5
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-float(a) * (q - centre)))


def _seq_bounds(cu_seqlens):
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    return [(int(cu[i]), int(cu[i + 1])) for i in range(len(cu) - 1)]


def score(Q, K, cu_seqlens, a, b, *, row_block=512, last=None):
    """Accumulative forgetting-curve attention score, fp64.

    For every sequence, query head h and KV head g = h // G:
    ``L[q, k] = Q[q, h] . K[k, g] / sqrt(d)`` for k <= q, ``P = softmax_k L``,
    ``s[g, k] += sum_q w[q] * P[q, k]`` (WAITS opening summary).

    Rows whose fp64 weight is exactly 0.0 are skipped; that is exact.
    Rows are processed in blocks of ``row_block`` only to bound memory: every
    row is an independent softmax, so the block size cannot change a value.

    With ``last`` only the last ``last`` rows of each sequence are summed:
    a key k receives attention only from rows q >= k, so the scores of the
    last ``last`` keys of each sequence are then exact (the rest are partial
    sums).  That makes long sequences checkable key by key at their tail.

    Returns ``s`` of shape ``[Hkv, T]`` (fp64), indexed by packed token.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    if Hq % Hkv:
        raise ValueError("query heads must be a multiple of KV heads")
    G = Hq // Hkv
    inv_sqrt_d = 1.0 / np.sqrt(float(d))
    s = np.zeros((Hkv, T), dtype=np.float64)
    for lo, hi in _seq_bounds(cu_seqlens):
        N = hi - lo
        if N == 0:
            continue
        w = forgetting_curve(np.arange(N), N, a, b)
        rows = np.nonzero(w != 0.0)[0]
        if last is not None:
            rows = rows[rows >= N - int(last)]
        keys = np.arange(N)
        for h in range(Hq):
            g = h // G
            Kg = K[lo:hi, g, :]
            for start in range(0, len(rows), row_block):
                q = rows[start:start + row_block]
                L = (Q[lo + q, h, :] @ Kg.T) * inv_sqrt_d
                L[keys[None, :] > q[:, None]] = -np.inf
                m = L.max(axis=1, keepdims=True)
                E = np.exp(L - m)
                P = E / E.sum(axis=1, keepdims=True)
                s[g, lo:hi] += (w[q][:, None] * P).sum(axis=0)
    return s


def row_lse(Q, K, cu_seqlens, last=None):
    """Natural-log log-sum-exp of every causal attention row, fp64.

    ``lse[h, t] = log sum_{k <= q} exp(Q[t, h] . K[lo + k, g] / sqrt(d))``
    for packed token ``t = lo + q`` of a sequence starting at ``lo``, with
    g = h // G: the normaliser of the causal softmax whose probabilities the
    WAITS score accumulates (opening summary).  It is what a FlashAttention
    forward returns as its row LSE, and what the caller hands to the scorer
    to skip the row-statistics pass.  Every row is computed, whatever its
    weight, unless ``last`` is given: then only the last ``last`` rows of
    each sequence are, and the others are NaN.

    Returns ``lse`` of shape ``[Hq, T]`` (fp64).
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    if Hq % Hkv:
        raise ValueError("query heads must be a multiple of KV heads")
    G = Hq // Hkv
    inv_sqrt_d = 1.0 / np.sqrt(float(d))
    lse = np.full((Hq, T), np.nan if last is not None else 0.0, dtype=np.float64)
    for lo, hi in _seq_bounds(cu_seqlens):
        N = hi - lo
        if N == 0:
            continue
        keys = np.arange(N)
        first = 0 if last is None else max(0, N - int(last))
        for h in range(Hq):
            Kg = K[lo:hi, h // G, :]
            for start in range(first, N, 512):
                q = np.arange(start, min(N, start + 512))
                L = (Q[lo + q, h, :] @ Kg.T) * inv_sqrt_d
                L[keys[None, :] > q[:, None]] = -np.inf
                m = L.max(axis=1)
                lse[h, lo + q] = m + np.log(np.exp(L - m[:, None]).sum(axis=1))
    return lse


def select(s, cu_seqlens, R, B):
    """Kept positions per (sequence, KV head), WAITS Quickstart budgets.

    Keeps the recent window [N-R, N) and the B-R highest-scoring positions of
    [0, N-R), ordering by score descending then index ascending (so ties go
    to the lower index).  N <= B keeps all N positions.

    Returns ``idx`` int32 ``[nseq, Hkv, B]`` (sequence-local, ascending,
    padded with -1) and ``kept_len`` int32 ``[nseq]``.
    """
    s = np.asarray(s)
    Hkv = s.shape[0]
    if not (0 <= R <= B and B >= 1):
        raise ValueError("need 0 <= R <= B and B >= 1")
    bounds = _seq_bounds(cu_seqlens)
    idx = np.full((len(bounds), Hkv, B), -1, dtype=np.int32)
    kept_len = np.zeros(len(bounds), dtype=np.int32)
    for i, (lo, hi) in enumerate(bounds):
        N = hi - lo
        if N <= B:
            kept_len[i] = N
            idx[i, :, :N] = np.arange(N, dtype=np.int32)
            continue
        kept_len[i] = B
        pool = N - R
        for g in range(Hkv):
            sc = s[g, lo:lo + pool]
            # lexsort sorts by the last key first: score descending, then index.
            order = np.lexsort((np.arange(pool), -sc))
            kept = np.concatenate([order[:B - R], np.arange(pool, N)])
            idx[i, g, :] = np.sort(kept).astype(np.int32)
    return idx, kept_len


def compact(K, V, cu_seqlens, idx, kept_len, B):
    """Dense compacted cache ``K'[s, g, j] = K[cu[s] + idx[s, g, j], g]``.

    Same for V; rows j >= kept_len[s] are zero.  Works on any dtype (pass the
    raw bf16 bit patterns for a bit-exact comparison).  Returns arrays of
    shape ``[nseq, Hkv, B, d]``.
    """
    K = np.asarray(K)
    V = np.asarray(V)
    bounds = _seq_bounds(cu_seqlens)
    Hkv, d = K.shape[1], K.shape[2]
    Ko = np.zeros((len(bounds), Hkv, B, d), dtype=K.dtype)
    Vo = np.zeros((len(bounds), Hkv, B, d), dtype=V.dtype)
    for i, (lo, _hi) in enumerate(bounds):
        n = int(kept_len[i])
        for g in range(Hkv):
            rows = lo + idx[i, g, :n].astype(np.int64)
            Ko[i, g, :n] = K[rows, g]
            Vo[i, g, :n] = V[rows, g]
    return Ko, Vo


def decode_attention(q, K_cache, V_cache, cache_len):
    """One decode step of attention over the compacted cache, fp64.

    After prefill the model generates from the compressed cache (WAITS
    README, Quickstart: ``model.generate`` after ``init_cache``).  For
    sequence s and query head h (KV head g = h // G):
    ``o[s, h] = sum_{j < cache_len[s]} softmax_j(q[s, h] . K[s, g, j] / sqrt(d)) V[s, g, j]``
    and ``lse[s, h]`` = the natural-log normaliser of that softmax.

    q ``[nseq, Hq, d]``, K_cache and V_cache ``[nseq, Hkv, C, d]`` (C slots,
    the first cache_len[s] valid), cache_len ``[nseq]``.  A sequence with an
    empty cache gets o = 0 and lse = -inf.  Returns ``(o, lse)``.
    """
    q = np.asarray(q, dtype=np.float64)
    Kc = np.asarray(K_cache, dtype=np.float64)
    Vc = np.asarray(V_cache, dtype=np.float64)
    nseq, Hq, d = q.shape
    Hkv = Kc.shape[1]
    G = Hq // Hkv
    o = np.zeros((nseq, Hq, d))
    lse = np.full((nseq, Hq), -np.inf)
    for s in range(nseq):
        n = int(cache_len[s])
        if n <= 0:
            continue
        for h in range(Hq):
            L = Kc[s, h // G, :n] @ q[s, h] / np.sqrt(float(d))
            m = L.max()
            e = np.exp(L - m)
            o[s, h] = (e[:, None] * Vc[s, h // G, :n]).sum(axis=0) / e.sum()
            lse[s, h] = m + np.log(e.sum())
    return o, lse


def compress(Q, K, V, cu_seqlens, a, b, R, B, *, K_bits=None, V_bits=None):
    """score -> select -> compact, as one call.

    ``K_bits``/``V_bits`` (optional) are the raw bit patterns to gather so the
    compacted cache can be compared bit for bit; by default K and V are
    gathered as given.
    """
    s = score(Q, K, cu_seqlens, a, b)
    idx, kept_len = select(s, cu_seqlens, R, B)
    Ko, Vo = compact(K if K_bits is None else K_bits,
                     V if V_bits is None else V_bits,
                     cu_seqlens, idx, kept_len, B)
    return s, idx, kept_len, Ko, Vo
