"""Brute-force WAITS score in 40-digit decimal arithmetic (tiny inputs only).

An independent restatement used to pin the fp64 oracle: dense N x N attention
per query head, every exp and square root in ``decimal``, no numpy, no
blocking, no skipped rows.  Source: WAITS README (stig.sh/Dirac-Notation/A2SF),
opening summary (forgetting curve and accumulative attention score), read as
causal softmax(QK^T/sqrt(d)) summed over the query heads of a KV head.
"""

from decimal import Decimal, localcontext


def brute_scores(Q, K, cu_seqlens, a, b, prec=40):
    """Q: nested lists / array [T][Hq][d], K: [T][Hkv][d]; returns [Hkv][T]
    as Decimal."""
    T = len(Q)
    Hq = len(Q[0]) if T else 0
    Hkv = len(K[0]) if T else 0
    d = len(Q[0][0]) if T else 0
    G = Hq // Hkv if Hkv else 1
    with localcontext() as ctx:
        ctx.prec = prec
        s = [[Decimal(0) for _ in range(T)] for _ in range(Hkv)]
        if T == 0:
            return s
        root_d = Decimal(d).sqrt()
        A = Decimal(repr(float(a)))
        for i in range(len(cu_seqlens) - 1):
            lo, hi = int(cu_seqlens[i]), int(cu_seqlens[i + 1])
            N = hi - lo
            centre = Decimal(N) - Decimal(int(b)) - Decimal("0.5")
            for h in range(Hq):
                g = h // G
                for q in range(N):
                    w = Decimal(1) / (Decimal(1) + (-A * (Decimal(q) - centre)).exp())
                    logits = []
                    for k in range(q + 1):
                        dot = sum(Decimal(float(Q[lo + q][h][j])) *
                                  Decimal(float(K[lo + k][g][j]))
                                  for j in range(d))
                        logits.append(dot / root_d)
                    m = max(logits)
                    ex = [(x - m).exp() for x in logits]
                    z = sum(ex)
                    for k in range(q + 1):
                        s[g][lo + k] += w * ex[k] / z
        return s


def brute_lse(Q, K, cu_seqlens, prec=40):
    """Natural-log row LSE [Hq][T] of the causal attention, in decimal."""
    T = len(Q)
    Hq = len(Q[0]) if T else 0
    Hkv = len(K[0]) if T else 0
    d = len(Q[0][0]) if T else 0
    G = Hq // Hkv if Hkv else 1
    with localcontext() as ctx:
        ctx.prec = prec
        out = [[Decimal(0) for _ in range(T)] for _ in range(Hq)]
        root_d = Decimal(d).sqrt() if d else Decimal(1)
        for i in range(len(cu_seqlens) - 1):
            lo, hi = int(cu_seqlens[i]), int(cu_seqlens[i + 1])
            for h in range(Hq):
                g = h // G
                for q in range(hi - lo):
                    logits = [sum(Decimal(float(Q[lo + q][h][j])) * Decimal(float(K[lo + k][g][j]))
                                  for j in range(d)) / root_d for k in range(q + 1)]
                    m = max(logits)
                    out[h][lo + q] = m + sum((x - m).exp() for x in logits).ln()
        return out
