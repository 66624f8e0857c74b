"""Write the oracle regression fixture ``tiny_oracle.json``.

Calls only ``oracle/`` (and numpy for the seeded inputs).  Re-run it only
when a change to the oracle's arithmetic is justified by the WAITS README;
the fixture is also checked against the decimal brute force.
"""

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402


def inputs():
    rng = np.random.default_rng(20261202)
    lens = (12, 5)
    T, Hq, Hkv, d = sum(lens), 4, 2, 8
    def bf16ish(x):
        m, e = np.frexp(x)
        return np.ldexp(np.round(m * 256.0) / 256.0, e)
    Q = bf16ish(rng.standard_normal((T, Hq, d)) * 1.5)
    K = bf16ish(rng.standard_normal((T, Hkv, d)) * 1.5)
    cu = np.array([0, 12, 17])
    return Q, K, cu


CASES = [(1.0, 3, 2, 6), (0.0, 1, 2, 8), (1e4, 1, 1, 4)]   # (a, b, R, B)


def main():
    Q, K, cu = inputs()
    out = {"_note": "oracle regression values; inputs from make_golden.inputs()",
           "cases": []}
    for a, b, R, B in CASES:
        s = oracle.score(Q, K, cu, a, b)
        idx, kept = oracle.select(s, cu, R, B)
        out["cases"].append({"a": a, "b": b, "R": R, "B": B,
                             "scores": s.tolist(), "idx": idx.tolist(),
                             "kept_len": kept.tolist()})
    with open(os.path.join(HERE, "tiny_oracle.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
