"""Stored fixtures: the README's parameters and an oracle regression case."""

import json
import os

import numpy as np

import oracle
from brute_decimal import brute_scores
from golden import make_golden

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_readme_parameters_match_the_workload_recipe():
    from prefill_eviction_scoring_b200 import workloads as wl
    with open(os.path.join(GOLDEN, "readme_parameters.json")) as f:
        p = json.load(f)
    acts = tuple((float(x.split(":")[0]), int(x.split(":")[1]))
                 for x in p["actions"]["value"].split(","))
    assert acts == wl.WAITS_ACTIONS
    qs = p["quickstart_init_cache"]
    assert (qs["recent_budget"], qs["select_budget"]) == (16, 128)
    tiny = wl.CONFIGS["tiny"]
    assert (tiny.recent, tiny.budgets[0]) == (16, 128)


def test_oracle_regression_fixture_and_brute_force():
    with open(os.path.join(GOLDEN, "tiny_oracle.json")) as f:
        fx = json.load(f)
    Q, K, cu = make_golden.inputs()
    for case in fx["cases"]:
        s = oracle.score(Q, K, cu, case["a"], case["b"])
        np.testing.assert_allclose(s, case["scores"], rtol=1e-14, atol=0)
        idx, kept = oracle.select(s, cu, case["R"], case["B"])
        assert idx.tolist() == case["idx"] and kept.tolist() == case["kept_len"]
        ref = brute_scores(Q.tolist(), K.tolist(), cu.tolist(),
                           case["a"], case["b"])
        ref = np.array([[float(x) for x in r] for r in ref])
        np.testing.assert_allclose(case["scores"], ref, rtol=1e-12, atol=1e-300)
