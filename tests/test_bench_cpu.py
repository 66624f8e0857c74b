"""The bench's algorithmic work counts (the roofline numerators), against
brute force over the causal mask and the fp32 active-row predicate."""

import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _brute_logits(N, a, b):
    q = np.arange(N, dtype=np.float32)
    c = np.float32(N) - np.float32(b) - np.float32(0.5)
    with np.errstate(over="ignore"):
        w = np.float32(1.0) / (np.float32(1.0) + np.exp(np.float32(-a) * (q - c)))
    active = w != 0
    causal = np.tril(np.ones((N, N), dtype=bool))          # key k <= query q
    return int(causal[active].sum())


@pytest.mark.parametrize("N,a,b", [(300, 1.0, 16), (257, 0.0, 16), (400, 10.0, 1),
                                   (128, 1e4, 1), (1000, 0.01, 128), (90, 1.0, 200)])
def test_scorer_logits_brute_force(N, a, b):
    Hq, d = 4, 64
    flops, logits = bench.scorer_flops([N], Hq, d, a, b)
    want = _brute_logits(N, a, b)
    assert logits == Hq * want
    assert flops == 2 * 2 * d * Hq * want


def test_headline_active_logits():
    # 105 active rows per head at N = 32768, a = 1, b = 16: keys 32664..32768 per row
    _, logits = bench.scorer_flops([32768], 32, 128, 1.0, 16)
    assert bench.first_active_row(32768, 1.0, 16) == 32768 - 105
    assert logits == 32 * 105 * (32664 + 32768) // 2


def test_select_compact_bytes():
    sel, comp = bench.select_compact_bytes([100, 5000], 2, 128, 1024)
    assert sel == 2 * 5100 * 4 + 2 * 2 * 1024 * 4
    assert comp == 2 * 2 * (100 + 1024) * 2 * 128 * 2 + 2 * 2 * 1024 * 4


def _peaks():
    return {"bf16_tflops": 1679.3, "bf16_tflops_sustained": 1437.5, "hbm_gbs": 6453.4,
            "sm_max_mhz": 1965.0}


def test_headline_roofline_is_the_tensor_term():
    # 8B layer: 2 passes x 2d FLOPs per active logit at the burst bf16 peak
    # binds (33.5 us); one pass of exponentials at 16/clk/SM x 148 x 1.965 GHz
    # is 23.6 us; K, the active Q rows and the scores at HBM peak ~10.9 us
    lens, Hq, Hkv, d = [32768], 32, 8, 128
    flops, logits = bench.scorer_flops(lens, Hq, d, 1.0, 16)
    t_meas_ms = 0.1148
    head, other = bench.rooflines(lens, Hq, Hkv, d, 1.0, 16, 2048, t_meas_ms, 0.0224,
                                  0.130, _peaks(), 148)
    t_tensor = flops / 1679.3e12
    t_mufu = logits / (16 * 148 * 1.965e9)
    assert head["bound"] == "tensor" and head["unit"] == "TFLOP/s"
    assert head["roofline_us"] == pytest.approx(t_tensor * 1e6, rel=1e-3)
    assert head["terms_us"]["mufu"] == pytest.approx(t_mufu * 1e6, rel=1e-3)
    assert head["frac"] == pytest.approx(t_tensor / (t_meas_ms / 1e3), rel=1e-3)
    assert head["frac"] == pytest.approx(0.29, abs=0.01)
    kb = 32768 * 8 * 128 * 2 + 105 * 32 * 128 * 2 + 8 * 32768 * 4
    assert head["algorithmic_bytes"] == kb
    assert head["terms_us"]["hbm"] == pytest.approx(kb / 6453.4e9 * 1e6, rel=1e-3)
    layer = other[0]
    sel, comp = bench.select_compact_bytes(lens, Hkv, d, 2048)
    assert layer["roofline_us"] == pytest.approx((t_tensor + (sel + comp) / 6453.4e9) * 1e6,
                                                 rel=1e-3)
    assert layer["frac"] == pytest.approx(layer["roofline_us"] / 130.0, rel=1e-3)


def test_roofline_binds_on_mufu_for_head_dim_64():
    # d = 64, every row active (a = 0): 256 FLOPs per logit over two passes is
    # less time at the tensor peak than one exponential per logit at the MUFU peak
    head, _ = bench.rooflines([4096], 32, 8, 64, 0.0, 1, 128, 0.2, 0.01, 0.25, _peaks(), 148)
    assert head["bound"] == "alu" and head["unit"] == "Gexp/s"
    logits = 32 * 4096 * 4097 // 2
    assert head["achieved"] == pytest.approx(logits / 0.2e-3 / 1e9, rel=1e-3)
    assert head["frac"] == pytest.approx(head["roofline_us"] / 200.0, rel=1e-3)


def test_oracle_prefix_keeps_the_sample_bounded():
    # the long workload's fp64-visited logits per KV head far exceed the
    # budget, so the CPU baseline runs on a prefix that fits it
    n = bench.oracle_active_logits(131072, 0.01, 128) * 4
    assert n > 2.5e9
    p = bench.oracle_prefix([131072], 0.01, 128, 4)
    assert p is not None and bench.oracle_active_logits(p, 0.01, 128) * 4 <= 2.5e9
    assert bench.oracle_active_logits(p + 1, 0.01, 128) * 4 > 2.5e9
    assert bench.oracle_prefix([512], 1.0, 16, 4) is None


def test_cases_cover_every_configuration():
    names = {(c.name, c.a, c.b, c.B) for cfg in bench.ALL_CONFIGS
             for c in bench.cases_for(cfg, None, None)}
    assert ("llama1b", 0.01, 128, 128) in names and ("stress", 0.0, 16, 2048) in names
    assert len([c for c in names if c[0] == "llama1b"]) == 5
    assert ("ragged", 10.0, 16, 1024) in names and ("long", 0.01, 128, 2048) in names
    sweep = bench.selected_cases(bench.parse(["--config", "all"]))
    assert {c.B for c in sweep if c.name == "llama8b"} == {128, 512, 2048}
    assert [c.B for c in bench.selected_cases(bench.parse([]))] == [2048]


def test_scorer_hash_ignores_comments_only():
    """The profiled-traffic key changes with the scorer's code, not with its
    comments or layout."""
    import bench
    a = "int f(int x) { // one\n  return x + 1; /* two\n lines */ }\n"
    b = "int f(int x)\n{\n  return x + 1;\n}"
    c = "int f(int x) { return x + 2; }"
    assert bench.code_only(a) == bench.code_only(b)
    assert bench.code_only(a) != bench.code_only(c)
    assert bench.profiled_traffic(bench.Case("llama8b", "llama8b", 1.0, 16, 16, 2048, 32)) \
        == bench.PROFILED_SCORER["dram_bytes"]
