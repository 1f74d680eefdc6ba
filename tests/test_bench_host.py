"""Host logic of the benchmark's JSON line (CPU only, no kernels run).

The roofline arithmetic (achieved = algorithmic work of one launch / its time,
against the measured or fallback peak and against the nominal figures the
layer's targets use), the workload list, the configuration dict both arms print,
and the parity summary that compares a step's rows with the oracle.
"""

import numpy as np
import pytest
import torch

import bench
import oracle
from workloads import CONFIGS, PERF_WORKLOADS, make_inputs


def test_headline_is_the_largest_configuration_and_others_follow():
    sizes = {n: CONFIGS[n].N * CONFIGS[n].k * CONFIGS[n].D for n in PERF_WORKLOADS}
    from workloads import DEFAULT_WORKLOAD
    assert DEFAULT_WORKLOAD == max(sizes, key=sizes.get) == "skew_grouped"
    class A:  # noqa: E306
        workload, workloads = "skew_grouped", "perf"
    assert bench.extra_workloads(A) == [n for n in PERF_WORKLOADS if n != "skew_grouped"]
    A.workloads = "none"
    assert bench.extra_workloads(A) == []
    A.workloads = "air_decode,nonexistent"
    assert bench.extra_workloads(A) == ["air_decode"]


def test_both_arms_describe_the_workload_with_one_dict():
    cfg = CONFIGS["skew_grouped"]
    d1 = bench.config_dict(cfg, None, 1)
    d2 = bench.config_dict(cfg, {}, 1)
    assert d1 == d2
    assert d1["workload"] == "skew_grouped" and d1["N"] == 16384 and d1["n_group"] == 8
    assert bench.config_dict(cfg, None, 4)["parallelism"] == "replicas"


def test_roofline_arithmetic():
    cfg = CONFIGS["skew_grouped"]
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1200.0}
    flops, byts = bench.kernel_work(cfg, "gate_up_swiglu", 200)
    # 2 * (N k 2d + N 2 d_sh) D FLOP; weights of the hit experts and the shared one, x once
    assert flops == 2.0 * (16384 * 8 * 4096 + 16384 * 4096) * 6144
    assert byts == (200 * 4096 + 4096) * 6144 * 2 + 16384 * 6144 * 2
    r = bench.roofline_of(cfg, "gate_up_swiglu", 200, 5.0, peaks, "measured")
    assert r["bound"] == "tensor"
    assert r["achieved"] == pytest.approx(flops / 5e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1200.0)
    assert r["vs_nominal"]["frac"] == pytest.approx(r["achieved"] / 2250.0)
    assert r["vs_nominal"]["target"] == 0.60
    dec = CONFIGS["air_decode"]
    r = bench.roofline_of(dec, "gate_up_swiglu", 100, 0.4, peaks, "fallback")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["vs_nominal"]["frac"] == pytest.approx(r["achieved"] / 8000.0)
    assert r["vs_nominal"]["target"] == 0.70
    assert r["peak_source"] == "fallback copy"


def test_parity_summary_counts_mismatches_and_errors():
    cfg = CONFIGS["glm5_prefill"].with_(N=24, D=256, E=16, k=4, d_moe=128, d_sh=128)
    inp = make_inputs(cfg, seed=3)
    r = oracle.router(inp.x, inp.W_g, inp.b, 1, 1, cfg.k, True, cfg.alpha)
    y = oracle.forward(inp.x, inp.gate_up, inp.down, inp.sh_gate, inp.sh_up, inp.sh_down,
                       r["idx"], r["w"])
    same = bench.parity_summary(cfg, r, y, r["idx"].copy(), r["w"].copy(), y.astype(np.float32), inp.b)
    assert same["id_mismatch_tokens"] == 0 and same["unexplained_mismatches"] == 0
    assert same["max_rel"] < 1e-6 and same["max_row_l2_rel"] < 1e-6
    # a swapped expert id on one token, far from any tie, is an unexplained mismatch;
    # a scaled row shows up in both error measures
    gi = r["idx"].copy()
    gi[3, 0] = (gi[3, 0] + 1) % cfg.E if (gi[3, 0] + 1) % cfg.E not in gi[3] else (gi[3, 0] + 5) % cfg.E
    gy = y.astype(np.float32).copy()
    gy[5] *= 1.1
    bad = bench.parity_summary(cfg, r, y, gi, r["w"], gy, inp.b)
    assert bad["id_mismatch_tokens"] == 1
    assert bad["unexplained_mismatches"] == 1 or bad["near_tie_tokens"] > 0
    assert bad["max_row_l2_rel"] == pytest.approx(0.1, rel=1e-3)
    assert bad["max_rel"] > 0.0


def test_compact_experts_keeps_the_oracle_result():
    cfg = CONFIGS["glm5_prefill"].with_(N=12, D=128, E=10, k=3, d_moe=64, d_sh=64)
    inp = make_inputs(cfg, seed=4)
    r = oracle.router(inp.x, inp.W_g, inp.b, 1, 1, cfg.k, True, cfg.alpha)
    idx = r["idx"].copy()
    idx[0, 1] = cfg.E  # the sentinel stays the sentinel
    y_full = oracle.forward(inp.x, inp.gate_up, inp.down, inp.sh_gate, inp.sh_up, inp.sh_down,
                            idx, r["w"])
    weights, remap = bench.compact_experts(inp, idx)
    assert weights[0].shape[0] == len(set(idx.ravel()) - {cfg.E})
    y_c = oracle.forward(inp.x, *weights, remap[idx], r["w"])
    assert np.array_equal(y_c, y_full)
