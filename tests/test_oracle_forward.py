"""Pins of the oracle's MoE forward against what the pages and the mathematics fix.

Sources: "GLM-4.5 MoE Forward", How it works (E_i(x) = W_down (SiLU(W_gate x) (.)
W_up x), gate rows first in gate_up_proj[i] (2 d_moe, D); y_n = sum w E_i + E_sh with
the shared expert at scale 1, alpha applied once, exactly k routed experts per
token).  "GLM-5 Mixture of experts", experts' forward excerpt (index E is a
skipped sentinel; down_proj[i] is (D, d_moe)) and Parameters table.  "GLM-5
Shared output" (shared MLP on the same input).
"""

import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from workloads import CONFIGS, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _small(E=6, D=24, d=16, d_sh=8, N=10, seed=0, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    t = lambda *s: (torch.randn(*s, generator=g) * 0.3).to(dtype)
    return dict(x=t(N, D), gate_up=t(E, 2 * d, D), down=t(E, D, d), sh_gate=t(d_sh, D),
                sh_up=t(d_sh, D), sh_down=t(D, d_sh))


def _routing(N, E, k, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(N)]).astype(np.int32)
    w = rng.uniform(0.1, 1.0, size=(N, k))
    return idx, w


def _lib_swiglu(x, wg, wu, wd):
    """SwiGLU MLP through torch library ops in fp64: down(silu(gate x) * up x)."""
    x, wg, wu, wd = (t.double() for t in (x, wg, wu, wd))
    return F.linear(F.silu(F.linear(x, wg)) * F.linear(x, wu), wd)


def test_selection_matrix_experts_closed_form():
    # D != d and asymmetric gate/up/down so a transposed operand, swapped gate/up halves
    # or a dropped term gives a different answer.  E_i(x)[c] = sum_r P[c,r] silu(x[r]) 2 x[r+1].
    D, d, E, N = 6, 4, 2, 5
    gate_up = torch.zeros(E, 2 * d, D)
    down = torch.zeros(E, D, d)
    for e in range(E):
        for r in range(d):
            gate_up[e, r, r] = 1.0  # gate row r picks x[r]
            gate_up[e, d + r, r + 1] = 2.0 + e  # up row r picks (2+e) x[r+1]
            down[e, (r + 2 + e) % D, r] = 1.0 + 0.5 * r
    sh_gate = torch.zeros(1, D)
    sh_up = torch.zeros(1, D)
    sh_down = torch.zeros(D, 1)
    x = torch.linspace(-2.0, 2.5, N * D).reshape(N, D)
    idx = np.array([[0, 1]] * N, dtype=np.int32)
    w = np.array([[0.25, 0.75]] * N)
    y = oracle.forward(x, gate_up, down, sh_gate, sh_up, sh_down, idx, w)
    xd = x.double()
    expect = torch.zeros(N, D, dtype=torch.float64)
    for e, we in ((0, 0.25), (1, 0.75)):
        for r in range(d):
            expect[:, (r + 2 + e) % D] += we * (1.0 + 0.5 * r) * F.silu(xd[:, r]) * (2.0 + e) * xd[:, r + 1]
    np.testing.assert_allclose(y, expect.numpy(), rtol=1e-14, atol=1e-15)


def test_clamped_swiglu_boundaries_closed_form():
    # "GLM-5.3-Flash Module 02", section 3: a = min(W_g x, 10) (above only),
    # u = clip(W_u x, -10, 10).  Gate rows pick x[r], up rows pick 1.5 x[r+1]; the
    # values straddle both limits on both projections, and a gate value of -30 must
    # stay -30 (a symmetric clamp would give -10, a visibly different SiLU).
    D, d, E = 6, 4, 1
    gate_up = torch.zeros(E, 2 * d, D)
    down = torch.zeros(E, D, d)
    for r in range(d):
        gate_up[0, r, r] = 1.0
        gate_up[0, d + r, r + 1] = 1.5
        down[0, r, r] = 1.0
    x = torch.tensor([[15.0, -30.0, 12.0, -20.0, 5.0, 8.0],
                      [9.5, 6.0, -11.0, 7.0, 10.5, -3.0],
                      [-30.0, 2.0, 10.0, -7.0, 0.5, 4.0]])
    sh = dict(sh_gate=torch.zeros(1, D), sh_up=torch.zeros(1, D), sh_down=torch.zeros(D, 1))
    idx = np.zeros((3, 1), dtype=np.int32)
    w = np.ones((3, 1))
    y = oracle.forward(x, gate_up, down, idx=idx, w=w, gate_max=10.0, up_max=10.0, **sh)
    xd = x.double()
    a = torch.clamp(xd[:, :d], max=10.0)
    u = torch.clamp(1.5 * xd[:, 1:d + 1], min=-10.0, max=10.0)
    expect = torch.zeros(3, D, dtype=torch.float64)
    expect[:, :d] = F.silu(a) * u
    np.testing.assert_allclose(y, expect.numpy(), rtol=1e-14, atol=1e-300)
    # no limits: the plain SwiGLU of the same selection matrices
    y0 = oracle.forward(x, gate_up, down, idx=idx, w=w, **sh)
    plain = torch.zeros(3, D, dtype=torch.float64)
    plain[:, :d] = F.silu(xd[:, :d]) * 1.5 * xd[:, 1:d + 1]
    np.testing.assert_allclose(y0, plain.numpy(), rtol=1e-14)
    assert not np.allclose(y, y0)


def test_clamp_applies_to_the_shared_expert_too():
    t = _small(seed=21)
    t = {k_: (v * 40.0 if k_ != "x" else v) for k_, v in t.items()}  # large activations
    t["down"] = torch.zeros_like(t["down"])
    idx, w = _routing(10, 6, 2, 22)
    y = oracle.forward(**t, idx=idx, w=w, gate_max=10.0, up_max=10.0)
    x, g, u_, dn = (v.double() for v in (t["x"], t["sh_gate"], t["sh_up"], t["sh_down"]))
    a = torch.clamp(F.linear(x, g), max=10.0)
    u = torch.clamp(F.linear(x, u_), -10.0, 10.0)
    np.testing.assert_allclose(y, F.linear(F.silu(a) * u, dn).numpy(), rtol=1e-12, atol=1e-12)


def test_shared_expert_alone_is_the_swiglu_mlp():
    t = _small()
    t["down"] = torch.zeros_like(t["down"])  # routed experts contribute nothing
    idx, w = _routing(10, 6, 3, 1)
    y = oracle.forward(**t, idx=idx, w=w)
    expect = _lib_swiglu(t["x"], t["sh_gate"], t["sh_up"], t["sh_down"])
    np.testing.assert_allclose(y, expect.numpy(), rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("n_shared", [2, 3])
def test_n_shared_experts_are_one_wider_mlp(n_shared):
    # "GLM-4.5 MoE Forward", How it works: the shared expert is one SwiGLU of
    # intermediate width d_moe * n_shared.  Its features are independent until
    # the down projection sums them, so the wide MLP must equal the sum of the
    # n_shared width-d_moe MLPs cut from its gate/up rows and down columns.
    d = 8
    t = _small(d=d, d_sh=d * n_shared, seed=31 + n_shared)
    idx, w = _routing(10, 6, 2, 32)
    y = oracle.forward(**t, idx=idx, w=w)
    zero = {k_: torch.zeros_like(v) for k_, v in t.items() if k_.startswith("sh_")}
    routed = oracle.forward(t["x"], t["gate_up"], t["down"], idx=idx, w=w, **zero)
    parts = sum(_lib_swiglu(t["x"], t["sh_gate"][j * d:(j + 1) * d], t["sh_up"][j * d:(j + 1) * d],
                            t["sh_down"][:, j * d:(j + 1) * d]).numpy() for j in range(n_shared))
    np.testing.assert_allclose(y, routed + parts, rtol=1e-12, atol=1e-13)


def test_routed_expert_matches_library_swiglu():
    t = _small(E=3, N=4)
    sh = dict(sh_gate=torch.zeros_like(t["sh_gate"]), sh_up=t["sh_up"], sh_down=t["sh_down"])
    idx = np.array([[2], [0], [1], [2]], dtype=np.int32)
    w = np.array([[1.0], [0.5], [2.0], [-1.0]])
    y = oracle.forward(t["x"], t["gate_up"], t["down"], idx=idx, w=w, **sh)
    d = t["gate_up"].shape[1] // 2
    for n in range(4):
        e = int(idx[n, 0])
        ref = _lib_swiglu(t["x"][n:n + 1], t["gate_up"][e, :d], t["gate_up"][e, d:], t["down"][e])
        np.testing.assert_allclose(y[n], w[n, 0] * ref[0].numpy(), rtol=1e-12, atol=1e-14)


def test_shared_expert_unscaled_and_alpha_linear():
    cfg = CONFIGS["tiny_fp32"]
    inp = make_inputs(cfg, seed=3)
    args = (inp.x, inp.gate_up, inp.down, inp.sh_gate, inp.sh_up, inp.sh_down)
    rt = lambda a: oracle.router(inp.x, inp.W_g, inp.b, cfg.n_group, cfg.topk_group, cfg.k, True, a)
    r1, r25 = rt(1.0), rt(2.5)
    np.testing.assert_array_equal(r1["idx"], r25["idx"])
    y1 = oracle.forward(*args, r1["idx"], r1["w"])
    y25 = oracle.forward(*args, r25["idx"], r25["w"])
    esh = _lib_swiglu(inp.x, inp.sh_gate, inp.sh_up, inp.sh_down).numpy()
    np.testing.assert_allclose(y25 - esh, 2.5 * (y1 - esh), rtol=1e-9, atol=1e-13)


def test_single_expert_special_case():
    # E = 1, k = 1, G = 1, normalised: w = alpha s / (s + 1e-20), y = w E_0(x) + E_sh(x).
    t = _small(E=1, N=3)
    W_g = torch.randn(1, 24)
    r = oracle.router(t["x"], W_g, torch.zeros(1), 1, 1, 1, True, 2.5)
    s = r["s"][:, 0]
    np.testing.assert_allclose(r["w"][:, 0], 2.5 * s / (s + 1e-20), rtol=1e-15)
    y = oracle.forward(**t, idx=r["idx"], w=r["w"])
    d = t["gate_up"].shape[1] // 2
    e0 = _lib_swiglu(t["x"], t["gate_up"][0, :d], t["gate_up"][0, d:], t["down"][0]).numpy()
    esh = _lib_swiglu(t["x"], t["sh_gate"], t["sh_up"], t["sh_down"]).numpy()
    np.testing.assert_allclose(y, r["w"][:, :1] * e0 + esh, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_token_major_equals_expert_major(dtype):
    t = _small(E=8, D=40, d=24, d_sh=16, N=33, seed=5, dtype=dtype)
    idx, w = _routing(33, 8, 3, 6)
    y1 = oracle.forward(**t, idx=idx, w=w)
    y2 = oracle.forward_expert_major(**t, idx=idx, w=w)
    np.testing.assert_allclose(y1, y2, rtol=1e-12, atol=1e-12 * np.abs(y2).max())


def test_token_permutation_permutes_output():
    t = _small(N=12, seed=7)
    idx, w = _routing(12, 6, 2, 8)
    y = oracle.forward(**t, idx=idx, w=w)
    p = np.random.default_rng(9).permutation(12)
    t2 = dict(t)
    t2["x"] = t["x"][torch.from_numpy(p)]
    y2 = oracle.forward(**t2, idx=idx[p], w=w[p])
    np.testing.assert_array_equal(y2, y[p])


def test_expert_relabelling_leaves_output_unchanged():
    cfg = CONFIGS["tiny_fp32"].with_(n_group=1, topk_group=1)
    inp = make_inputs(cfg, seed=11)
    perm = torch.from_numpy(np.random.default_rng(12).permutation(cfg.E))
    run = lambda W_g, b, gu, dn: oracle.forward(
        inp.x, gu, dn, inp.sh_gate, inp.sh_up, inp.sh_down,
        *(lambda r: (r["idx"], r["w"]))(oracle.router(inp.x, W_g, b, 1, 1, cfg.k, True, cfg.alpha)))
    y = run(inp.W_g, inp.b, inp.gate_up, inp.down)
    y2 = run(inp.W_g[perm], inp.b[perm], inp.gate_up[perm], inp.down[perm])
    np.testing.assert_array_equal(y, y2)


def test_sentinel_expert_is_skipped():
    t = _small(E=5, N=6, seed=13)
    idx, w = _routing(6, 5, 3, 14)
    idx_s = idx.copy()
    idx_s[::2, 1] = 5  # the sentinel id E
    w0 = w.copy()
    w0[::2, 1] = 0.0
    np.testing.assert_allclose(oracle.forward(**t, idx=idx_s, w=w),
                               oracle.forward(**t, idx=idx, w=w0), rtol=1e-14, atol=1e-16)
    with pytest.raises(ValueError):
        bad = idx.copy()
        bad[0, 0] = 6
        oracle.forward(**t, idx=bad, w=w)


def test_token_subset_matches_full_evaluation():
    t = _small(N=9, seed=15)
    idx, w = _routing(9, 6, 2, 16)
    y = oracle.forward(**t, idx=idx, w=w)
    sub = np.array([7, 0, 3], dtype=np.int32)
    np.testing.assert_array_equal(oracle.forward(**t, idx=idx, w=w, tokens=sub), y[sub])


def test_parameter_counts_match_pages():
    gold = json.load(open(os.path.join(GOLDEN, "param_counts.json")))
    g5 = gold["glm5"]
    pc = oracle.param_counts(g5["D"], g5["E"], g5["d_moe"], g5["n_shared"])
    for key in ("expert", "routed", "shared", "router", "block"):
        assert pc[key] == g5[key], key
    assert pc["block"] * g5["blocks"] == g5["all_blocks"]
    assert g5["E"] * g5["blocks"] == g5["bias_values"]
    used = g5["k"] * pc["expert"] + pc["shared"] + pc["router"]
    assert used == g5["used_per_token"]
    assert round(pc["block"] * 2 / 2 ** 30, 1) == g5["held_gib_bf16"]
    assert round(used * 2 / 2 ** 20) == g5["used_mib_bf16"]
    m2 = gold["module02_expert"]
    assert oracle.param_counts(m2["D"], 1, m2["d_moe"])["expert"] == m2["expert"]


def test_configuration_shapes_match_pages():
    c = CONFIGS["glm5_prefill"]
    assert oracle.param_counts(c.D, c.E, c.d_moe)["block"] == 9702998272
    assert oracle.param_counts(c.D, c.E, c.d_moe)["expert"] == 37748736
