"""Pins of the oracle's router against what the pages and the mathematics fix.

Sources: "GLM-4.5 Group Router", How it works (s = sigma(x W_g^T) in float32,
s' = s + b for selection only, group score = sum of the two largest s' of each
contiguous group, keep topk_group groups, top-k inside them, weights from raw s
renormalised with eps 1e-20 and scaled by alpha; G = 1 is plain top-k).
"GLM-5.3-Flash Module 02", section 2 (selection uses score + bias, weighting the
raw score; the two must be tested independently).
"""

import itertools
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _rand_logits(N, E, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return rng.normal(0.0, scale, size=(N, E))


def _bias(E, beta, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.rand(E, generator=g) * 2 - 1) * beta


def test_sigmoid_closed_forms_and_weights():
    # r = 0 -> s = 1/2; r = ln 3 -> s = 3/4; r = -ln 3 -> s = 1/4 (exact identities).
    r = np.array([[0.0, math.log(3.0), -math.log(3.0)]])
    b = torch.zeros(3)
    out = oracle.select(r, b, 1, 1, 3, True, 2.0)
    np.testing.assert_allclose(out["s"][0], [0.5, 0.75, 0.25], rtol=0, atol=1e-15)
    # Order: descending s' (b = 0): experts 1, 0, 2.
    assert out["idx"][0].tolist() == [1, 0, 2]
    # Weights alpha * s / (sum s + 1e-20): sum s = 1.5 -> 2 * [0.5, 1/3, 1/6].
    np.testing.assert_allclose(out["w"][0], [1.0, 2.0 / 3.0, 1.0 / 3.0], rtol=1e-15)


def test_g1_reduces_to_full_sort():
    # G = 1 and topk_group = 1: T is ordinary top-k of s' over all experts.
    N, E, k = 200, 160, 8
    r = _rand_logits(N, E, 1, 1.5)
    b = _bias(E, 0.05, 2)
    out = oracle.select(r, b, 1, 1, k, True, 2.5)
    sp = scipy.special.expit(r) + b.double().numpy()[None, :]
    # stable descending sort: ties keep the lower index first
    order = np.argsort(-sp, axis=1, kind="stable")[:, :k]
    np.testing.assert_array_equal(out["idx"], order)
    assert np.all(out["margin_grp"] == np.inf)
    srt = -np.sort(-sp, axis=1)
    np.testing.assert_allclose(out["margin_exp"], srt[:, k - 1] - srt[:, k], rtol=0, atol=1e-15)


def test_weights_from_raw_scores_not_biased_scores():
    # Bias large enough to reorder selection: weights must still be alpha*s/sum(s) over T.
    N, E, k, alpha = 300, 32, 4, 2.5
    r = _rand_logits(N, E, 3, 0.5)
    b = _bias(E, 0.3, 4)
    out = oracle.select(r, b, 1, 1, k, True, alpha)
    s = scipy.special.expit(r)
    sel = np.take_along_axis(s, out["idx"].astype(np.int64), axis=1)
    expect = alpha * sel / (sel.sum(axis=1, keepdims=True) + 1e-20)
    np.testing.assert_allclose(out["w"], expect, rtol=1e-14)
    # The bias really changes the selection on these inputs (else this test proves nothing).
    plain = oracle.select(r, torch.zeros(E), 1, 1, k, True, alpha)
    assert np.any(np.sort(plain["idx"], 1) != np.sort(out["idx"], 1))
    # Ratios w_i / w_j equal s_i / s_j.
    np.testing.assert_allclose(out["w"][:, 0] / out["w"][:, 1], sel[:, 0] / sel[:, 1], rtol=1e-13)


def test_weights_invariant_to_bias_that_keeps_the_set():
    N, E, k = 100, 16, 4
    r = _rand_logits(N, E, 5)
    b = _bias(E, 0.01, 6)
    a = oracle.select(r, b, 1, 1, k, True, 1.0)
    # Push every selected expert further up: the chosen set cannot change.
    for n in range(N):
        b2 = b.clone()
        b2[torch.from_numpy(a["idx"][n].astype(np.int64))] += 0.5
        c = oracle.select(r[n:n + 1], b2, 1, 1, k, True, 1.0)
        assert sorted(c["idx"][0]) == sorted(a["idx"][n])
        wa = dict(zip(a["idx"][n], a["w"][n]))
        wc = dict(zip(c["idx"][0], c["w"][0]))
        for e in wa:
            assert wa[e] == wc[e]


def test_weight_sum_is_alpha_and_unnormalised_branch():
    N, E, k = 64, 64, 8
    r = _rand_logits(N, E, 7)
    b = _bias(E, 0.05, 8)
    out = oracle.select(r, b, 1, 1, k, True, 2.5)
    np.testing.assert_allclose(out["w"].sum(1), 2.5, rtol=0, atol=1e-12)
    raw = oracle.select(r, b, 1, 1, k, False, 2.5)
    s = scipy.special.expit(r)
    np.testing.assert_allclose(raw["w"], 2.5 * np.take_along_axis(s, raw["idx"].astype(np.int64), 1),
                               rtol=1e-15)


def _brute_force(sp, G, tg, k):
    """Enumerate group subsets then expert subsets; return the chosen expert set."""
    E = len(sp)
    m = E // G
    gscore = [sum(sorted(sp[g * m:(g + 1) * m], reverse=True)[:2]) for g in range(G)]
    best_groups = max(itertools.combinations(range(G), tg), key=lambda c: sum(gscore[g] for g in c))
    cands = [e for g in best_groups for e in range(g * m, (g + 1) * m)]
    best = max(itertools.combinations(cands, k), key=lambda c: sum(sp[e] for e in c))
    return set(best)


def test_group_router_matches_brute_force_enumeration():
    # Tiny group-routed shape (E=16, G=4 groups of 4, keep 2, k=4): 6 group subsets x 70 sets.
    N, E, G, tg, k = 400, 16, 4, 2, 4
    r = _rand_logits(N, E, 9, 0.4)
    b = _bias(E, 0.1, 10)
    out = oracle.select(r, b, G, tg, k, True, 2.5)
    sp = scipy.special.expit(r) + b.double().numpy()[None, :]
    checked = 0
    for n in range(N):
        if out["margin_exp"][n] < 1e-9 or out["margin_grp"][n] < 1e-9:
            continue
        assert set(out["idx"][n].tolist()) == _brute_force(sp[n].tolist(), G, tg, k)
        checked += 1
    assert checked > N * 0.95


def test_group_score_is_top2_sum_not_top1_or_full_sum():
    # Group 0: one big entry (top-1 winner); group 1: two good entries (top-2 winner);
    # group 2: many medium entries (full-sum winner).  keep 1 group, k = 2.
    sp = np.array([0.95, 0.05, 0.05, 0.05,
                   0.70, 0.70, 0.00, 0.00,
                   0.60, 0.60, 0.60, 0.60])
    r = scipy.special.logit(np.clip(sp, 1e-9, 1 - 1e-9))[None, :]
    out = oracle.select(r, torch.zeros(12), 3, 1, 2, True, 1.0)
    assert sorted(out["idx"][0].tolist()) == [4, 5]


def test_ties_go_to_lower_index():
    r = np.zeros((1, 8))
    out = oracle.select(r, torch.zeros(8), 1, 1, 3, True, 1.0)
    assert out["idx"][0].tolist() == [0, 1, 2]
    out = oracle.select(r, torch.zeros(8), 4, 2, 3, True, 1.0)
    assert out["idx"][0].tolist() == [0, 1, 2]


def test_discarded_groups_are_minus_infinity_and_zero_fill_flagged():
    # Kept group members all have negative s'; a zero fill would pull in discarded experts.
    E, G = 8, 2
    r = np.zeros((1, E))
    b = torch.tensor([-0.6, -0.6, -0.6, -0.6, -0.9, -0.9, -0.9, -0.9])
    out = oracle.select(r, b, G, 1, 2, True, 1.0)
    assert set(out["idx"][0].tolist()) <= {0, 1, 2, 3}
    assert out["zero_fill_differs"][0] == 1
    # Ordinary case: positive scores, the two readings agree.
    out = oracle.select(_rand_logits(50, 16, 11, 0.3), _bias(16, 0.1, 12), 4, 2, 4, True, 2.5)
    assert out["zero_fill_differs"].sum() == 0


@pytest.mark.parametrize("E,G,tg,k", [(16, 3, 1, 2), (16, 16, 2, 2), (16, 4, 1, 8), (8, 1, 1, 9)])
def test_invalid_configurations_rejected(E, G, tg, k):
    with pytest.raises(ValueError):
        oracle.select(np.zeros((1, E)), torch.zeros(E), G, tg, k, True, 1.0)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_logits_exact_on_integer_inputs(dtype):
    # Small integers are exact in bf16/fp32, so x W_g^T equals the integer product.
    rng = np.random.default_rng(13)
    x = rng.integers(-8, 9, size=(7, 40))
    W = rng.integers(-8, 9, size=(5, 40))
    r = oracle.router_logits(torch.tensor(x, dtype=dtype), torch.tensor(W, dtype=dtype))
    np.testing.assert_array_equal(r, (x @ W.T).astype(np.float64))
    # Basis rows pick coordinates: r[n, e] = x[n, e].
    xb = torch.randn(3, 6).to(dtype)
    r = oracle.router_logits(xb, torch.eye(6, dtype=dtype)[:4])
    np.testing.assert_array_equal(r, xb.double().numpy()[:, :4])


def test_mixed_precision_inputs_widen_exactly():
    # bf16 tokens against an fp32 router matrix (the GLM-4.5 shapes).
    x = torch.tensor([[1.5, -2.0, 0.25]], dtype=torch.bfloat16)
    W = torch.tensor([[0.1, 0.2, 0.3]], dtype=torch.float32)
    r = oracle.router_logits(x, W)
    w = W.double().numpy()
    assert r[0, 0] == 1.5 * w[0, 0] - 2.0 * w[0, 1] + 0.25 * w[0, 2]
