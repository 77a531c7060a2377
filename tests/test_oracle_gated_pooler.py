"""Pins of the oracle's Eq.5 gated key pooler ("Pooler Distillation"), forward only.

Each test checks a property that the pages' formula and the stated readings fix,
against something other than the oracle's own formula: closed forms (the mean,
the selected child), library routines (numpy's mean and std, torch's SiLU),
symmetries (translation, scale, permutation) and reductions to already-pinned
paths (Eq.1 values, dense attention when k exceeds every list).
"""
import numpy as np
import pytest
import torch

from long_context_recsa_b200 import inputs as I
from oracle import recsa_oracle as O


def params(d, **over):
    P = {k: (v.numpy().copy() if hasattr(v, "numpy") else v)
         for k, v in I.gated_pooler_params(d).items()}
    P.update(over)
    return P


def children(n, m, d, seed=3):
    return np.random.default_rng(seed).standard_normal((n, m, d))


def test_mlp_off_gate_one_uniform_softmax_is_the_mean():
    d, m = 16, 7
    X = children(5, m, d)
    P = params(d, g=1.0, w=np.zeros(d), W2=np.zeros((d, d)))
    np.testing.assert_allclose(O.gated_pool_keys(X, P), X.mean(axis=1), rtol=0, atol=1e-12)


def test_gate_zero_mlp_off_is_the_mean_for_any_w():
    d, m = 16, 16
    X = children(4, m, d, seed=5)
    P = params(d, g=0.0, W2=np.zeros((d, d)), tau=7.0)
    np.testing.assert_allclose(O.gated_pool_keys(X, P), X.mean(axis=1), rtol=0, atol=1e-12)


def test_sharp_softmax_picks_the_child_with_the_largest_projection():
    d, m = 16, 9
    X = children(6, m, d, seed=8)
    w = np.random.default_rng(1).standard_normal(d)
    P = params(d, g=1.0, W2=np.zeros((d, d)), w=w, tau=1e5)
    best = X[np.arange(6), np.argmax(X @ w, axis=1)]
    np.testing.assert_allclose(O.gated_pool_keys(X, P), best, rtol=0, atol=1e-9)
    # the opposite sign of tau picks the smallest projection instead
    P["tau"] = -1e5
    worst = X[np.arange(6), np.argmin(X @ w, axis=1)]
    np.testing.assert_allclose(O.gated_pool_keys(X, P), worst, rtol=0, atol=1e-9)


def test_translation_equivariance_without_the_mean_branch():
    d, m = 16, 16
    X = children(3, m, d, seed=9)
    v = np.random.default_rng(2).standard_normal(d) * 3
    P = params(d)
    P["W1"] = P["W1"].copy()
    P["W1"][:, :d] = 0.0          # the MLP no longer sees mu / rho
    K0 = O.gated_pool_keys(X, P)
    np.testing.assert_allclose(O.gated_pool_keys(X + v, P), K0 + v, rtol=0, atol=1e-10)
    # with the mean branch on, a translation also moves the MLP's output
    Q = params(d)
    assert not np.allclose(O.gated_pool_keys(X + v, Q), O.gated_pool_keys(X, Q) + v, atol=1e-6)


def test_scale_equivariance_without_the_mean_branch():
    """sigma is a spread (degree 1): K(sX) = s K(X) up to the eps inside the root."""
    d, m = 16, 16
    X = children(3, m, d, seed=10)
    P = params(d)
    P["W1"] = P["W1"].copy()
    P["W1"][:, :d] = 0.0
    s = 3.0
    np.testing.assert_allclose(O.gated_pool_keys(s * X, P), s * O.gated_pool_keys(X, P),
                               rtol=1e-5, atol=1e-7)


def test_permutation_of_children_leaves_the_key_unchanged():
    d, m = 16, 11
    X = children(2, m, d, seed=12)
    perm = np.random.default_rng(4).permutation(m)
    P = params(d)
    np.testing.assert_allclose(O.gated_pool_keys(X[:, perm], P), O.gated_pool_keys(X, P),
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("half", [0, 1])
def test_mlp_wiring_against_torch_silu(half):
    """W1 = identity on [mu/rho ; (p-mu)/sigma], b1 = 0, W2 selects one half.  With
    uniform attention (w = 0) p = mu, so the key is mu + sigma SiLU(mu/rho) for the
    first half and mu + sigma SiLU(0) = mu for the second; sigma from numpy's std."""
    d, m = 8, 6
    X = children(4, m, d, seed=14)
    W2 = np.zeros((d, 2 * d))
    W2[:, half * d:(half + 1) * d] = np.eye(d)
    P = params(d, w=np.zeros(d), W1=np.eye(2 * d), b1=np.zeros(2 * d), W2=W2, g=0.5)
    mu = X.mean(axis=1)
    sigma = np.sqrt(np.std(X - mu[:, None, :], axis=(1, 2)) ** 2 + O.GATED_EPS)
    if half == 0:
        act = torch.nn.functional.silu(torch.from_numpy(mu / P["rho"])).numpy()
        expect = mu + sigma[:, None] * act
    else:
        expect = mu
    np.testing.assert_allclose(O.gated_pool_keys(X, P), expect, rtol=0, atol=1e-12)


def test_ragged_node_uses_only_its_present_children():
    """Five tokens make one ragged node under C = 16 and under C = 32: the same key."""
    d = 16
    K0 = np.random.default_rng(6).standard_normal((5, d))
    V0 = np.random.default_rng(7).standard_normal((5, d))
    P = params(d)
    a = O.build_tree_gated(K0, V0, 16, P, "f32")
    b = O.build_tree_gated(K0, V0, 32, P, "f32")
    assert len(a) == len(b) == 2
    np.testing.assert_array_equal(a[1][0], b[1][0])


def test_values_keep_eq1_means():
    d, C, n = 16, 4, 37
    K0 = O.round_bf16(np.random.default_rng(8).standard_normal((n, d)))
    V0 = O.round_bf16(np.random.default_rng(9).standard_normal((n, d)))
    g = O.build_tree_gated(K0, V0, C, params(d), "bf16")
    e = O.build_tree(K0, V0, C, I.pooler_w(C).numpy(), "bf16")
    assert len(g) == len(e)
    for (_, Vg), (_, Ve) in zip(g, e):
        np.testing.assert_array_equal(Vg, Ve)


def test_dense_attention_when_k_exceeds_every_list():
    """Selection keeps everything, so the gated keys of the summaries never enter:
    the result is plain softmax attention over the tokens."""
    d, C, n, G = 16, 4, 50, 2
    rng = np.random.default_rng(10)
    K0, V0 = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    q = rng.standard_normal((G, d))
    levels = O.build_tree_gated(K0, V0, C, params(d), "f32")
    t = n - 1
    res = O.select_and_attend(levels, q, t, C, k=10_000)
    K, V = levels[0]
    s = O.level_logits(q, K[: t + 1], t, np.arange(t + 1), 1.0 / np.sqrt(d), 1e6)
    wts = np.exp(s - s.max(axis=1, keepdims=True))
    dense = (wts @ V[: t + 1]) / wts.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(res.out, dense, rtol=1e-10, atol=1e-12)
