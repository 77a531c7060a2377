"""Pins of the fp64 oracle to facts the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a closed
form, an invariant, a library routine, a brute-force textbook computation or a
number printed on (or worked by hand from) the pages.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import recsa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(12345)


def _golden_constants():
    out = {}
    for line in open(os.path.join(GOLDEN, "paper_constants.txt")):
        line = line.split("#")[0].strip()
        if line:
            name, val = line.split()
            out[name] = float(val)
    return out


# --------------------------------------------------------------------- rounding

def test_round_bf16_matches_torch_single_rounding():
    # fp32 inputs: torch's fp32 -> bf16 conversion is a single RNE rounding.
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
        rng.standard_normal(2000) * 1e-39,              # fp32/bf16 subnormals
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-45]),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_round_bf16_ties_to_even_and_overflow():
    ulp = 2.0 ** -7
    assert O.round_bf16(1.0 + ulp / 2) == 1.0                    # tie -> even (1.0)
    assert O.round_bf16(1.0 + 3 * ulp / 2) == 1.0 + 2 * ulp      # tie -> even
    assert O.round_bf16(1.0 + ulp / 2 + 2.0 ** -40) == 1.0 + ulp  # above the tie
    big = (2.0 - 2.0 ** -8) * 2.0 ** 127                          # halfway to 2^128
    assert np.isinf(O.round_bf16(big))
    assert O.round_bf16((2.0 - 2.0 ** -7) * 2.0 ** 127) == (2.0 - 2.0 ** -7) * 2.0 ** 127
    assert O.round_bf16(2.0 ** -134) == 0.0                       # tie to even subnormal 0
    assert O.round_bf16(3 * 2.0 ** -134) == 2.0 ** -132


# ------------------------------------------------------------ Eq.1: tree build

def test_summary_values_closed_form_ramp():
    """P1: a complete level-l node is the mean of its C^l tokens (mean of means
    over equal groups); with V_j = j the node i has value i*C^l + (C^l - 1)/2."""
    for C in (2, 4, 16):
        n = C ** 3 + 5
        d = 3
        V = np.repeat(np.arange(n, dtype=np.float64)[:, None], d, axis=1)
        K = rng.standard_normal((n, d))
        w = rng.standard_normal(C)
        levels = O.build_tree(K, V, C, w, "f64")
        for l in range(1, len(levels)):
            Vl = levels[l][1]
            full = n // C ** l
            i = np.arange(full)
            expect = i * C ** l + (C ** l - 1) / 2
            np.testing.assert_array_equal(Vl[:full, 0], expect)


def test_pooled_keys_closed_form_digits():
    """P2: K^l_i = sum_{r < C^l} prod_m alpha_{digit_m(r)} K_{i C^l + r}."""
    C, d = 4, 5
    n = C ** 3 * 2
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    w = rng.standard_normal(C)
    e = np.exp(w - w.max())
    alpha = e / e.sum()
    levels = O.build_tree(K, V, C, w, "f64")
    for l in (1, 2, 3):
        span = C ** l
        coef = np.ones(span)
        for r in range(span):
            rr = r
            for _ in range(l):
                coef[r] *= alpha[rr % C]
                rr //= C
        for i in range(n // span):
            expect = coef @ K[i * span:(i + 1) * span]
            np.testing.assert_allclose(levels[l][0][i], expect, rtol=1e-13, atol=1e-13)


def test_pooler_special_cases():
    C, d = 16, 8
    n = 16 * 16 * 3 + 7                       # ragged at every level
    K = rng.standard_normal((n, d))
    # w = 0: plain mean, equal to the value pooling (also on ragged nodes)
    lv = O.build_tree(K, K, C, np.zeros(C), "f64")
    for l in range(1, len(lv)):
        np.testing.assert_allclose(lv[l][0], lv[l][1], rtol=1e-14, atol=1e-14)
    # constant keys are preserved at every level (weights sum to one)
    Kc = np.tile(rng.standard_normal(d), (n, 1))
    lv = O.build_tree(Kc, Kc, C, rng.standard_normal(C), "f64")
    for l in range(1, len(lv)):
        np.testing.assert_allclose(lv[l][0], np.tile(Kc[0], (lv[l][0].shape[0], 1)),
                                   rtol=1e-14, atol=1e-14)
    # one-hot w: each node's key is the key of the first token of its subtree
    w = np.zeros(C)
    w[0] = 60.0
    lv = O.build_tree(K, K, C, w, "f64")
    for l in range(1, len(lv)):
        first = K[:: C ** l][: lv[l][0].shape[0]]
        np.testing.assert_allclose(lv[l][0], first, rtol=1e-20, atol=1e-20)


def test_tree_level_count_and_upper_fraction():
    """Levels until one node; levels >= 1 hold sum_l C^-l ~ 1/15 of level 0,
    below the pages' "< 7%" (picx.dev summary, Practical Implications)."""
    g = _golden_constants()
    C = int(g["C"])
    n = C ** 4
    lv = O.build_tree(np.zeros((n, 2)), np.zeros((n, 2)), C, np.zeros(C), "bf16")
    sizes = [x[0].shape[0] for x in lv]
    assert sizes == [n // C ** l for l in range(5)]
    assert sum(sizes[1:]) / sizes[0] < g["upper_levels_fraction"]


def test_bf16_storage_rounding_applied_per_level():
    C, d = 16, 4
    n = 300
    K = O.round_bf16(rng.standard_normal((n, d)))
    V = O.round_bf16(rng.standard_normal((n, d)))
    w = rng.standard_normal(C)
    lv = O.build_tree(K, V, C, w, "bf16")
    for l in range(1, len(lv)):
        for arr in lv[l]:
            np.testing.assert_array_equal(arr, O.round_bf16(arr))
        # next level pools the rounded level below
        Kp, Vp = O.pool_level(lv[l - 1][0], lv[l - 1][1], C, w, "bf16")
        np.testing.assert_array_equal(Kp, lv[l][0])
        np.testing.assert_array_equal(Vp, lv[l][1])


# ------------------------------------------------------------------ RoPE pins

def _rope_complex(x, pos, base):
    """Independent route: pair (j, j+d/2) as the complex number x_j + i x_{j+d/2}
    multiplied by exp(i * pos * base^(-2j/d))."""
    d = x.shape[-1]
    h = d // 2
    z = x[..., :h] + 1j * x[..., h:]
    theta = np.array([base ** (-(2.0 * j) / d) for j in range(h)])
    z = z * np.exp(1j * np.asarray(pos, dtype=np.float64)[..., None] * theta)
    return np.concatenate([z.real, z.imag], axis=-1)


def test_rope_matches_complex_rotation_and_qwen_convention():
    x = rng.standard_normal((7, 64))
    pos = np.array([0, 1, 2, 17, 255, 4095, 8191])
    np.testing.assert_allclose(O.rope(x, pos, 1e6), _rope_complex(x, pos, 1e6), rtol=1e-12, atol=1e-12)
    # library routine: transformers' rotate-half application (Qwen-style)
    from transformers.models.qwen3.modeling_qwen3 import apply_rotary_pos_emb
    theta = O.rope_theta(64, 1e6)
    ang = pos[:, None] * theta
    cos = torch.from_numpy(np.concatenate([np.cos(ang)] * 2, axis=-1))[None]
    sin = torch.from_numpy(np.concatenate([np.sin(ang)] * 2, axis=-1))[None]
    xt = torch.from_numpy(x)[None, None]
    qr, _ = apply_rotary_pos_emb(xt, xt, cos, sin)
    np.testing.assert_allclose(O.rope(x, pos, 1e6), qr[0, 0].numpy(), rtol=1e-12, atol=1e-12)
    # relative-position property: <R(a)q, R(b)k> = <R(a-b)q, k>
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for a_, b_ in [(5, 3), (4095, 0), (100, 100)]:
        lhs = O.rope(q, a_, 1e4) @ O.rope(k, b_, 1e4)
        rhs = O.rope(q, a_ - b_, 1e4) @ k
        assert abs(lhs - rhs) < 1e-10


# ---------------------------------------------------------- Eq.3 / Eq.4 pins

def _tree(n, d, C, seed, dtype="f64", w=None):
    r = np.random.default_rng(seed)
    K = r.standard_normal((n, d))
    V = r.standard_normal((n, d))
    if w is None:
        w = r.standard_normal(C)
    return O.build_tree(K, V, C, w, dtype), K, V


def _covered(levels_e, nodes_e, C):
    out = []
    for l, i in zip(levels_e, nodes_e):
        out.append(np.arange(i * C ** l, (i + 1) * C ** l))
    return np.concatenate(out)


@pytest.mark.parametrize("C,k,n", [(2, 2, 200), (4, 3, 700), (16, 8, 4096), (16, 4, 5000), (3, 5, 1000)])
def test_partition_distance_bound_and_sizes(C, k, n):
    """P3 + P5: the attended entries' subtrees tile [0..t] exactly; every list
    has at most C*k entries, the current entry is last and every candidate-local
    distance lies in [0, C*k - 1]; sizes agree with the hand count."""
    d, G = 8, 2
    lv, _, _ = _tree(n, d, C, 7)
    q = rng.standard_normal((G, d))
    for t in sorted(set([0, 1, C - 1, C, n // 2, n - 2, n - 1] + list(rng.integers(0, n, 6)))):
        res = O.select_and_attend(lv, q, int(t), C, k)
        cov = np.sort(_covered(res.E_levels, res.E_nodes, C))
        np.testing.assert_array_equal(cov, np.arange(t + 1))
        sizes, nE = O.list_sizes(int(t), C, k)
        assert nE == len(res.E_nodes)
        for tr in res.levels:
            assert len(tr.A) <= C * k
            assert tr.A[-1] == t // C ** tr.level
            assert tr.S[-1] == tr.A[-1]
            assert np.all(np.diff(tr.S) > 0)
            if tr.level in sizes:
                assert sizes[tr.level] == len(tr.A)
            if tr.scored:
                dist = tr.p_q - tr.positions
                assert dist.min() >= 1 and dist.max() <= C * k - 1
                assert len(tr.S) == k
        assert len(res.A0) <= C * k and res.A0[-1] == t
        assert sizes[0] == len(res.A0)


def test_golden_list_sizes_and_distance_bound():
    g = _golden_constants()
    C, k = int(g["C"]), int(g["k"])
    assert C * k == g["max_distance_exclusive"]
    for line in open(os.path.join(GOLDEN, "list_sizes.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        L, C_, k_, nE, a0, a1, a2, a3 = (int(v) for v in line.split())
        sizes, got = O.list_sizes(L - 1, C_, k_)
        assert got == nE
        assert [sizes[0], sizes[1], sizes[2], sizes[3]] == [a0, a1, a2, a3]
        # O(log L) reads (summary page, Theoretical Contributions 1): every list
        # is bounded by C*k, so the total is at most (#levels) * C*k.
        assert sum(sizes.values()) <= len(sizes) * C_ * k_


@pytest.mark.parametrize("C", [2, 4, 16])
def test_dense_reduction_when_k_exceeds_lists(C):
    """P6: with k >= every list size RecSA selects everything, the level-0 list is
    [0..t] at its absolute positions, and Eq.4 is dense causal RoPE attention.
    Checked against a textbook loop (complex-number RoPE) and torch SDPA."""
    n, d, G = 300, 16, 3
    lv, K, V = _tree(n, d, C, 11)
    q = rng.standard_normal((G, d))
    base = 1e4
    for t in (0, 1, 37, n - 1):
        res = O.select_and_attend(lv, q, t, C, k=10 ** 6, base=base)
        assert len(res.E_nodes) == t + 1 and np.all(res.E_levels == 0)
        qr = _rope_complex(q, np.full(G, t), base)
        kr = _rope_complex(K[: t + 1], np.arange(t + 1), base)
        expect = np.zeros((G, d))
        for h in range(G):
            s = np.array([qr[h] @ kr[j] for j in range(t + 1)]) / math.sqrt(d)
            p = np.exp(s - s.max())
            expect[h] = (p[:, None] * V[: t + 1]).sum(0) / p.sum()
        np.testing.assert_allclose(res.out, expect, rtol=1e-12, atol=1e-12)
        sd = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qr)[None, :, None, :],
            torch.from_numpy(np.repeat(kr[None], G, 0))[None],
            torch.from_numpy(np.repeat(V[: t + 1][None], G, 0))[None])
        np.testing.assert_allclose(res.out, sd[0, :, 0].numpy(), rtol=1e-12, atol=1e-12)


def test_zero_query_tie_break_and_equal_weights():
    """P7: q = 0 makes every importance 0, so TopK keeps the k-1 lowest indices
    of each list, and Eq.4 gives every attended entry the same weight."""
    C, k, n, d = 4, 3, 500, 6
    lv, _, _ = _tree(n, d, C, 3)
    q = np.zeros((2, d))
    t = n - 1
    res = O.select_and_attend(lv, q, t, C, k)
    for tr in res.levels:
        if tr.scored:
            np.testing.assert_array_equal(tr.S[:-1], tr.A[: k - 1])
    rows = np.stack([lv[l][1][i] for l, i in zip(res.E_levels, res.E_nodes)])
    np.testing.assert_allclose(res.out, np.tile(rows.mean(0), (2, 1)), rtol=1e-13, atol=1e-13)


def test_needle_is_found_through_every_level():
    """A token whose key points along the query dominates: each of its ancestors
    is selected at every scored level and the output approaches its value."""
    C, k, n, d = 16, 8, 4096, 64
    r = np.random.default_rng(5)
    K = r.standard_normal((n, d)) * 0.1
    V = r.standard_normal((n, d))
    q = r.standard_normal((2, d))
    j = 1234
    K[j] = 40.0 * q.mean(0)          # before RoPE; candidate-local positions move it
    lv = O.build_tree(K, V, C, np.zeros(C), "f64")
    t = n - 1
    res = O.select_and_attend(lv, q, t, C, k, base=1e6)
    for tr in res.levels:
        if tr.scored:
            assert j // C ** tr.level in tr.S
    assert j in res.A0


def test_token_weights_of_unified_softmax():
    """Eq.4 assembly, pinned through linearity in V: with V = identity rows each
    output coordinate is the weight Eq.4 gives one token.  Tokens inside an
    unselected summary share its weight equally (its value is their mean), level-0
    tokens get exp(s)/Z, all tokens of [0..t] get positive weight, and the weights
    sum to one.  Logits are recomputed here via the complex-number RoPE route."""
    C, k, d = 2, 2, 64
    n = 64
    r = np.random.default_rng(9)
    K = r.standard_normal((n, d))
    V = np.eye(n, d)
    lv = O.build_tree(K, V, C, r.standard_normal(C), "f64")
    q = r.standard_normal((1, d))
    t = n - 1
    base = 1e4
    res = O.select_and_attend(lv, q, t, C, k, base=base)
    wts = res.out[0]
    assert np.all(wts[: t + 1] > 0)
    assert abs(wts.sum() - 1) < 1e-12
    # recompute each attended entry's logit independently
    logits, spans = [], []
    for tr in res.levels:
        if not tr.scored:
            continue
        Kl = lv[tr.level][0]
        for pos, node in enumerate(tr.A[:-1]):
            if node in tr.S:
                continue
            qr = _rope_complex(q[0], tr.p_q, base)
            kr = _rope_complex(Kl[node], pos, base)
            logits.append(qr @ kr / math.sqrt(d))
            spans.append(np.arange(node * C ** tr.level, (node + 1) * C ** tr.level))
    A0 = res.A0
    for pos, tok in enumerate(A0):
        qr = _rope_complex(q[0], len(A0) - 1, base)
        kr = _rope_complex(K[tok], pos, base)
        logits.append(qr @ kr / math.sqrt(d))
        spans.append(np.array([tok]))
    logits = np.array(logits)
    p = np.exp(logits - logits.max())
    p /= p.sum()
    expect = np.zeros(n)
    for pi, sp in zip(p, spans):
        expect[sp] += pi / len(sp)
    np.testing.assert_allclose(wts, expect, rtol=1e-12, atol=1e-14)


def test_near_tie_band():
    assert O.is_near_tie(1.0, 1.0 - 5e-6)
    assert not O.is_near_tie(1.0, 1.0 - 5e-5)
    assert O.is_near_tie(0.0, 5e-8)


def test_forced_selection_reproduces_own_choice():
    C, k, n, d = 16, 8, 4096, 16
    lv, _, _ = _tree(n, d, C, 21)
    q = rng.standard_normal((2, d))
    res = O.select_and_attend(lv, q, n - 1, C, k)
    forced = {tr.level: tr.S for tr in res.levels if tr.scored}
    res2 = O.select_and_attend(lv, q, n - 1, C, k, forced=forced)
    np.testing.assert_array_equal(res.out, res2.out)


# --------------------------------------------------------------- GQA pins

def _brute_selection(levels, q, t, C, k, base):
    """Eq.3 top-down written out with explicit loops, for a GQA group q [G, d]:
    per-head logits through the complex-number RoPE route at candidate-local
    positions, importance = (1/G) * the sum over the group's heads, TopK by a
    sort on (importance descending, node ascending), then the children of the kept
    nodes.  Returns {level: S} for the scored levels and {0: A^(0)}."""
    G, d = q.shape
    top = len(levels) - 1
    a = [t // C ** l for l in range(top + 1)]
    A = list(range(a[top] + 1))
    out = {}
    for l in range(top, 0, -1):
        if len(A) > k:
            p_q = len(A) - 1
            qr = [_rope_complex(q[g], p_q, base) for g in range(G)]
            imp = {}
            for pos, node in enumerate(A[:-1]):
                kr = _rope_complex(levels[l][0][node], pos, base)
                tot = 0.0
                for g in range(G):
                    tot += float(np.dot(qr[g], kr)) / math.sqrt(d)
                imp[node] = tot / G
            ranked = sorted(A[:-1], key=lambda n: (-imp[n], n))
            S = sorted(ranked[: k - 1]) + [A[-1]]
            out[l] = S
        else:
            S = A
        A = [c for i in S for c in range(C * i, min(C * i + C - 1, a[l - 1]) + 1)]
    out[0] = A
    return out


def test_gqa_importance_is_the_group_mean_against_brute_force():
    """The importance of Eq.3 for a GQA group is the mean of its heads' logits
    (the stand-in for the importance the pages do not define).  Two heads that
    disagree (q1 ~ -q0) make the mean's ranking differ from either head's own, so
    selecting by one head, or by anything but the mean, changes some S; the oracle's
    sets must equal the brute-force mean selection at every scored level."""
    C, k, n, d = 4, 5, 1500, 16
    r = np.random.default_rng(31)
    K = r.standard_normal((n, d))
    V = r.standard_normal((n, d))
    lv = O.build_tree(K, V, C, r.standard_normal(C), "f64")
    q0 = r.standard_normal(d)
    q = np.stack([q0, -q0 + 0.4 * r.standard_normal(d)])
    base = 1e4
    differs_from_single_head = set()
    for t in (n - 1, 1234, 777):
        res = O.select_and_attend(lv, q, t, C, k, base=base)
        want = _brute_selection(lv, q, t, C, k, base)
        by_head = [_brute_selection(lv, q[[g]], t, C, k, base) for g in range(2)]
        scored = [tr for tr in res.levels if tr.scored]
        assert scored and sorted(want) == sorted([tr.level for tr in scored] + [0])
        for tr in scored:
            np.testing.assert_array_equal(tr.S, want[tr.level], err_msg=f"t={t} level {tr.level}")
            for g in range(2):
                if list(by_head[g][tr.level]) != list(want[tr.level]):
                    differs_from_single_head.add(g)
        np.testing.assert_array_equal(res.A0, want[0])
    # the case has teeth: each head alone would have chosen differently somewhere
    assert differs_from_single_head == {0, 1}


def test_token_weights_per_head_with_gqa():
    """Eq.4 indexes the logits by head: with G = 3 heads sharing one selection and
    V = identity rows, row h of the output is the weight head h's own softmax gives
    every token (a summary's weight split equally over its tokens), recomputed here
    from that head's logits via the complex-number RoPE route."""
    C, k, d, n, G = 2, 2, 64, 64, 3
    r = np.random.default_rng(17)
    K = r.standard_normal((n, d))
    V = np.eye(n, d)
    lv = O.build_tree(K, V, C, r.standard_normal(C), "f64")
    q = r.standard_normal((G, d)) * np.array([[1.0], [2.0], [-1.5]])
    t, base = n - 1, 1e4
    res = O.select_and_attend(lv, q, t, C, k, base=base)
    entries = []                       # (level, node, candidate-local position, p_q)
    for tr in res.levels:
        if tr.scored:
            for pos, node in enumerate(tr.A[:-1]):
                if node not in tr.S:
                    entries.append((tr.level, node, pos, tr.p_q))
    for pos, tok in enumerate(res.A0):
        entries.append((0, tok, pos, len(res.A0) - 1))
    assert any(e[0] > 0 for e in entries)
    for h in range(G):
        lg = np.array([_rope_complex(q[h], pq, base) @ _rope_complex(lv[l][0][node], pos, base)
                       / math.sqrt(d) for l, node, pos, pq in entries])
        p = np.exp(lg - lg.max())
        p /= p.sum()
        expect = np.zeros(n)
        for pi, (l, node, _, _) in zip(p, entries):
            span = np.arange(node * C ** l, (node + 1) * C ** l)
            expect[span] += pi / len(span)
        np.testing.assert_allclose(res.out[h], expect, rtol=1e-12, atol=1e-14,
                                   err_msg=f"head {h}")
    # heads with different queries get different weights (the pin can tell them apart)
    assert np.abs(res.out[0] - res.out[1]).max() > 1e-3
