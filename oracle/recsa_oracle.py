"""Plain fp64 CPU oracle for the RecSA build -> select -> attend path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code, table or
constant with the CUDA library; its inputs are plain arrays.

Source: "Recursive Sparse Attention: Million-Token Length Extrapolation at
Logarithmic Cost" (arXiv:2611.07232), as summarised on the picx.dev page
(sections "Tree Construction" Eq.1, "Hierarchical Selection" Eq.3, "Unified
Softmax" Eq.4, "Key Theoretical Insight" for candidate-local RoPE) and on the
arXiv abstract page.

Every floating-point step runs in fp64.  The only narrower arithmetic is the
storage rounding of each tree level (round-to-nearest-even to the storage
dtype), because the stored, rounded level is what the next level and the
attention read.

Readings where the pages are silent (each also listed in the design notes):
  * pooler: stand-in ``alpha = softmax(w)`` over the C children, one w in R^C
    shared by every level and head; a ragged last node with m < C children
    renormalises the softmax over its m present children and averages V over m.
  * depth: the tree is built until a level has one node; Eq.3 starts there.
  * importance I (Eq.2 is missing from the pages): the same scaled RoPE'd logit
    Eq.4 uses, averaged over the query heads of one GQA group.
  * scale 1/sqrt(d); RoPE half-split pairing (j, j+d/2), theta_j = base^(-2j/d).
  * Eq.3 concatenation in ascending node order, so each list is in sequence
    order and the query's own ("current") entry is the last one.
  * ties in TopK go to the lower node index.
  * summaries enter Eq.4 with their per-head logits and no count bias.

Eq.5 ("Pooler Distillation"): ``gated_pool_keys`` / ``build_tree_gated``, the
gated key pooler, forward only, with seeded stand-in parameters (its readings are
listed beside it).  Its pins are in ``tests/test_oracle_gated_pooler.py``; the GPU
path is compared with it in ``tests/test_gpu_gated.py``.

Parity pins: see ``tests/test_oracle_pins.py`` (closed forms for summary values
and pooled keys, the C*k distance bound, the partition of [0..t] by the
attended entries, dense-attention reduction when k exceeds every list, the
q = 0 tie-break, needles, the GQA group-mean importance against a brute-force
selection with disagreeing heads, and per-head token weights of Eq.4 with
several heads).  No function here is "parity unpinned".
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# ---------------------------------------------------------------------------
# storage rounding
# ---------------------------------------------------------------------------

_BF16_MANT = 8          # significant bits of bfloat16 (1 implicit + 7 stored)
_BF16_MIN_QEXP = -133   # spacing of bfloat16 subnormals: 2^-126 * 2^-7


def round_bf16(x) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 (ties to even), return fp64.

    Exact single rounding: for |x| in [2^(e-1), 2^e) the bf16 spacing is
    2^(e-8) (clamped at the subnormal spacing 2^-133); scaling by a power of two
    is exact in fp64 and ``np.rint`` rounds half to even.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    q = np.maximum(e.astype(np.int64) - _BF16_MANT, _BF16_MIN_QEXP)
    y = np.ldexp(np.rint(np.ldexp(x, -q)), q)
    y = np.where(np.abs(y) >= 2.0 ** 128, np.copysign(np.inf, x), y)
    return np.where(np.isfinite(x), y, x)


def round_f32(x) -> np.ndarray:
    """Round fp64 values to the nearest fp32 (ties to even), return fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def storage_round(x, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return round_bf16(x)
    if dtype == "f32":
        return round_f32(x)
    if dtype == "f64":
        return np.asarray(x, dtype=np.float64)
    raise ValueError(f"unknown storage dtype {dtype!r}")


# ---------------------------------------------------------------------------
# Eq.1: tree construction
# ---------------------------------------------------------------------------

def pool_alpha(w: np.ndarray, m: int) -> np.ndarray:
    """Stand-in pooler weights for a node with m present children:
    softmax of w[0..m-1] in fp64."""
    z = np.asarray(w, dtype=np.float64)[:m]
    e = np.exp(z - z.max())
    return e / e.sum()


def pool_level(Kc: np.ndarray, Vc: np.ndarray, C: int, w: np.ndarray, dtype: str):
    """One application of Eq.1: parents of the n rows (Kc, Vc) of a level.

    Parent i has children C*i .. min(C*i+C-1, n-1).  K_i = sum_c alpha_c K_c
    (the stand-in pooler), V_i = mean of the children's V.  Both are rounded to
    the storage dtype.
    """
    n, d = Kc.shape
    n_par = -(-n // C)
    Kp = np.empty((n_par, d))
    Vp = np.empty((n_par, d))
    full = n // C
    if full:
        a = pool_alpha(w, C)
        Kp[:full] = np.einsum("c,icd->id", a, Kc[: full * C].reshape(full, C, d))
        Vp[:full] = Vc[: full * C].reshape(full, C, d).sum(axis=1) / C
    if n_par > full:                       # ragged last node
        m = n - full * C
        a = pool_alpha(w, m)
        Kp[full] = a @ Kc[full * C:]
        Vp[full] = Vc[full * C:].sum(axis=0) / m
    return storage_round(Kp, dtype), storage_round(Vp, dtype)


def build_tree(K0, V0, C: int, w, dtype: str):
    """Eq.1 applied until a level has a single node.

    K0, V0: [n, d] level-0 keys/values (already representable in ``dtype``).
    Returns a list of (K, V) per level, level 0 first.  An empty or single-token
    sequence has only level 0.
    """
    K = storage_round(K0, dtype)
    V = storage_round(V0, dtype)
    levels = [(K, V)]
    while levels[-1][0].shape[0] > 1:
        levels.append(pool_level(levels[-1][0], levels[-1][1], C, w, dtype))
    return levels


# ---------------------------------------------------------------------------
# Eq.5 gated pooler ("Pooler Distillation"), forward only
# ---------------------------------------------------------------------------
# Readings where the pages leave the step open (also in the design notes):
#   * x_c are the node's present children's stored keys (m <= C of them);
#   * mu = their mean (a vector); sigma = their scalar spread about mu, the root
#     of the mean squared deviation over children and dimensions, plus GATED_EPS
#     inside the root so that identical children give a finite result;
#   * g, tau, rho are scalars; w in R^d; the MLP has hidden width h (a parameter),
#     W1 [h][2d], b1 [h], W2 [d][h] and no output bias;
#   * values keep Eq.1: the mean of the children's values;
#   * the result is rounded once to the storage dtype, as for Eq.1.
GATED_EPS = 1e-6


def _silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def gated_pool_keys(X: np.ndarray, P: dict) -> np.ndarray:
    """Eq.5 for nodes given as X [n][m][d] (n nodes of m present children each):
    alpha = softmax_c(tau w.(x_c - mu) / sigma), p = sum_c alpha_c x_c,
    m = W2 SiLU(W1 [mu/rho ; (p - mu)/sigma] + b1), K = mu + g (p - mu) + sigma m.
    Returns [n][d] in fp64 (not rounded)."""
    X = np.asarray(X, dtype=np.float64)
    n, mc, d = X.shape
    w = np.asarray(P["w"], dtype=np.float64)
    W1 = np.asarray(P["W1"], dtype=np.float64)
    b1 = np.asarray(P["b1"], dtype=np.float64)
    W2 = np.asarray(P["W2"], dtype=np.float64)
    tau, g, rho = float(P["tau"]), float(P["g"]), float(P["rho"])
    mu = X.mean(axis=1)                                               # [n][d]
    dev = X - mu[:, None, :]
    sigma = np.sqrt((dev ** 2).sum(axis=(1, 2)) / (mc * d) + GATED_EPS)   # [n]
    logits = tau * (dev @ w) / sigma[:, None]                         # [n][m]
    logits -= logits.max(axis=1, keepdims=True)
    a = np.exp(logits)
    a /= a.sum(axis=1, keepdims=True)
    p = np.einsum("nc,ncd->nd", a, X)
    z = np.concatenate([mu / rho, (p - mu) / sigma[:, None]], axis=1)    # [n][2d]
    mlp = _silu(z @ W1.T + b1) @ W2.T                                  # [n][d]
    return mu + g * (p - mu) + sigma[:, None] * mlp


def pool_level_gated(Kc: np.ndarray, Vc: np.ndarray, C: int, P: dict, dtype: str):
    """One level of the tree with the Eq.5 key pooler: parent i has children
    C*i .. min(C*i+C-1, n-1); K_i by Eq.5 over them, V_i their mean; both rounded
    to the storage dtype."""
    n, d = Kc.shape
    n_par = -(-n // C)
    Kp = np.empty((n_par, d))
    Vp = np.empty((n_par, d))
    full = n // C
    if full:
        Kp[:full] = gated_pool_keys(Kc[: full * C].reshape(full, C, d), P)
        Vp[:full] = Vc[: full * C].reshape(full, C, d).sum(axis=1) / C
    if n_par > full:                       # ragged last node
        m = n - full * C
        Kp[full] = gated_pool_keys(Kc[full * C:][None], P)[0]
        Vp[full] = Vc[full * C:].sum(axis=0) / m
    return storage_round(Kp, dtype), storage_round(Vp, dtype)


def build_tree_gated(K0, V0, C: int, P: dict, dtype: str):
    """build_tree with the Eq.5 key pooler at every level."""
    K = storage_round(K0, dtype)
    V = storage_round(V0, dtype)
    levels = [(K, V)]
    while levels[-1][0].shape[0] > 1:
        levels.append(pool_level_gated(levels[-1][0], levels[-1][1], C, P, dtype))
    return levels


# ---------------------------------------------------------------------------
# candidate-local RoPE and the per-entry logits
# ---------------------------------------------------------------------------

def rope_theta(d: int, base: float) -> np.ndarray:
    j = np.arange(d // 2, dtype=np.float64)
    return base ** (-2.0 * j / d)


def rope(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Half-split rotary embedding of rows x[..., d] at integer positions pos.

    Pair (j, j + d/2) is rotated by the angle pos * theta_j.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_theta(d, base)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def level_logits(q: np.ndarray, Krows: np.ndarray, p_q: int, p_e: np.ndarray,
                 scale: float, base: float) -> np.ndarray:
    """s[h, e] = scale * <R(p_q) q_h, R(p_e) K_e> for the G query heads q[h]."""
    qr = rope(q, np.full(q.shape[0], p_q), base)        # [G, d]
    kr = rope(Krows, p_e, base)                          # [n, d]
    return scale * (qr @ kr.T)                           # [G, n]


# ---------------------------------------------------------------------------
# Eq.3 selection and Eq.4 unified softmax
# ---------------------------------------------------------------------------

@dataclass
class LevelTrace:
    level: int
    A: np.ndarray                 # candidate node indices, ascending
    S: np.ndarray                 # selected node indices, ascending (current last)
    scored: bool                  # False when |A| <= k (everything selected)
    logits: np.ndarray | None = None   # [G, |A|-1] for A without the current entry
    importance: np.ndarray | None = None  # [|A|-1]
    positions: np.ndarray | None = None   # candidate-local positions used
    p_q: int = 0
    near_tie: bool = False        # (k-1)-th and k-th importance within the band
    kth: float = float("nan")     # (k-1)-th kept importance
    first_dropped: float = float("nan")


@dataclass
class QueryResult:
    out: np.ndarray               # [G, d]
    levels: list = field(default_factory=list)   # LevelTrace, top level first
    A0: np.ndarray | None = None
    E_levels: np.ndarray | None = None   # level of each attended entry
    E_nodes: np.ndarray | None = None    # node index of each attended entry
    E_logits: np.ndarray | None = None   # [G, |E|]


NEAR_TIE_REL = 1e-5
NEAR_TIE_ABS = 1e-7


def is_near_tie(u: float, v: float) -> bool:
    return abs(u - v) <= NEAR_TIE_REL * max(abs(u), abs(v)) + NEAR_TIE_ABS


def _expand(S: np.ndarray, C: int, a_below: int) -> np.ndarray:
    """Eq.3 third line: concat over i in S (ascending) of
    [C*i, ..., min(C*i + C - 1, a_below)]."""
    parts = [np.arange(C * i, min(C * i + C - 1, a_below) + 1) for i in S]
    return np.concatenate(parts).astype(np.int64)


def select_and_attend(levels, q, t: int, C: int, k: int, scale: float | None = None,
                      base: float = 1e6, forced: dict | None = None) -> QueryResult:
    """Run Eq.3 top-down for query position t, then Eq.4.

    levels: output of ``build_tree`` over a sequence of length n > t.
    q: [G, d] the query heads of one GQA group (fp64 values).
    forced: optional {level: S array}.  Used only where the tests have checked
      that the given set is one of the valid TopK sets at a stated near-tie
      (several results are correct there); the oracle then continues from that
      valid choice.
    """
    q = np.asarray(q, dtype=np.float64)
    G, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    top = len(levels) - 1
    a = [t // C ** l for l in range(top + 1)]
    A = np.arange(0, a[top] + 1, dtype=np.int64)
    res = QueryResult(out=np.zeros((G, d)))
    sum_lv, sum_nd, sum_lg, sum_V = [], [], [], []
    for l in range(top, 0, -1):
        Kl, Vl = levels[l]
        cur = a[l]
        assert A[-1] == cur, "the current entry must be last"
        nA = len(A)
        tr = LevelTrace(level=l, A=A, S=A, scored=False, p_q=nA - 1)
        if nA > k:
            cand = A[:-1]
            pos = np.arange(nA - 1)
            s = level_logits(q, Kl[cand], nA - 1, pos, scale, base)
            imp = s.mean(axis=0)
            order = np.lexsort((cand, -imp))            # I desc, then index asc
            keep = np.zeros(nA - 1, dtype=bool)
            keep[order[: k - 1]] = True
            if forced is not None and l in forced:
                fs = np.asarray(forced[l], dtype=np.int64)
                keep = np.isin(cand, fs)
                assert keep.sum() == k - 1 and fs[-1] == cur
            S = np.concatenate([cand[keep], [cur]])
            tr = LevelTrace(level=l, A=A, S=S, scored=True, logits=s, importance=imp,
                            positions=pos, p_q=nA - 1)
            if k - 1 >= 1:
                tr.kth = float(imp[order[k - 2]])
                tr.first_dropped = float(imp[order[k - 1]])
                tr.near_tie = is_near_tie(tr.kth, tr.first_dropped)
            un = ~keep
            sum_lv.append(np.full(un.sum(), l))
            sum_nd.append(cand[un])
            sum_lg.append(s[:, un])
            sum_V.append(Vl[cand[un]])
        res.levels.append(tr)
        A = _expand(tr.S, C, a[l - 1])
    K0, V0 = levels[0]
    res.A0 = A
    s0 = level_logits(q, K0[A], len(A) - 1, np.arange(len(A)), scale, base)
    lg = np.concatenate([s0] + sum_lg, axis=1)
    Vall = np.concatenate([V0[A]] + sum_V, axis=0)
    mx = lg.max(axis=1, keepdims=True)
    p = np.exp(lg - mx)
    res.out = (p @ Vall) / p.sum(axis=1, keepdims=True)
    res.E_levels = np.concatenate([np.zeros(len(A), dtype=np.int64)] + sum_lv)
    res.E_nodes = np.concatenate([A] + sum_nd)
    res.E_logits = lg
    return res


# ---------------------------------------------------------------------------
# list sizes without scoring (they depend only on t, C, k)
# ---------------------------------------------------------------------------

def list_sizes(t: int, C: int, k: int):
    """Sizes |A^(l)| for l = top..0 and the number of attended entries |E|.

    The sizes of Eq.3's lists do not depend on which nodes are selected, only on
    how many: |S| = min(k, |A|), the current node last with its children
    clamped at a^(l-1).
    """
    top = 0
    while C ** top <= t:
        top += 1
    a = [t // C ** l for l in range(top + 1)]
    nA = a[top] + 1
    sizes = {}
    n_sum = 0
    for l in range(top, 0, -1):
        sizes[l] = nA
        nS = min(k, nA)
        n_sum += nA - nS
        nA = C * (nS - 1) + (a[l - 1] - C * a[l] + 1)
    sizes[0] = nA
    return sizes, nA + n_sum
