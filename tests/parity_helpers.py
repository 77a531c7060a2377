"""Helpers for the GPU-vs-oracle parity tests (imported by tests only)."""
from __future__ import annotations

import math

import numpy as np
import torch

from long_context_recsa_b200 import inputs as I
from oracle import recsa_oracle as O

TOL_OUT = {"bf16": 2e-2, "f32": 1e-5}   # max-abs on attention outputs


def to64(x: torch.Tensor) -> np.ndarray:
    return x.detach().to("cpu", torch.float64).numpy()


def make_inputs(config_id, B, Hkv, Hq, d, L_cap, lengths, dtype, n_needles=0, gain=4.0,
                device="cuda", q_rows=1):
    """Seeded K, V (per slice, CPU generator) in a [B][Hkv][L_cap][d] device cache,
    q [B][q_rows][Hq][d]; needles placed along the group-mean query (first row)."""
    dt = I.torch_dtype(dtype)
    K = torch.zeros(B, Hkv, L_cap, d, dtype=dt)
    V = torch.zeros(B, Hkv, L_cap, d, dtype=dt)
    q = torch.stack([I.q_rows(config_id, b, q_rows, Hq, d, dtype) for b in range(B)])
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hkv):
            Ks, Vs = I.kv_slice(config_id, b, h, lengths[b], d, dtype)
            if n_needles:
                pos = I.needle_positions(config_id, b, n_needles, lengths[b])
                Ks[pos] = I.needle_keys(q[b, 0, h * G:(h + 1) * G], gain, dtype)
            K[b, h, : lengths[b]] = Ks
            V[b, h, : lengths[b]] = Vs
    return K.to(device), V.to(device), q.to(device)


def oracle_unit(K, V, q_group, L, t, C, k, w, dtype, base):
    """Oracle tree over L tokens of one (b, kvh) and its result at query position t."""
    levels = O.build_tree(to64(K[:L]), to64(V[:L]), C, np.asarray(w, dtype=np.float64), dtype)
    res = O.select_and_attend(levels, to64(q_group), t, C, k, base=base)
    return levels, res


def compare_tree(tree, levels, b, h, dtype):
    """GPU level tables of (b, h) against the oracle's levels, bit for bit."""
    for l in range(1, len(levels)):
        Kg, Vg = tree.level_tables(l)
        n = levels[l][0].shape[0]
        kg = to64(Kg[b, h, :n])
        vg = to64(Vg[b, h, :n])
        np.testing.assert_array_equal(kg, levels[l][0], err_msg=f"K level {l} (b={b}, h={h})")
        np.testing.assert_array_equal(vg, levels[l][1], err_msg=f"V level {l} (b={b}, h={h})")


def check_selection(levels, q_group, t, C, k, base, res, sel_gpu, cnt_gpu, NL):
    """Compare per-level selections.  Returns the oracle result to compare outputs
    with: the oracle's own, or, after a validated near-tie at some level, the
    oracle continued from the GPU's (valid) choice there."""
    forced = {}
    cur = res
    for _ in range(NL + 1):
        redo = False
        for tr in cur.levels:
            if not tr.scored:
                continue
            l = tr.level
            assert 1 <= l <= NL, (l, NL)
            assert int(cnt_gpu[l]) == len(tr.A), f"|A^({l})| gpu {int(cnt_gpu[l])} oracle {len(tr.A)}"
            g = np.asarray(sel_gpu[l - 1][:k], dtype=np.int64)
            if np.array_equal(g, tr.S):
                continue
            # accept only a near-tie swap: every differing node's importance lies in
            # the stated band around the (k-1)-th kept importance
            cand = tr.A[:-1]
            imp = dict(zip(cand.tolist(), tr.importance.tolist()))
            diff = set(g.tolist()) ^ set(tr.S.tolist())
            assert g[-1] == tr.S[-1], f"level {l}: current node must be last"
            assert len(set(g.tolist())) == k and np.all(np.diff(g) > 0), f"level {l}: GPU S invalid"
            for node in diff:
                assert node in imp, f"level {l}: node {node} not a candidate"
                assert O.is_near_tie(imp[node], tr.kth), (
                    f"level {l}: selection differs beyond the near-tie band: node {node} "
                    f"I={imp[node]!r} vs (k-1)-th {tr.kth!r}")
            forced[l] = g
            cur = O.select_and_attend(levels, q_group, t, C, k, base=base, forced=dict(forced))
            redo = True
            break
        if not redo:
            break
    for l in range(1, NL + 1):
        scored = [tr for tr in cur.levels if tr.scored and tr.level == l]
        if not scored:
            assert int(cnt_gpu[l]) == 0, f"level {l} should be unscored"
            assert np.all(np.asarray(sel_gpu[l - 1]) == -1)
    assert int(cnt_gpu[0]) == len(cur.A0)
    return cur


def max_abs(a, b):
    return float(np.max(np.abs(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64))))


def w_for(C):
    return I.pooler_w(C).tolist()


def scale_default(d):
    return 1.0 / math.sqrt(d)
