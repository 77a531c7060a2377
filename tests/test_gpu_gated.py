"""GPU parity of the Eq.5 gated key pooler ("Pooler Distillation"), forward only,
through the C ABI (recsa_tree_set_gated_pooler), against the fp64 oracle.

Tolerance: each level of the GPU tree is compared with the oracle's Eq.5 pooling of
the GPU's own level below (so a rounding difference never cascades): keys within one
unit in the last place of the storage dtype (both sides compute in fp64, but the
MLP's and the reductions' summation orders differ, which can move a result that lies
within ~1e-15 of a rounding boundary), values bit for bit (Eq.1's mean, the same
sums on both sides).  Selections and outputs of a decode on the gated tree are then
checked against the oracle run on that same tree.
"""
import numpy as np
import pytest
import torch

from long_context_recsa_b200 import inputs as I
from oracle import recsa_oracle as O
from tests import parity_helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def R():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_recsa_b200 import build
    build.build()
    import long_context_recsa_b200.recsa as R
    return R


def gated_params(d, h):
    """The seeded stand-in parameters: numpy for the oracle, fp64 device tensors
    (W1 and W2 transposed) for the library."""
    P = {k: (v.numpy().copy() if hasattr(v, "numpy") else v)
         for k, v in I.gated_pooler_params(d, hidden=h).items()}
    dev = {"hidden": h, "tau": P["tau"], "g": P["g"], "rho": P["rho"],
           "w": torch.from_numpy(P["w"]).cuda(),
           "W1t": torch.from_numpy(np.ascontiguousarray(P["W1"].T)).cuda(),
           "b1": torch.from_numpy(P["b1"]).cuda(),
           "W2t": torch.from_numpy(np.ascontiguousarray(P["W2"].T)).cuda()}
    return P, dev


def ulp_diff(got, want, dtype):
    """|got - want| in units of the storage dtype's last place at the larger magnitude."""
    bits = 8 if dtype == "bf16" else 24
    mag = np.maximum(np.abs(got), np.abs(want))
    e = np.floor(np.log2(np.where(mag > 0, mag, 1.0)))
    ulp = np.ldexp(1.0, (e - (bits - 1)).astype(np.int64))
    return np.abs(got - want) / ulp


def gpu_levels(tree, K, V, b, h, L, C):
    """The GPU tree of unit (b, h) as the oracle's level list (fp64)."""
    levels = [(H.to64(K[b, h, :L]), H.to64(V[b, h, :L]))]
    n, lvl = L, 1
    while n > 1:
        n = -(-n // C)
        Kl, Vl = tree.level_tables(lvl)
        levels.append((H.to64(Kl[b, h, :n]), H.to64(Vl[b, h, :n])))
        lvl += 1
    return levels


def check_gated_tree(levels, C, P, dtype):
    """Each GPU level against the oracle's gated pooling of the GPU level below."""
    worst, ndiff, ntot = 0.0, 0, 0
    for lvl in range(1, len(levels)):
        Kp, Vp = O.pool_level_gated(levels[lvl - 1][0], levels[lvl - 1][1], C, P, dtype)
        Kg, Vg = levels[lvl]
        np.testing.assert_array_equal(Vg, Vp, err_msg=f"V level {lvl}")
        u = ulp_diff(Kg, Kp, dtype)
        worst = max(worst, float(u.max()))
        ndiff += int((u > 0).sum())
        ntot += u.size
        assert float(u.max()) <= 1.0, f"K level {lvl}: {float(u.max())} ulp"
    return worst, ndiff, ntot


@pytest.mark.parametrize("dtype,d,C,G", [("bf16", 128, 16, 4), ("f32", 64, 4, 2), ("bf16", 64, 8, 1)])
def test_gated_tree_and_decode_against_oracle(R, dtype, d, C, G):
    k, Hkv, B = 8, 2, 2
    Hq = G * Hkv
    lengths = [3000, 1234]
    cap = 3000
    cfg = R.Config(head_dim=d, n_q_heads=Hq, n_kv_heads=Hkv, C=C, k=k, dtype=dtype,
                   pooler_w=H.w_for(C))
    K, V, q = H.make_inputs(31, B, Hkv, Hq, d, cap, lengths, dtype, n_needles=3)
    q = q[:, 0].contiguous()
    P, Pd = gated_params(d, 64)
    tree = R.RecsaTree(cfg, cap, B, k0=K, v0=V)
    tree.recsa_tree_set_gated_pooler(Pd)
    tree.recsa_build(lengths)
    out, sel, cnt = tree.decode(q, with_sel=True)
    torch.cuda.synchronize()
    assert tree.recsa_get_status() == R.RECSA_OK
    worst = 0.0
    for b in range(B):
        for h in range(Hkv):
            L = lengths[b]
            levels = gpu_levels(tree, K, V, b, h, L, C)
            w_ulp, nd, nt = check_gated_tree(levels, C, P, dtype)
            worst = max(worst, w_ulp)
            qg = H.to64(q[b, h * G:(h + 1) * G])
            res = O.select_and_attend(levels, qg, L - 1, C, k, base=1e6)
            cur = H.check_selection(levels, qg, L - 1, C, k, 1e6, res, sel[b, h].cpu().numpy(),
                                    cnt[b, h].cpu().numpy(), tree.n_sel_levels)
            err = H.max_abs(H.to64(out[b, h * G:(h + 1) * G]), cur.out)
            assert err <= H.TOL_OUT[dtype], f"unit {(b, h)}: output max-abs {err}"
    print(f"gated {dtype} d={d} C={C}: worst key difference {worst} ulp")


def test_gated_append_equals_build_bitwise(R):
    """Single-token appends and a multi-token append re-pool the ancestors with the same
    per-node routine as the build: tables bit for bit, and the decode outputs."""
    C, k, d, Hkv, Hq, B = 16, 8, 128, 2, 8, 2
    L0, steps, chunk = 3000, 5, 100
    cap = L0 + steps + chunk
    cfg = R.Config(head_dim=d, n_q_heads=Hq, n_kv_heads=Hkv, C=C, k=k, dtype="bf16",
                   pooler_w=H.w_for(C))
    K, V, q = H.make_inputs(32, B, Hkv, Hq, d, cap, [cap] * B, "bf16")
    q = q[:, 0].contiguous()
    _, Pd = gated_params(d, 32)
    Ka, Va = K.clone(), V.clone()
    Ka[:, :, L0:] = 0
    Va[:, :, L0:] = 0
    inc = R.RecsaTree(cfg, cap, B, k0=Ka, v0=Va)
    inc.recsa_tree_set_gated_pooler(Pd)
    inc.recsa_build([L0] * B)
    for s in range(steps):
        inc.recsa_append(K[:, :, L0 + s:L0 + s + 1].contiguous(),
                         V[:, :, L0 + s:L0 + s + 1].contiguous())
    inc.recsa_append(K[:, :, L0 + steps:].contiguous(), V[:, :, L0 + steps:].contiguous())
    out_inc = inc.decode(q)[0]
    full = R.RecsaTree(cfg, cap, B, k0=K.clone(), v0=V.clone())
    full.recsa_tree_set_gated_pooler(Pd)
    full.recsa_build([cap] * B)
    out_full = full.decode(q)[0]
    torch.cuda.synchronize()
    assert inc.recsa_get_status() == R.RECSA_OK and full.recsa_get_status() == R.RECSA_OK
    for lvl in range(1, full.n_levels):
        Ki, Vi = inc.level_tables(lvl)
        Kf, Vf = full.level_tables(lvl)
        n = -(-cap // C ** lvl)
        assert torch.equal(Ki[:, :, :n], Kf[:, :, :n]), f"K level {lvl}"
        assert torch.equal(Vi[:, :, :n], Vf[:, :, :n]), f"V level {lvl}"
    assert torch.equal(out_inc, out_full)


def test_gated_switch_back_and_rejections(R):
    """p = NULL restores the stand-in pooler (tables equal a plain build); widths
    beyond the shared-memory limit and bad pointers are rejected on the host."""
    C, k, d = 16, 8, 64
    cfg = R.Config(head_dim=d, n_q_heads=2, n_kv_heads=1, C=C, k=k, dtype="f32",
                   pooler_w=H.w_for(C))
    K, V, _ = H.make_inputs(33, 1, 1, 2, d, 700, [700], "f32")
    _, Pd = gated_params(d, 16)
    a = R.RecsaTree(cfg, 700, 1, k0=K, v0=V)
    a.recsa_tree_set_gated_pooler(Pd)
    a.recsa_build([700])
    Kg, _ = a.level_tables(1)
    Kg = Kg.clone()
    a.recsa_tree_set_gated_pooler(None)
    a.recsa_build([700])
    b = R.RecsaTree(cfg, 700, 1, k0=K.clone(), v0=V.clone())
    b.recsa_build([700])
    torch.cuda.synchronize()
    for lvl in range(1, b.n_levels):
        assert torch.equal(a.level_tables(lvl)[0], b.level_tables(lvl)[0])
    assert not torch.equal(Kg, b.level_tables(1)[0])   # the gated keys differ
    big = dict(Pd, hidden=65)
    with pytest.raises(R.RecsaError) as e:
        a.recsa_tree_set_gated_pooler(big)
    assert e.value.status == R.RECSA_E_UNSUPPORTED
    bad = dict(Pd, rho=0.0)
    with pytest.raises(R.RecsaError) as e:
        a.recsa_tree_set_gated_pooler(bad)
    assert e.value.status == R.RECSA_E_INVAL
