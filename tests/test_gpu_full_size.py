"""GPU parity at the workloads' full sizes, in the launch configuration the bench
times, on sampled units and rows that the fp64 oracle computes one by one.

Inputs are drawn per (sequence, KV head) slice on the device from the seeded
generators (drawing gigabytes on the host would take minutes); the oracle gets a
copy of exactly the sampled slices.  Trees of the sampled units are compared bit
for bit, selections exactly (up to stated near-ties), outputs within 2e-2.
"""
import numpy as np
import pytest
import torch

from long_context_recsa_b200 import inputs as I
from tests import parity_helpers as H

pytestmark = pytest.mark.gpu

Hq, Hkv, d, C, k = 32, 8, 128, 16, 256
G = Hq // Hkv


@pytest.fixture(scope="module")
def R():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_recsa_b200 import build
    build.build()
    import long_context_recsa_b200.recsa as R
    return R


def device_inputs(config_id, B, L_cap, lengths, n_needles=0, q_rows=1):
    """K, V [B][Hkv][L_cap][d] and q [B][q_rows][Hq][d], bf16 on the device, drawn
    per slice from the seeded generators; needles along the group-mean of row 0."""
    dev = "cuda"
    K = torch.zeros(B, Hkv, L_cap, d, dtype=torch.bfloat16, device=dev)
    V = torch.zeros_like(K)
    q = torch.stack([I.q_rows(config_id, b, q_rows, Hq, d, "bf16", device=dev) for b in range(B)])
    for b in range(B):
        pos = I.needle_positions(config_id, b, n_needles, lengths[b]).to(dev) if n_needles else None
        for h in range(Hkv):
            Ks, Vs = I.kv_slice(config_id, b, h, lengths[b], d, "bf16", device=dev)
            if n_needles:
                Ks[pos] = I.needle_keys(q[b, 0, h * G:(h + 1) * G], 4.0, "bf16")
            K[b, h, :lengths[b]] = Ks
            V[b, h, :lengths[b]] = Vs
            del Ks, Vs
    return K, V, q


def check_unit(R, tree, K, V, q_group, b, h, L, t, w, sel_u, cnt_u, out_u, check_tree=True):
    levels, res = H.oracle_unit(K[b, h], V[b, h], q_group, L, t, C, k, w, "bf16", 1e6)
    if check_tree:
        H.compare_tree(tree, levels, b, h, "bf16")
    q64 = H.to64(q_group)
    cur = H.check_selection(levels, q64, t, C, k, 1e6, res, sel_u, cnt_u, tree.n_sel_levels)
    err = H.max_abs(H.to64(out_u), cur.out)
    assert err <= H.TOL_OUT["bf16"], f"unit {(b, h)} t={t}: output max-abs {err}"
    return err


def cfg_for(R, w):
    return R.Config(head_dim=d, n_q_heads=Hq, n_kv_heads=Hkv, C=C, k=k, dtype="bf16",
                    rope_base=1e6, pooler_w=w)


def test_decode_131k_all_heads_with_needles(R):
    """Single-layer decode at L = 131072, batch 1, 64 needles: every KV head."""
    L = 131072
    w = H.w_for(C)
    K, V, q = device_inputs(2, 1, L, [L], n_needles=64)
    q = q[:, 0].contiguous()
    tree = R.RecsaTree(cfg_for(R, w), L, 1, k0=K, v0=V)
    tree.recsa_build([L])
    out, sel, cnt = tree.decode(q, with_sel=True)
    torch.cuda.synchronize()
    assert tree.recsa_get_status() == R.RECSA_OK
    for h in range(Hkv):
        check_unit(R, tree, K, V, q[0, h * G:(h + 1) * G], 0, h, L, L - 1, w,
                   sel[0, h].cpu().numpy(), cnt[0, h].cpu().numpy(), out[0, h * G:(h + 1) * G])


def test_decode_524k_batch4_with_append_sampled_units(R):
    """The bench's workload: 4 sequences of 524288 tokens built, one token appended
    to each, then decode at t = L; three sampled (sequence, KV head) units."""
    L = 524288
    w = H.w_for(C)
    cap = L + 16
    K, V, q = device_inputs(3, 4, cap, [L + 1] * 4)
    q = q[:, 0].contiguous()
    Kb, Vb = K.clone(), V.clone()          # the build sees L tokens, the append adds one
    Kb[:, :, L:] = 0
    Vb[:, :, L:] = 0
    tree = R.RecsaTree(cfg_for(R, w), cap, 4, k0=Kb, v0=Vb)
    tree.recsa_build([L] * 4)
    tree.recsa_append(K[:, :, L:L + 1].contiguous(), V[:, :, L:L + 1].contiguous())
    out, sel, cnt = tree.decode(q, with_sel=True)
    torch.cuda.synchronize()
    assert tree.recsa_get_status() == R.RECSA_OK
    assert tree.host_lengths() == [L + 1] * 4
    del Kb, Vb
    for b, h in [(0, 0), (1, 5), (3, 7)]:
        check_unit(R, tree, K, V, q[b, h * G:(h + 1) * G], b, h, L + 1, L, w,
                   sel[b, h].cpu().numpy(), cnt[b, h].cpu().numpy(), out[b, h * G:(h + 1) * G])


def test_prefill_chunk_524k_sampled_rows(R):
    """A 4096-row chunk at positions 520192..524287 of a 524288-token tree with 256
    needles, on the tensor-core top level (max_queries 1024): sampled rows."""
    L, n = 524288, 4096
    pos0 = L - n
    w = H.w_for(C)
    K, V, Q = device_inputs(4, 1, L, [L], n_needles=256, q_rows=n)
    tree = R.RecsaTree(cfg_for(R, w), L, 1, max_queries=1024, k0=K, v0=V)
    assert tree.tc_queries > 0
    tree.recsa_build([L])
    O, sel, cnt = tree.prefill(Q, pos0, with_sel=True)
    torch.cuda.synchronize()
    assert tree.recsa_get_status() == R.RECSA_OK
    from oracle import recsa_oracle as O_
    for h in (0, 6):
        levels = O_.build_tree(H.to64(K[0, h]), H.to64(V[0, h]), C,
                               np.asarray(w, dtype=np.float64), "bf16")
        for i in (0, 1000, 2047, 4095):
            t = pos0 + i
            qg = H.to64(Q[0, i, h * G:(h + 1) * G])
            res = O_.select_and_attend(levels, qg, t, C, k, base=1e6)
            cur = H.check_selection(levels, qg, t, C, k, 1e6, res, sel[i, h].cpu().numpy(),
                                    cnt[i, h].cpu().numpy(), tree.n_sel_levels)
            err = H.max_abs(H.to64(O[0, i, h * G:(h + 1) * G]), cur.out)
            assert err <= H.TOL_OUT["bf16"], f"row {i} head {h}: output max-abs {err}"


def test_decode_2m_with_append_sampled_unit(R):
    """Long decode at L = 2097152, batch 1: build, append one token, decode; one
    sampled unit checked in full (tree, selections at all levels, output)."""
    L = 2097152
    w = H.w_for(C)
    cap = L + 16
    K, V, q = device_inputs(5, 1, cap, [L + 1])
    q = q[:, 0].contiguous()
    tree = R.RecsaTree(cfg_for(R, w), cap, 1, k0=K, v0=V)
    tree.recsa_build([L])
    tree.recsa_append(K[:, :, L:L + 1].contiguous(), V[:, :, L:L + 1].contiguous())
    out, sel, cnt = tree.decode(q, with_sel=True)
    torch.cuda.synchronize()
    assert tree.recsa_get_status() == R.RECSA_OK
    check_unit(R, tree, K, V, q[0, 2 * G:3 * G], 0, 2, L + 1, L, w,
               sel[0, 2].cpu().numpy(), cnt[0, 2].cpu().numpy(), out[0, 2 * G:3 * G])


def test_captured_decode_graph_long_replay_524k(R):
    """The bench's timed path: one captured append + decode graph replayed 120 times
    at L = 524288 (device-side lengths advance, the appended tokens' ancestors are
    re-pooled by the pass kernel's extra CTAs).  Replays 0, 1, 60 and 119 of two units
    are checked against the oracle, which is built once over the final length: for a
    query at t every listed node other than the current one covers tokens <= t only,
    and the current node is never scored nor a summary.  The final trees bit for bit."""
    L0, reps = 524288, 120
    checks = (0, 1, 60, reps - 1)
    units = (0, 5)
    w = H.w_for(C)
    cap = L0 + reps + 16
    K, V, _ = device_inputs(7, 1, cap, [L0 + reps])
    Q = I.q_rows(7, 0, reps, Hq, d, "bf16", device="cuda")
    Kb, Vb = K.clone(), V.clone()
    Kb[:, :, L0:] = 0
    Vb[:, :, L0:] = 0
    tree = R.RecsaTree(cfg_for(R, w), cap, 1, k0=Kb, v0=Vb)
    tree.recsa_build([L0])
    kst = torch.empty(1, Hkv, 1, d, dtype=torch.bfloat16, device="cuda")
    vst, qst = torch.empty_like(kst), torch.empty(1, Hq, d, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(qst)
    nl = tree.n_sel_levels
    sel = torch.empty(1, Hkv, nl, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(1, Hkv, nl + 1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.Stream()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(gr, stream=stream):
            tree.recsa_append(kst, vst)
            tree.recsa_decode(qst, out, sel, cnt)
    torch.cuda.synchronize()
    got = {}
    for r in range(reps):
        kst.copy_(K[:, :, L0 + r:L0 + r + 1])
        vst.copy_(V[:, :, L0 + r:L0 + r + 1])
        qst.copy_(Q[r:r + 1])
        gr.replay()
        if r in checks:
            torch.cuda.synchronize()
            got[r] = (out.clone(), sel.cpu().numpy(), cnt.cpu().numpy())
    torch.cuda.synchronize()
    del gr
    assert tree.recsa_get_status() == R.RECSA_OK
    # the host copy of the lengths saw the captured append once; replays advance only
    # the device-side lengths
    assert tree.host_lengths() == [L0 + 1]
    from oracle import recsa_oracle as O_
    for h in units:
        levels = O_.build_tree(H.to64(K[0, h, :L0 + reps]), H.to64(V[0, h, :L0 + reps]), C,
                               np.asarray(w, dtype=np.float64), "bf16")
        H.compare_tree(tree, levels, 0, h, "bf16")
        for r in checks:
            t = L0 + r
            qg = H.to64(Q[r, h * G:(h + 1) * G])
            res = O_.select_and_attend(levels, qg, t, C, k, base=1e6)
            o, sl, cn = got[r]
            cur = H.check_selection(levels, qg, t, C, k, 1e6, res, sl[0, h], cn[0, h], nl)
            err = H.max_abs(H.to64(o[0, h * G:(h + 1) * G]), cur.out)
            assert err <= H.TOL_OUT["bf16"], f"replay {r} head {h}: output max-abs {err}"
