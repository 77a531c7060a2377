"""GPU parity: librecsa.so (through its C ABI) against the fp64 oracle.

Tree tables bit-exact; selected sets bit-exact except at stated near-ties (the
(k-1)-th and k-th importances within 1e-5 relative); attention outputs within
2e-2 max-abs for bf16 and 1e-5 for fp32.
"""
import numpy as np
import pytest
import torch

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


def run_decode_case(R, *, config_id, B, Hkv, Hq, d, C, k, lengths, dtype, cap=None,
                    n_needles=0, base=1e6, check_units=None, check_tree=True, q_fn=None):
    cap = cap or max(lengths)
    w = H.w_for(C)
    cfg = R.Config(head_dim=d, n_q_heads=Hq, n_kv_heads=Hkv, C=C, k=k, dtype=dtype,
                   rope_base=base, pooler_w=w)
    K, V, q = H.make_inputs(config_id, B, Hkv, Hq, d, cap, lengths, dtype, n_needles=n_needles)
    q = q[:, 0].contiguous()
    if q_fn is not None:
        q = q_fn(q).contiguous()
    tree = R.RecsaTree(cfg, cap, B, k0=K, v0=V)
    tree.recsa_build(lengths)
    out, sel, cnt = tree.decode(q, with_sel=True)
    torch.cuda.synchronize()
    assert tree.recsa_get_status() == R.RECSA_OK
    G = Hq // Hkv
    units = check_units or [(b, h) for b in range(B) for h in range(Hkv)]
    worst = 0.0
    for b, h in units:
        L = lengths[b]
        if L == 0:
            assert torch.all(out[b] == 0)
            continue
        t = L - 1
        levels, res = H.oracle_unit(K[b, h], V[b, h], q[b, h * G:(h + 1) * G], L, t, C, k, w,
                                    dtype, base)
        if check_tree:
            H.compare_tree(tree, levels, b, h, dtype)
        sel_u = sel[b, h].cpu().numpy() if tree.n_sel_levels else np.zeros((0, k))
        cur = H.check_selection(levels, H.to64(q[b, h * G:(h + 1) * G]), t, C, k, base, res,
                                sel_u, cnt[b, h].cpu().numpy(), tree.n_sel_levels)
        err = H.max_abs(H.to64(out[b, h * G:(h + 1) * G]), cur.out)
        worst = max(worst, err)
        assert err <= H.TOL_OUT[dtype], f"unit {(b, h)}: output max-abs {err}"
    return tree, worst


def test_tiny_fp32_config(R):
    """Tiny decode: 1 KV head, 2 query heads, d=64, L=4096, C=16, k=8, fp32."""
    _, worst = run_decode_case(R, config_id=1, B=1, Hkv=1, Hq=2, d=64, C=16, k=8,
                               lengths=[4096], dtype="f32")
    print("tiny fp32 worst max-abs", worst)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("C,k,d,G", [(4, 3, 64, 2), (16, 8, 128, 4), (2, 5, 64, 1), (8, 16, 128, 8),
                                     (16, 8, 128, 1), (16, 4, 128, 2), (16, 8, 128, 8)])
def test_small_ragged_batches(R, dtype, C, k, d, G):
    Hkv = 2
    lengths = [1000, 777, 64 * C + 1, 5]
    run_decode_case(R, config_id=11, B=4, Hkv=Hkv, Hq=G * Hkv, d=d, C=C, k=k, lengths=lengths,
                    dtype=dtype, cap=1100, n_needles=3)


def test_gqa_heads_that_disagree(R):
    """G = 4 query heads per KV head whose logits disagree (head 1 ~ -head 0, heads 2
    and 3 other directions): the selection follows the mean of the group's logits,
    which no single head's ranking gives, and each head keeps its own logits in the
    unified softmax."""
    G = 4

    def disagree(q):
        g = torch.Generator(device="cpu").manual_seed(4242)
        noise = torch.randn(q.shape, generator=g).to(q.device, q.dtype)
        qg = q.view(q.shape[0], -1, G, q.shape[-1]).clone()
        nz = noise.view_as(qg)
        qg[:, :, 1] = -qg[:, :, 0] + 0.4 * nz[:, :, 1]
        qg[:, :, 3] = -qg[:, :, 2] + 0.4 * nz[:, :, 3]
        return qg.view_as(q)

    run_decode_case(R, config_id=22, B=2, Hkv=2, Hq=2 * G, d=128, C=16, k=16,
                    lengths=[5000, 4321], dtype="bf16", cap=5000, q_fn=disagree)
    run_decode_case(R, config_id=22, B=1, Hkv=1, Hq=G, d=64, C=16, k=16, lengths=[5000],
                    dtype="f32", cap=5000, q_fn=disagree)


@pytest.mark.parametrize("L", [1, 2, 15, 16, 17, 255, 256, 257, 4095, 4096, 4097, 6000])
def test_edge_lengths(R, L):
    """Single token, exact powers of C, one past them, the dense regime (t < C*k,
    nothing scored) and the first scored lengths."""
    run_decode_case(R, config_id=12, B=1, Hkv=1, Hq=4, d=128, C=16, k=16, lengths=[L],
                    dtype="bf16", cap=max(L, 16))


def test_zero_length_sequence_outputs_zero(R):
    run_decode_case(R, config_id=13, B=2, Hkv=1, Hq=2, d=64, C=4, k=2, lengths=[0, 50],
                    dtype="f32", cap=64)


@pytest.mark.parametrize("C,k,d,L,dtype", [
    (4, 3, 64, 900, "f32"),          # short lists
    (16, 16, 128, 5000, "bf16"),     # every key tied inside the cluster's candidate bin
    (16, 64, 128, 30000, "bf16"),    # a tied bin too large for it: the exchange path
])
def test_zero_query_tie_break(R, C, k, d, L, dtype):
    """q = 0: all importances equal, TopK keeps the lowest indices (ties to the
    lower index), identical on GPU and oracle."""
    w = H.w_for(C)
    cfg = R.Config(head_dim=d, n_q_heads=2, n_kv_heads=1, C=C, k=k, dtype=dtype, pooler_w=w)
    K, V, _ = H.make_inputs(14, 1, 1, 2, d, L, [L], dtype)
    q = torch.zeros(1, 2, d, device="cuda", dtype=K.dtype)
    tree = R.RecsaTree(cfg, L, 1, k0=K, v0=V)
    tree.recsa_build([L])
    out, sel, cnt = tree.decode(q, with_sel=True)
    assert tree.recsa_get_status() == R.RECSA_OK
    levels, res = H.oracle_unit(K[0, 0], V[0, 0], q[0], L, L - 1, C, k, w, dtype, 1e6)
    n_scored = 0
    for tr in res.levels:
        if tr.scored:
            n_scored += 1
            np.testing.assert_array_equal(sel[0, 0, tr.level - 1].cpu().numpy(), tr.S)
            np.testing.assert_array_equal(tr.S[:-1], tr.A[: k - 1])
    assert n_scored >= 1
    assert H.max_abs(H.to64(out[0]), res.out) <= H.TOL_OUT[dtype]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_append_equals_build_bitwise(R, dtype):
    """build(L) then append one token at a time (and a multi-token chunk) equals
    build(L + n) bit for bit, tables and decode outputs."""
    C, k, d, Hkv, Hq, B = 16, 8, 128, 2, 8, 2
    L0, steps, chunk = 4000, 40, 300
    cap = L0 + steps + chunk
    w = H.w_for(C)
    cfg = R.Config(head_dim=d, n_q_heads=Hq, n_kv_heads=Hkv, C=C, k=k, dtype=dtype, pooler_w=w)
    K, V, q = H.make_inputs(15, B, Hkv, Hq, d, cap, [cap] * B, dtype)
    q = q[:, 0].contiguous()
    Ka = K.clone()
    Va = V.clone()
    Ka[:, :, L0:] = 0
    Va[:, :, L0:] = 0
    inc = R.RecsaTree(cfg, cap, B, k0=Ka, v0=Va)
    inc.recsa_build([L0] * B)
    outs_inc = []
    for s in range(steps):
        kn = K[:, :, L0 + s: L0 + s + 1].contiguous()
        vn = V[:, :, L0 + s: L0 + s + 1].contiguous()
        inc.recsa_append(kn, vn)
        outs_inc.append(inc.decode(q)[0])
    kn = K[:, :, L0 + steps:].contiguous()
    vn = V[:, :, L0 + steps:].contiguous()
    inc.recsa_append(kn, vn)
    out_inc_final = inc.decode(q)[0]
    torch.cuda.synchronize()
    assert inc.recsa_get_status() == R.RECSA_OK
    assert inc.host_lengths() == [cap] * B
    full = R.RecsaTree(cfg, cap, B, k0=K.clone(), v0=V.clone())
    full.recsa_build([cap] * B)
    for l in range(1, full.n_levels):
        Ki, Vi = inc.level_tables(l)
        Kf, Vf = full.level_tables(l)
        n = -(-cap // C ** l)
        assert torch.equal(Ki[:, :, :n], Kf[:, :, :n]), f"K level {l}"
        assert torch.equal(Vi[:, :, :n], Vf[:, :, :n]), f"V level {l}"
    assert torch.equal(out_inc_final, full.decode(q)[0])
    # intermediate steps against fresh builds at a few lengths
    for s in (0, 7, steps - 1):
        ref = R.RecsaTree(cfg, cap, B, k0=K.clone(), v0=V.clone())
        ref.recsa_build([L0 + s + 1] * B)
        assert torch.equal(outs_inc[s], ref.decode(q)[0]), f"step {s}"


def test_prefill_rows_equal_decode_on_truncated_tree(R):
    """Causality: prefill row t equals decode of a tree holding only [0..t]
    (bitwise, same kernels), and matches the oracle."""
    C, k, d, Hkv, Hq = 16, 8, 128, 2, 8
    L = 5000
    pos0, n = 4990, 10
    w = H.w_for(C)
    cfg = R.Config(head_dim=d, n_q_heads=Hq, n_kv_heads=Hkv, C=C, k=k, dtype="bf16", pooler_w=w)
    K, V, Q = H.make_inputs(16, 1, Hkv, Hq, d, L, [L], "bf16", q_rows=n, n_needles=5)
    tree = R.RecsaTree(cfg, L, 1, max_queries=8, k0=K, v0=V)
    tree.recsa_build([L])
    O, sel, cnt = tree.prefill(Q, pos0, with_sel=True)
    torch.cuda.synchronize()
    assert tree.recsa_get_status() == R.RECSA_OK
    G = Hq // Hkv
    for i in range(n):
        t = pos0 + i
        trunc = R.RecsaTree(cfg, L, 1, k0=K.clone(), v0=V.clone())
        trunc.recsa_build([t + 1])
        od, sd, cd = trunc.decode(Q[:, i].contiguous(), with_sel=True)
        assert torch.equal(O[:, i], od), f"row {i}"
        assert torch.equal(sel[i], sd[0]) and torch.equal(cnt[i], cd[0])
        for h in range(Hkv):
            levels, res = H.oracle_unit(K[0, h], V[0, h], Q[0, i, h * G:(h + 1) * G], L, t, C, k,
                                        w, "bf16", 1e6)
            cur = H.check_selection(levels, H.to64(Q[0, i, h * G:(h + 1) * G]), t, C, k, 1e6, res,
                                    sel[i, h].cpu().numpy(), cnt[i, h].cpu().numpy(),
                                    tree.n_sel_levels)
            assert H.max_abs(H.to64(O[0, i, h * G:(h + 1) * G]), cur.out) <= 2e-2


def test_host_errors_are_returned_not_launched(R):
    cfg = R.Config(head_dim=64, n_q_heads=2, n_kv_heads=1, C=4, k=2, dtype="f32",
                   pooler_w=H.w_for(4))
    tree = R.RecsaTree(cfg, 100, 1)
    tree.recsa_build([90])
    kn = torch.zeros(1, 1, 20, 64, device="cuda")
    with pytest.raises(R.RecsaError) as e:
        tree.recsa_append(kn, kn)
    assert e.value.status == R.RECSA_E_CAPACITY
    with pytest.raises(R.RecsaError) as e:
        tree.recsa_build([101])
    assert e.value.status == R.RECSA_E_CAPACITY
    Q = torch.zeros(1, 5, 2, 64, device="cuda")
    with pytest.raises(R.RecsaError):
        tree.prefill(Q, 88)
    assert tree.recsa_get_status() == R.RECSA_OK


@pytest.mark.parametrize("k,L", [(128, 40000), (64, 30000)])
def test_long_lists_sampled_select(R, k, L):
    """Lists of 1024-2048 entries spread over a cluster's CTAs: the distributed
    histogram, the published boundary-bin candidates and the list-order ranks across
    CTAs; sets must still be exact."""
    run_decode_case(R, config_id=17, B=2, Hkv=2, Hq=8, d=128, C=16, k=k, lengths=[L, L - 777],
                    dtype="bf16", cap=L, n_needles=16)



def test_k512_two_selecting_levels(R):
    """k = 512 (C*k = 8192, the largest list the library takes): L = 140000 selects
    at level 2 (547 nodes) and at level 1 (8192 children), then attends level 0."""
    tree, worst = run_decode_case(R, config_id=19, B=1, Hkv=2, Hq=8, d=128, C=16, k=512,
                                  lengths=[140000], dtype="bf16", cap=140000, n_needles=16)
    assert tree.n_sel_levels >= 2


def test_whole_sequence_chunked_prefill(R):
    """A whole sequence through the public calls, as a model runs it: per chunk, append
    its K/V rows (the tree grows, starting empty), then prefill its query rows.
    Sampled rows of every chunk (first, middle, last) against the oracle, whose rows
    depend only on tokens <= t; the final tree bit for bit."""
    from oracle import recsa_oracle as O_
    C, k, d, Hkv, Hq = 16, 64, 128, 2, 8
    L, n = 9000, 2048
    G = Hq // Hkv
    w = H.w_for(C)
    cfg = R.Config(head_dim=d, n_q_heads=Hq, n_kv_heads=Hkv, C=C, k=k, dtype="bf16", pooler_w=w)
    K, V, Q = H.make_inputs(20, 1, Hkv, Hq, d, L, [L], "bf16", q_rows=L, n_needles=8)
    tree = R.RecsaTree(cfg, L, 1, max_queries=256, k0=torch.zeros_like(K),
                       v0=torch.zeros_like(V))
    levels = [O_.build_tree(H.to64(K[0, h]), H.to64(V[0, h]), C, np.asarray(w, dtype=np.float64),
                            "bf16") for h in range(Hkv)]
    for p0 in range(0, L, n):
        m = min(n, L - p0)
        tree.recsa_append(K[:, :, p0:p0 + m].contiguous(), V[:, :, p0:p0 + m].contiguous())
        O, sel, cnt = tree.prefill(Q[:, p0:p0 + m].contiguous(), p0, with_sel=True)
        torch.cuda.synchronize()
        assert tree.recsa_get_status() == R.RECSA_OK
        assert tree.host_lengths() == [p0 + m]
        for i in sorted({0, m // 2, m - 1}):
            t = p0 + i
            for h in range(Hkv):
                qg = H.to64(Q[0, t, h * G:(h + 1) * G])
                res = O_.select_and_attend(levels[h], qg, t, C, k, base=1e6)
                cur = H.check_selection(levels[h], qg, t, C, k, 1e6, res, sel[i, h].cpu().numpy(),
                                        cnt[i, h].cpu().numpy(), tree.n_sel_levels)
                err = H.max_abs(H.to64(O[0, i, h * G:(h + 1) * G]), cur.out)
                assert err <= H.TOL_OUT["bf16"], f"row {t} head {h}: output max-abs {err}"
    for h in range(Hkv):
        H.compare_tree(tree, levels[h], 0, h, "bf16")

def test_prefill_tensor_core_top_level(R):
    """Prefill on a tree with max_queries >= 128 scores the first scored level with
    one tensor-core product per group of rows.  The product's logits equal
    scale * <R(a_t) q, R(j) K_j> over the stored level (fp64 here) within fp32
    rounding, and sampled rows match the oracle: selections exact except at
    near-ties, outputs within 2e-2."""
    from oracle import recsa_oracle as O
    C, k, d, Hkv, Hq = 16, 64, 128, 2, 8
    L = 40000
    n = 160                       # one product of 128 rows, then one of 32
    pos0 = L - n
    G = Hq // Hkv
    scale = 1.0 / np.sqrt(d)
    w = H.w_for(C)
    cfg = R.Config(head_dim=d, n_q_heads=Hq, n_kv_heads=Hkv, C=C, k=k, dtype="bf16", pooler_w=w)
    K, V, Q = H.make_inputs(18, 1, Hkv, Hq, d, L, [L], "bf16", q_rows=n, n_needles=16)
    small = R.RecsaTree(cfg, L, 1, max_queries=64, k0=K, v0=V)
    assert small.tc_queries == 0
    del small
    tree = R.RecsaTree(cfg, L, 1, max_queries=128, k0=K, v0=V)
    assert tree.tc_queries == 128
    tree.recsa_build([L])
    Out, sel, cnt = tree.prefill(Q, pos0, with_sel=True)
    torch.cuda.synchronize()
    assert tree.recsa_get_status() == R.RECSA_OK

    # 1. the last product's logits (rows 128..159 of the chunk) against fp64
    lt = 2
    assert (pos0 + n - 1) // C ** lt >= k and (pos0 + n - 1) // C ** (lt + 1) < k
    nrows, stride = n - 128, tree.tc_row_stride
    off = tree.tc_logits_offset
    logits = tree.workspace[off: off + 4 * nrows * Hkv * G * stride].view(torch.float32)
    logits = logits.reshape(nrows, Hkv, G, stride).double().cpu().numpy()
    Kl, _ = tree.level_tables(lt)
    worst = 0.0
    for qi in (0, 13, nrows - 1):
        t = pos0 + 128 + qi
        a = t // C ** lt
        for h in range(Hkv):
            qg = H.to64(Q[0, 128 + qi, h * G:(h + 1) * G])
            kr = H.to64(Kl[0, h, :a + 1])
            ref = O.level_logits(qg, kr, a, np.arange(a + 1), scale, 1e6)
            got = logits[qi, h, :, :a + 1]
            bound = 1e-5 * scale * np.outer(np.linalg.norm(qg, axis=1), np.linalg.norm(kr, axis=1))
            err = np.abs(got - ref)
            worst = max(worst, float(np.max(err / bound)))
            assert np.all(err <= bound), f"row {qi} head {h}: logit error {err.max()}"
    print("tensor-core logits: worst error / bound", worst)

    # 2. sampled rows of both products against the oracle
    NL = tree.n_sel_levels
    for h in range(Hkv):
        levels = O.build_tree(H.to64(K[0, h, :L]), H.to64(V[0, h, :L]), C,
                              np.asarray(w, dtype=np.float64), "bf16")
        for i in (0, 64, 127, 128, n - 1):
            t = pos0 + i
            qg = H.to64(Q[0, i, h * G:(h + 1) * G])
            res = O.select_and_attend(levels, qg, t, C, k, base=1e6)
            cur = H.check_selection(levels, qg, t, C, k, 1e6, res, sel[i, h].cpu().numpy(),
                                    cnt[i, h].cpu().numpy(), NL)
            err = H.max_abs(H.to64(Out[0, i, h * G:(h + 1) * G]), cur.out)
            assert err <= H.TOL_OUT["bf16"], f"row {i} head {h}: output max-abs {err}"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_single_appends_without_decode_equal_build(R, dtype):
    """Single-token appends leave the ancestors to the next call: back-to-back
    appends and a status query complete them as a separate launch, a decode inside
    its level-0 launch.  Tables and outputs equal a fresh build bit for bit."""
    C, k, d, Hkv, Hq, B = 16, 8, 64, 2, 4, 2
    L0, cap = 3000, 3100
    w = H.w_for(C)
    cfg = R.Config(head_dim=d, n_q_heads=Hq, n_kv_heads=Hkv, C=C, k=k, dtype=dtype, pooler_w=w)
    K, V, q = H.make_inputs(19, B, Hkv, Hq, d, cap, [cap] * B, dtype)
    q = q[:, 0].contiguous()
    Ka, Va = K.clone(), V.clone()
    Ka[:, :, L0:] = 0
    Va[:, :, L0:] = 0
    inc = R.RecsaTree(cfg, cap, B, k0=Ka, v0=Va)
    inc.recsa_build([L0] * B)

    def tables_equal(n):
        ref = R.RecsaTree(cfg, cap, B, k0=K.clone(), v0=V.clone())
        ref.recsa_build([n] * B)
        for l in range(1, ref.n_levels):
            rows = -(-n // C ** l)
            Ki, Vi = inc.level_tables(l)
            Kr, Vr = ref.level_tables(l)
            assert torch.equal(Ki[:, :, :rows], Kr[:, :, :rows]), f"K level {l} at {n}"
            assert torch.equal(Vi[:, :, :rows], Vr[:, :, :rows]), f"V level {l} at {n}"
        return ref

    n = L0
    for _ in range(5):
        inc.recsa_append(K[:, :, n:n + 1].contiguous(), V[:, :, n:n + 1].contiguous())
        n += 1
    assert inc.recsa_get_status() == R.RECSA_OK        # completes the last append
    tables_equal(n)
    for _ in range(3):
        inc.recsa_append(K[:, :, n:n + 1].contiguous(), V[:, :, n:n + 1].contiguous())
        n += 1
    out = inc.decode(q)[0]                              # completes it in its own launch
    torch.cuda.synchronize()
    ref = tables_equal(n)
    assert torch.equal(out, ref.decode(q)[0])
    assert inc.recsa_get_status() == R.RECSA_OK


def test_bounded_wait_gives_up_and_reports_timeout(R):
    """The device-side timeout path: a wait on an mbarrier that nothing completes
    gives up after its poll limit and records the timeout; the context stays usable
    (a decode afterwards is still correct)."""
    import ctypes
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = R.lib.recsa_probe_bounded_wait(ctypes.c_void_p(st.data_ptr()), None)
    assert rc == R.RECSA_E_TIMEOUT
    assert int(st.item()) == 3
    run_decode_case(R, config_id=21, B=1, Hkv=1, Hq=2, d=64, C=4, k=3, lengths=[300],
                    dtype="f32", cap=300)


def test_query_written_by_the_kernel_just_before_decode(R):
    """The caller's own kernel may write q right before the decode on the same stream
    (a projection or a RoPE kernel).  The decode is launched with programmatic
    dependent launch and stages q only after its dependency wait, so it reads that
    kernel's output: here q is written by a conversion kernel that follows a long
    elementwise kernel, with no library kernel in between, and every output must equal
    the one from a decode whose q was written and synchronised long before."""
    C, k, d, Hkv, Hq, B, L0, steps = 16, 16, 128, 2, 8, 2, 6000, 4
    cfg = R.Config(head_dim=d, n_q_heads=Hq, n_kv_heads=Hkv, C=C, k=k, dtype="bf16",
                   pooler_w=H.w_for(C))
    K, V, q_all = H.make_inputs(51, B, Hkv, Hq, d, L0, [L0] * B, "bf16", q_rows=steps)
    tree = R.RecsaTree(cfg, L0, B, k0=K, v0=V)
    tree.recsa_build([L0] * B)
    ref = []
    for s in range(steps):
        qs = q_all[:, s].contiguous()
        torch.cuda.synchronize()
        ref.append(tree.decode(qs)[0].clone())
    torch.cuda.synchronize()
    big = torch.ones(64 << 20, dtype=torch.float32, device="cuda")   # 256 MB
    src = [q_all[:, s].float().contiguous() for s in range(steps)]
    qbuf = torch.empty_like(q_all[:, 0].contiguous())
    torch.cuda.synchronize()
    for s in range(steps):
        big.mul_(1.0)        # a long kernel, so the next one ends late
        qbuf.copy_(src[s])   # the kernel that writes q, launched right before the decode
        out = tree.decode(qbuf)[0]
        torch.cuda.synchronize()
        assert tree.recsa_get_status() == R.RECSA_OK
        assert torch.equal(out, ref[s]), f"step {s}: the decode read a stale query"
