"""recsa_append_decode: one launch that appends a token to every sequence and decodes
at its position ("Practical Implications": one token per decode step), against
recsa_append followed by recsa_decode on a second tree.  Outputs, selections and
counts must be equal bit for bit at every step, and the trees equal afterwards."""
import pytest
import torch

from long_context_recsa_b200 import inputs as I
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


def two_trees(R, dtype, d, C, k, G, lengths, steps, seed):
    Hkv, B = 2, len(lengths)
    Hq = G * Hkv
    cap = max(lengths) + steps + 1
    cfg = R.Config(head_dim=d, n_q_heads=Hq, n_kv_heads=Hkv, C=C, k=k, dtype=dtype,
                   pooler_w=H.w_for(C))
    K, V, q = H.make_inputs(seed, B, Hkv, Hq, d, cap, [cap] * B, dtype, q_rows=steps)
    Kc, Vc = K.clone(), V.clone()
    for b in range(B):
        Kc[b, :, lengths[b]:] = 0
        Vc[b, :, lengths[b]:] = 0
    a = R.RecsaTree(cfg, cap, B, k0=Kc.clone(), v0=Vc.clone())
    f = R.RecsaTree(cfg, cap, B, k0=Kc.clone(), v0=Vc.clone())
    for tr in (a, f):
        tr.recsa_build(lengths)
    return a, f, K, V, q, cfg


def token(X, lengths, s):
    """The token each sequence appends at step s: its row at position lengths[b] + s."""
    return torch.stack([X[b, :, lengths[b] + s:lengths[b] + s + 1] for b in range(len(lengths))]).contiguous()


def compare_trees(a, f, lengths, C):
    B = len(lengths)
    for b in range(B):
        L = lengths[b]
        assert torch.equal(a.k0[b, :, :L], f.k0[b, :, :L]) and torch.equal(a.v0[b, :, :L], f.v0[b, :, :L])
        for lvl in range(1, a.n_levels):
            if -(-L // C ** (lvl - 1)) <= 1:
                break
            n = -(-L // C ** lvl)
            for i in (0, 1):
                assert torch.equal(a.level_tables(lvl)[i][b, :, :n], f.level_tables(lvl)[i][b, :, :n]), \
                    f"level {lvl} seq {b}"


@pytest.mark.parametrize("dtype,d,C,k,G,lengths", [
    ("bf16", 128, 16, 16, 4, [5000, 3327]),
    ("f32", 64, 4, 8, 2, [700, 255]),
    ("bf16", 64, 8, 8, 1, [1, 0]),
])
def test_fused_equals_append_then_decode(R, dtype, d, C, k, G, lengths):
    steps = 20
    a, f, K, V, q, cfg = two_trees(R, dtype, d, C, k, G, lengths, steps, 61)
    for s in range(steps):
        kn, vn, qs = token(K, lengths, s), token(V, lengths, s), q[:, s].contiguous()
        a.recsa_append(kn, vn)
        oa, sa, ca = a.decode(qs, with_sel=True)
        of = torch.empty_like(qs)
        sf = torch.empty_like(sa)
        cf = torch.empty_like(ca)
        f.recsa_append_decode(kn, vn, qs, of, sf, cf)
        torch.cuda.synchronize()
        assert a.recsa_get_status() == R.RECSA_OK and f.recsa_get_status() == R.RECSA_OK
        assert torch.equal(oa, of), f"step {s}: outputs differ"
        assert torch.equal(ca, cf), f"step {s}: counts differ"
        if a.n_sel_levels > 0:   # (no selecting level: the buffer is never written)
            assert torch.equal(sa, sf), f"step {s}: selections differ"
    compare_trees(a, f, [L + steps for L in lengths], C)
    # a plain decode on both trees afterwards: the lengths advanced alike
    qs = q[:, 0].contiguous()
    assert torch.equal(a.decode(qs)[0], f.decode(qs)[0])


def test_fused_after_a_plain_append(R):
    """A plain append leaves its ancestor walk pending; the fused call runs it first."""
    lengths, steps = [4097, 2049], 4
    a, f, K, V, q, cfg = two_trees(R, "bf16", 128, 16, 16, 4, lengths, steps, 62)
    for s in range(steps):
        kn, vn, qs = token(K, lengths, s), token(V, lengths, s), q[:, s].contiguous()
        a.recsa_append(kn, vn)
        oa = a.decode(qs)[0]
        if s % 2 == 0:
            f.recsa_append(kn, vn)
            of = f.decode(qs)[0]
        else:
            of = torch.empty_like(qs)
            f.recsa_append_decode(kn, vn, qs, of)
        torch.cuda.synchronize()
        assert torch.equal(oa, of), f"step {s}"
    compare_trees(a, f, [L + steps for L in lengths], 16)


def test_fused_rejections(R):
    cfg = R.Config(head_dim=64, n_q_heads=2, n_kv_heads=1, C=4, k=4, dtype="f32", pooler_w=H.w_for(4))
    K, V, q = H.make_inputs(63, 1, 1, 2, 64, 40, [40], "f32")
    tr = R.RecsaTree(cfg, 40, 1, k0=K, v0=V)
    tr.recsa_build([40])
    kn = torch.zeros(1, 1, 1, 64, device="cuda")
    out = torch.empty(1, 2, 64, device="cuda")
    with pytest.raises(R.RecsaError) as e:   # the sequence is at capacity
        tr.recsa_append_decode(kn, kn.clone(), q[:, 0].contiguous(), out)
    assert e.value.status == R.RECSA_E_CAPACITY
