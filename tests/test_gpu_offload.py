"""Level 0 in pinned host memory ("Efficiency Results": decode at 1M/2M tokens with
the KV cache offloaded; "Practical Implications": the levels above 0 stay on the GPU):
decode through the C ABI gathers each query's level-0 list into a device staging
buffer and attends it there.  Every kernel computes the same things on the same
values as with level 0 in device memory, so outputs, selections and list counts must
be equal bit for bit; a 2M-token case is also checked against the fp64 oracle.
"""
import numpy as np
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


def pinned_copy(x):
    h = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    h.copy_(x)
    return h


@pytest.mark.parametrize("dtype,d,C,k,G", [("bf16", 128, 16, 16, 4), ("f32", 64, 4, 8, 2)])
def test_offloaded_decode_equals_device_decode(R, dtype, d, C, k, G):
    Hkv, B = 2, 2
    Hq = G * Hkv
    lengths = [5000, 3333]
    steps = 3
    cap = 5000 + steps
    cfg = R.Config(head_dim=d, n_q_heads=Hq, n_kv_heads=Hkv, C=C, k=k, dtype=dtype,
                   pooler_w=H.w_for(C))
    K, V, q = H.make_inputs(41, B, Hkv, Hq, d, cap, [cap] * B, dtype, n_needles=4, q_rows=steps + 1)
    Kd, Vd = K.clone(), V.clone()
    for b in range(B):
        Kd[b, :, lengths[b]:] = 0
        Vd[b, :, lengths[b]:] = 0
    dev = R.RecsaTree(cfg, cap, B, k0=Kd.clone(), v0=Vd.clone())
    host = R.RecsaTree(cfg, cap, B, k0=pinned_copy(Kd.cpu()), v0=pinned_copy(Vd.cpu()))
    with pytest.raises(R.RecsaError) as e:          # no staging buffer yet
        host.decode(q[:, 0].contiguous())
    assert e.value.status == R.RECSA_E_UNSUPPORTED
    host.recsa_tree_set_offload_staging()
    for tr in (dev, host):
        tr.recsa_build(lengths)
    for s in range(steps + 1):
        qs = q[:, s].contiguous()
        od, sd, cd = dev.decode(qs, with_sel=True)
        oh, sh, ch = host.decode(qs, with_sel=True)
        torch.cuda.synchronize()
        assert dev.recsa_get_status() == R.RECSA_OK and host.recsa_get_status() == R.RECSA_OK
        assert torch.equal(od, oh), f"step {s}: outputs differ"
        assert torch.equal(sd, sh) and torch.equal(cd, ch), f"step {s}: selections differ"
        if s < steps:   # one appended token per sequence (the ancestors re-pooled via host memory)
            kn = K[:, :, 5000 + s:5000 + s + 1].contiguous()
            vn = V[:, :, 5000 + s:5000 + s + 1].contiguous()
            dev.recsa_append(kn, vn)
            host.recsa_append(kn, vn)
    for lvl in range(1, dev.n_levels):   # the rows each sequence's tree holds
        for b in range(B):
            n = -(-(lengths[b] + steps) // C ** lvl)
            if -(-(lengths[b] + steps) // C ** (lvl - 1)) <= 1:
                continue   # the level below is already this sequence's root
            for i in (0, 1):
                assert torch.equal(dev.level_tables(lvl)[i][b, :, :n],
                                   host.level_tables(lvl)[i][b, :, :n]), f"level {lvl} seq {b}"
    with pytest.raises(R.RecsaError) as e:
        host.prefill(q[:, :2].contiguous(), 100)
    assert e.value.status == R.RECSA_E_UNSUPPORTED
    with pytest.raises(R.RecsaError) as e:
        dev.recsa_tree_set_offload_staging()
    assert e.value.status == R.RECSA_E_UNSUPPORTED


def test_offloaded_short_sequences_level0_only(R):
    """Sequences shorter than C*k: no level is scored and the level-0 list is [0..t]."""
    C, k, d, Hkv, Hq, B = 16, 16, 128, 1, 4, 2
    lengths = [100, 1]
    cfg = R.Config(head_dim=d, n_q_heads=Hq, n_kv_heads=Hkv, C=C, k=k, dtype="bf16",
                   pooler_w=H.w_for(C))
    K, V, q = H.make_inputs(42, B, Hkv, Hq, d, 128, lengths, "bf16")
    q = q[:, 0].contiguous()
    dev = R.RecsaTree(cfg, 128, B, k0=K.clone(), v0=V.clone())
    host = R.RecsaTree(cfg, 128, B, k0=pinned_copy(K.cpu()), v0=pinned_copy(V.cpu()))
    host.recsa_tree_set_offload_staging()
    for tr in (dev, host):
        tr.recsa_build(lengths)
    od = dev.decode(q)[0]
    oh = host.decode(q)[0]
    torch.cuda.synchronize()
    assert host.recsa_get_status() == R.RECSA_OK
    assert torch.equal(od, oh)


def test_offloaded_decode_2m_against_oracle(R):
    """2M tokens, one KV head with four query heads, level 0 in host memory (1 GB
    pinned): build, append one token, decode; selections and output against the
    oracle, and against the same decode with level 0 in device memory."""
    Hkv, Hq, d, C, k = 1, 4, 128, 16, 256
    L = 2097152
    cap = L + 16
    w = H.w_for(C)
    cfg = R.Config(head_dim=d, n_q_heads=Hq, n_kv_heads=Hkv, C=C, k=k, dtype="bf16",
                   rope_base=1e6, pooler_w=w)
    Ks, Vs = I.kv_slice(6, 0, 0, L + 1, d, "bf16")
    q = I.q_rows(6, 0, 1, Hq, d, "bf16")[0:1].cuda().contiguous()
    Kh = torch.zeros(1, Hkv, cap, d, dtype=torch.bfloat16, pin_memory=True)
    Vh = torch.zeros(1, Hkv, cap, d, dtype=torch.bfloat16, pin_memory=True)
    Kh[0, 0, :L] = Ks[:L]
    Vh[0, 0, :L] = Vs[:L]
    host = R.RecsaTree(cfg, cap, 1, k0=Kh, v0=Vh)
    host.recsa_tree_set_offload_staging()
    host.recsa_build([L])
    kn = Ks[L:L + 1].reshape(1, 1, 1, d).cuda().contiguous()
    vn = Vs[L:L + 1].reshape(1, 1, 1, d).cuda().contiguous()
    host.recsa_append(kn, vn)
    out, sel, cnt = host.decode(q, with_sel=True)
    torch.cuda.synchronize()
    assert host.recsa_get_status() == R.RECSA_OK
    Kd = Kh.cuda()
    Vd = Vh.cuda()
    dev = R.RecsaTree(cfg, cap, 1, k0=Kd, v0=Vd)
    dev.recsa_build([L + 1])
    od, sd, cd = dev.decode(q, with_sel=True)
    torch.cuda.synchronize()
    assert torch.equal(out, od) and torch.equal(sel, sd) and torch.equal(cnt, cd)
    del Kd, Vd, dev
    levels, res = H.oracle_unit(Ks, Vs, q[0], L + 1, L, C, k, w, "bf16", 1e6)
    H.compare_tree(host, levels, 0, 0, "bf16")
    cur = H.check_selection(levels, H.to64(q[0]), L, C, k, 1e6, res, sel[0, 0].cpu().numpy(),
                            cnt[0, 0].cpu().numpy(), host.n_sel_levels)
    err = H.max_abs(H.to64(out[0]), cur.out)
    assert err <= H.TOL_OUT["bf16"], f"output max-abs {err}"
