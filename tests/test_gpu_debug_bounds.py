"""The bounds-checked build (librecsa_bounds.so, -DRECSA_DEBUG_BOUNDS): every gather row
of the select/attend pass, every selection rank it stores, every ancestor the append
walk re-pools and every token the level-0 gather copies is range-checked on the device,
and a failed check is recorded in the status word.  A set of small cases through that
build must finish with status OK and give the same results, bit for bit, as the
normal build: decode over ragged batches (both staging paths), appends, prefill rows
(per row and with the tensor-core top level), level 0 in host memory and the gated
pooler."""
import importlib.util
import os
import sys

import pytest
import torch

from tests import parity_helpers as H

pytestmark = pytest.mark.gpu


def _binding(path, name):
    """A separate instance of the ctypes binding bound to the library at `path`."""
    os.environ["RECSA_LIBRARY"] = path
    try:
        here = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "long_context_recsa_b200", "recsa.py")
        spec = importlib.util.spec_from_file_location(name, here)
        mod = importlib.util.module_from_spec(spec)
        sys.modules[name] = mod
        spec.loader.exec_module(mod)
        return mod
    finally:
        del os.environ["RECSA_LIBRARY"]


@pytest.fixture(scope="module")
def libs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_recsa_b200 import build
    build.build()
    bounds = build.build(debug_bounds=True)
    import long_context_recsa_b200.recsa as R
    Rb = _binding(bounds, "recsa_bounds_binding")
    assert Rb.lib._name.endswith("librecsa_bounds.so")
    return R, Rb


def _run(R, cfg, K, V, q, lengths, cap, B, appends=None, prefill=None, host=False, gated=None):
    tr = R.RecsaTree(cfg, cap, B, max_queries=max(B, prefill[2] if prefill else B),
                     k0=K.clone() if not host else K.cpu().pin_memory(),
                     v0=V.clone() if not host else V.cpu().pin_memory())
    if host:
        tr.recsa_tree_set_offload_staging()
    if gated is not None:
        tr.recsa_tree_set_gated_pooler(gated)
    tr.recsa_build(lengths)
    outs = []
    for a in appends or []:
        tr.recsa_append(*a)
        outs.append(tr.decode(q, with_sel=True))
    outs.append(tr.decode(q, with_sel=True))
    if prefill is not None:
        Q, pos0, _ = prefill
        outs.append(tr.prefill(Q, pos0, with_sel=True))
    torch.cuda.synchronize()
    st = tr.recsa_get_status()
    return outs, st


@pytest.mark.parametrize("dtype,d,C,k,G", [("bf16", 128, 16, 8, 4), ("f32", 64, 4, 3, 2),
                                          ("bf16", 64, 16, 16, 8)])
def test_bounds_build_decode_append_prefill(libs, dtype, d, C, k, G):
    R, Rb = libs
    Hkv, B = 2, 3
    lengths = [1500, 777, 17]
    cap = 1700
    K, V, Qr = H.make_inputs(51, B, Hkv, G * Hkv, d, cap, [cap] * B, dtype, n_needles=3, q_rows=140)
    for b in range(B):
        K[b, :, lengths[b]:] = 0
        V[b, :, lengths[b]:] = 0
    q = Qr[:, 0].contiguous()
    Kn = torch.randn(B, Hkv, 1, d, device="cuda").to(K.dtype)
    appends = [(Kn, Kn.clone()), (Kn.clone(), Kn.clone())]
    Q = Qr[:1, :130].contiguous()
    results = []
    for mod in (R, Rb):
        cfg = mod.Config(head_dim=d, n_q_heads=G * Hkv, n_kv_heads=Hkv, C=C, k=k, dtype=dtype,
                         pooler_w=H.w_for(C))
        outs, st = _run(mod, cfg, K, V, q, lengths, cap, B, appends=appends)
        assert st == mod.RECSA_OK
        # a single sequence for the prefill rows (tensor-core top level with 128 rows)
        cfg1 = mod.Config(head_dim=d, n_q_heads=G * Hkv, n_kv_heads=Hkv, C=C, k=k, dtype=dtype,
                          pooler_w=H.w_for(C))
        pouts, pst = _run(mod, cfg1, K[:1], V[:1], q[:1], [1500], cap, 1,
                          prefill=(Q, 1500 - 130, 128))
        assert pst == mod.RECSA_OK
        results.append(outs + pouts)
    for a, b in zip(*results):
        for x, y in zip(a, b):
            assert torch.equal(x, y)


def test_bounds_build_offload_and_gated(libs):
    R, Rb = libs
    C, k, d, Hkv, G, B = 16, 16, 128, 2, 4, 2
    lengths = [5000, 999]
    cap = 5000
    K, V, q = H.make_inputs(52, B, Hkv, G * Hkv, d, cap, lengths, "bf16")
    q = q[:, 0].contiguous()
    from tests.test_gpu_gated import gated_params
    _, Pd = gated_params(d, 32)
    results = []
    for mod in (R, Rb):
        cfg = mod.Config(head_dim=d, n_q_heads=G * Hkv, n_kv_heads=Hkv, C=C, k=k, dtype="bf16",
                         pooler_w=H.w_for(C))
        o1, s1 = _run(mod, cfg, K, V, q, lengths, cap, B, host=True)
        o2, s2 = _run(mod, cfg, K, V, q, lengths, cap, B, gated=Pd)
        assert s1 == mod.RECSA_OK and s2 == mod.RECSA_OK
        results.append(o1 + o2)
    for a, b in zip(*results):
        for x, y in zip(a, b):
            assert torch.equal(x, y)
