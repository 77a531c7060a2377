"""The C-ABI library loads on a host without a GPU, exports every symbol the
header declares, and rejects bad arguments on the host (no compute calls)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def R():
    from long_context_recsa_b200 import build
    build.build()
    import long_context_recsa_b200.recsa as R
    return R


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "recsa.h")).read()
    return sorted(set(re.findall(r"RECSA_API[^;(]*?\b(recsa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("recsa_build", "recsa_append", "recsa_decode", "recsa_prefill_chunk",
                 "recsa_query_sizes", "recsa_tree_init", "recsa_get_status", "recsa_tree_free"):
        assert name in syms


def test_library_exports_every_declared_symbol(R):
    lib = ctypes.CDLL(R.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_query_sizes_and_host_validation(R):
    cfg = R.Config(head_dim=128, n_q_heads=32, n_kv_heads=8, C=16, k=256, dtype="bf16")
    lb, wb, nl = R.recsa_query_sizes(cfg, 524288, 4, 4)
    # levels >= 1 hold about 1/15 of level 0 (K and V, bf16, d = 128)
    level0 = 4 * 8 * 524288 * 128 * 2 * 2
    assert 0.06 < lb / level0 < 0.07
    assert nl == 6                     # 524288 -> 32768 -> 2048 -> 128 -> 8 -> 1
    bad = [
        dict(head_dim=96), dict(n_q_heads=12, n_kv_heads=8), dict(C=1), dict(C=64),
        dict(k=0), dict(k=1024), dict(C=32, k=512), dict(rope_base=1.0), dict(n_q_heads=48),
    ]
    for kw in bad:
        c = R.Config(**{**cfg.__dict__, **kw})
        with pytest.raises(R.RecsaError) as e:
            R.recsa_query_sizes(c, 1024, 1, 1)
        assert e.value.status in (R.RECSA_E_INVAL, R.RECSA_E_UNSUPPORTED), kw
    for cap, B, Q in [(0, 1, 1), (100, 0, 1), (100, 65, 65), (100, 4, 2)]:
        with pytest.raises(R.RecsaError):
            R.recsa_query_sizes(cfg, cap, B, Q)


def test_tree_init_rejects_bad_pointers_before_any_cuda_call(R):
    lib = R.lib
    cfg = R.Config(head_dim=64, n_q_heads=2, n_kv_heads=1, C=4, k=2, dtype="f32").to_c()
    lb, wb, _ = R.recsa_query_sizes(R.Config(head_dim=64, n_q_heads=2, n_kv_heads=1, C=4, k=2,
                                             dtype="f32"), 100, 1, 1)
    strides = (ctypes.c_int64 * 3)(100 * 64, 100 * 64, 64)
    h = ctypes.c_void_p()
    fake = ctypes.c_void_p(1 << 20)        # never dereferenced: validation fails first
    mis = ctypes.c_void_p((1 << 20) + 8)
    cases = [
        (None, fake, strides, fake, fake),            # NULL k0
        (fake, fake, None, fake, fake),               # NULL strides
        (mis, fake, strides, fake, fake),             # misaligned k0
        (fake, fake, strides, mis, fake),             # misaligned level buffer
    ]
    for k0, v0, st, lv, ws in cases:
        r = lib.recsa_tree_init(ctypes.byref(cfg), 100, 1, 1, k0, v0, st, lv, lb, ws, wb, None,
                                ctypes.byref(h))
        assert r == R.RECSA_E_INVAL
        assert not h.value
    bad_stride = (ctypes.c_int64 * 3)(100 * 64, 100 * 64, 60)
    r = lib.recsa_tree_init(ctypes.byref(cfg), 100, 1, 1, fake, fake, bad_stride, fake, lb, fake,
                            wb, None, ctypes.byref(h))
    assert r == R.RECSA_E_INVAL
    r = lib.recsa_tree_init(ctypes.byref(cfg), 100, 1, 1, fake, fake, strides, fake, lb - 256,
                            fake, wb, None, ctypes.byref(h))
    assert r == R.RECSA_E_CAPACITY
    for fn, args in [("recsa_build", (None, None, None)), ("recsa_decode", (None,) * 6),
                     ("recsa_append", (None, None, None, 1, None)),
                     ("recsa_prefill_chunk", (None, None, 0, 1, None, None, None, None)),
                     ("recsa_get_status", (None, None)), ("recsa_tree_free", (None,))]:
        assert getattr(lib, fn)(*args) == R.RECSA_E_INVAL, fn
    assert lib.recsa_status_str(3) == b"capacity exceeded or buffer too small"
