"""recsa_decode_noalloc: the decode entry point for callers that cannot allocate
device memory where they call it (inside a stream capture in global capture mode,
under a fixed pre-planned memory budget, or in a runtime without a device allocator
for per-call scratch).  Its scratch is a fixed array inside the library.

Checked through the C ABI against recsa_decode on the same buffers, on two calls in
a row with different queries, so that nothing left over from one call leaks into
the next.  Both run the same kernels on the same inputs, so the outputs must be
equal bit for bit (which is inside the tolerance of the other parity tests).  The
device-side status each call writes into the caller's status word is checked too.
This file is collected last on purpose."""
import ctypes

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


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_decode_matches_decode_on_two_calls(R, dtype):
    C, k, d, Hkv, Hq, B = 16, 8, 128, 2, 8, 2
    cap, lengths = 5000, [5000, 3333]
    cfg = R.Config(head_dim=d, n_q_heads=Hq, n_kv_heads=Hkv, C=C, k=k, dtype=dtype,
                   pooler_w=H.w_for(C))
    K, V, Q = H.make_inputs(21, B, Hkv, Hq, d, cap, lengths, dtype, q_rows=2, n_needles=4)
    tree = R.RecsaTree(cfg, cap, B, k0=K, v0=V)
    tree.recsa_build(lengths)
    status = torch.full((1,), 77, dtype=torch.int32, device="cuda")
    for call in range(2):
        q = Q[:, call].contiguous()
        ref = tree.decode(q)[0]
        out = torch.full_like(q, float("nan"))
        status.fill_(77)
        st = R.recsa_decode_noalloc(cfg, cap, K, V, tree.levels, lengths, q, out, status)
        torch.cuda.synchronize()
        assert st == R.RECSA_OK, R.lib.recsa_status_str(st)
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        err = (out.double() - ref.double()).abs().max().item()
        assert err <= H.TOL_OUT[dtype], f"call {call}: max-abs {err}"
        assert torch.equal(out, ref), f"call {call}: not bitwise equal (max-abs {err})"


def test_noalloc_rejects_shapes_beyond_its_scratch(R):
    cfg = R.Config(head_dim=128, n_q_heads=64, n_kv_heads=8, C=32, k=256, dtype="bf16",
                   pooler_w=H.w_for(32))
    fake = torch.empty(256, dtype=torch.uint8, device="cuda")
    q = torch.zeros(64, 64, 128, dtype=torch.bfloat16, device="cuda")
    st = R.recsa_decode_noalloc(cfg, 1 << 24, fake.view(torch.bfloat16), fake.view(torch.bfloat16),
                                fake, [0] * 64, q, q)
    assert st == R.RECSA_E_CAPACITY
