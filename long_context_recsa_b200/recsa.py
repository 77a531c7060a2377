"""Thin Python binding of librecsa.so (the RecSA C ABI declared in include/recsa.h).

Argument marshalling only: every step of build, append, selection and attention
runs in the library's CUDA kernels.  PyTorch supplies device memory and streams.
There is no fallback: if the library is missing, importing this module fails.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librecsa.so")

RECSA_OK, RECSA_E_INVAL, RECSA_E_UNSUPPORTED, RECSA_E_CAPACITY = 0, 1, 2, 3
RECSA_E_CUDA, RECSA_E_TIMEOUT, RECSA_E_DEVICE = 4, 5, 6
RECSA_F32, RECSA_BF16 = 0, 1
MAX_C = 32

_DTYPES = {"f32": (RECSA_F32, torch.float32), "bf16": (RECSA_BF16, torch.bfloat16)}


class RecsaConfigC(ctypes.Structure):
    _fields_ = [
        ("head_dim", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("C", ctypes.c_int32),
        ("k", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("rope_base", ctypes.c_double),
        ("scale", ctypes.c_float),
        ("pooler_w", ctypes.c_float * MAX_C),
    ]


class RecsaGatedPoolerC(ctypes.Structure):
    _fields_ = [
        ("hidden", ctypes.c_int32),
        ("tau", ctypes.c_double),
        ("g", ctypes.c_double),
        ("rho", ctypes.c_double),
        ("w", ctypes.c_void_p),
        ("W1t", ctypes.c_void_p),
        ("b1", ctypes.c_void_p),
        ("W2t", ctypes.c_void_p),
    ]


class RecsaTreeInfoC(ctypes.Structure):
    _fields_ = [
        ("n_levels", ctypes.c_int32),
        ("n_sel_levels", ctypes.c_int32),
        ("splits", ctypes.c_int32),
        ("splits0", ctypes.c_int32),
        ("capacity", ctypes.c_int64),
        ("batch", ctypes.c_int32),
        ("max_queries", ctypes.c_int32),
        ("tc_queries", ctypes.c_int32),
        ("tc_row_stride", ctypes.c_int32),
        ("tc_logits_offset", ctypes.c_int64),
    ]


def _load():
    # RECSA_LIBRARY selects another build of this library (the bounds-checked
    # librecsa_bounds.so in its tests); there is no fallback when it is missing
    path = os.environ.get("RECSA_LIBRARY", LIB_PATH)
    if not os.path.exists(path):
        raise ImportError(f"{path} not built; run python -m long_context_recsa_b200.build")
    lib = ctypes.CDLL(path)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "recsa_query_sizes": [ctypes.POINTER(RecsaConfigC), I64, I32, I32, ctypes.POINTER(SZ),
                              ctypes.POINTER(SZ), ctypes.POINTER(I32)],
        "recsa_tree_init": [ctypes.POINTER(RecsaConfigC), I64, I32, I32, P, P, ctypes.POINTER(I64),
                            P, SZ, P, SZ, P, ctypes.POINTER(P)],
        "recsa_build": [P, ctypes.POINTER(I64), P],
        "recsa_append": [P, P, P, I32, P],
        "recsa_decode": [P, P, P, P, P, P],
        "recsa_append_decode": [P, P, P, P, P, P, P, P],
        "recsa_prefill_chunk": [P, P, I64, I32, P, P, P, P],
        "recsa_get_status": [P, P],
        "recsa_tree_info": [P, ctypes.POINTER(RecsaTreeInfoC)],
        "recsa_level_info": [P, I32, ctypes.POINTER(I64), ctypes.POINTER(I64), ctypes.POINTER(I64)],
        "recsa_host_lengths": [P, ctypes.POINTER(I64)],
        "recsa_set_profile_events": [P, I32, P, P],
        "recsa_decode_noalloc": [ctypes.POINTER(RecsaConfigC), I64, I32, P, P, ctypes.POINTER(I64),
                                 P, SZ, ctypes.POINTER(I64), P, P, P, P],
        "recsa_probe_bounded_wait": [P, P],
        "recsa_tree_set_gated_pooler": [P, ctypes.POINTER(RecsaGatedPoolerC)],
        "recsa_offload_staging_bytes": [ctypes.POINTER(RecsaConfigC), I32, ctypes.POINTER(SZ)],
        "recsa_tree_set_offload_staging": [P, P, SZ],
        "recsa_tree_free": [P],
        "recsa_status_str": [I32],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name == "recsa_status_str" else ctypes.c_int
    return lib


lib = _load()


class RecsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.recsa_status_str(status).decode()} ({status})")


def _check(status: int, where: str):
    if status != RECSA_OK:
        raise RecsaError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


@dataclass
class Config:
    head_dim: int = 128
    n_q_heads: int = 32
    n_kv_heads: int = 8
    C: int = 16
    k: int = 256
    dtype: str = "bf16"
    rope_base: float = 1e6
    scale: float = 0.0
    pooler_w: list = field(default_factory=lambda: [0.0] * 16)

    def to_c(self) -> RecsaConfigC:
        c = RecsaConfigC()
        c.head_dim, c.n_q_heads, c.n_kv_heads = self.head_dim, self.n_q_heads, self.n_kv_heads
        c.C, c.k, c.dtype = self.C, self.k, _DTYPES[self.dtype][0]
        c.rope_base, c.scale = self.rope_base, self.scale
        w = [float(x) for x in self.pooler_w]
        for i in range(MAX_C):
            c.pooler_w[i] = w[i] if i < len(w) else 0.0
        return c

    @property
    def torch_dtype(self):
        return _DTYPES[self.dtype][1]

    @property
    def G(self):
        return self.n_q_heads // self.n_kv_heads


def recsa_query_sizes(cfg: Config, capacity: int, batch: int, max_queries: int):
    lb, wb, nl = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_int32()
    c = cfg.to_c()
    _check(lib.recsa_query_sizes(ctypes.byref(c), capacity, batch, max_queries, ctypes.byref(lb),
                                 ctypes.byref(wb), ctypes.byref(nl)), "recsa_query_sizes")
    return lb.value, wb.value, nl.value


def recsa_decode_noalloc(cfg: Config, capacity: int, k0: torch.Tensor, v0: torch.Tensor,
                         levels: torch.Tensor, lengths, q: torch.Tensor, out: torch.Tensor,
                         status_out: torch.Tensor | None = None, stream=None) -> int:
    """Decode with the library's fixed device scratch instead of a caller workspace
    (for callers that cannot allocate device memory at the call site).  Returns the
    status code of the host-side checks; the buffers are the caller's (k0, v0 and
    levels as built for a tree of this capacity and batch).  status_out: optional
    one-element 32-bit device tensor that receives the call's device-side status
    (0 when nothing went wrong)."""
    c = cfg.to_c()
    batch = q.shape[0]
    lens = (ctypes.c_int64 * batch)(*[int(x) for x in lengths])
    strides = (ctypes.c_int64 * 3)(*k0.stride()[:3])
    return lib.recsa_decode_noalloc(ctypes.byref(c), capacity, batch, _ptr(k0), _ptr(v0), strides,
                                    _ptr(levels), levels.numel(), lens, _ptr(q), _ptr(out),
                                    _ptr(status_out), _stream(stream))


class RecsaTree:
    """A tree bound to torch-allocated device buffers.

    k0, v0: level-0 cache [batch][Hkv][capacity][d] (allocated here unless given).
    """

    def __init__(self, cfg: Config, capacity: int, batch: int, max_queries: int | None = None,
                 k0: torch.Tensor | None = None, v0: torch.Tensor | None = None,
                 device="cuda", stream=None):
        self.cfg = cfg
        self.capacity, self.batch = capacity, batch
        self.max_queries = max_queries or batch
        dt = cfg.torch_dtype
        if k0 is None:
            k0 = torch.empty(batch, cfg.n_kv_heads, capacity, cfg.head_dim, dtype=dt, device=device)
        if v0 is None:
            v0 = torch.empty_like(k0)
        assert k0.dtype == dt and v0.dtype == dt and k0.stride() == v0.stride()
        self.k0, self.v0 = k0, v0
        lb, wb, self.n_levels = recsa_query_sizes(cfg, capacity, batch, self.max_queries)
        self.levels = torch.empty(lb, dtype=torch.uint8, device=device)
        self.workspace = torch.empty(wb, dtype=torch.uint8, device=device)
        strides = (ctypes.c_int64 * 3)(*k0.stride()[:3])
        c = cfg.to_c()
        h = ctypes.c_void_p()
        _check(lib.recsa_tree_init(ctypes.byref(c), capacity, batch, self.max_queries, _ptr(k0),
                                   _ptr(v0), strides, _ptr(self.levels), lb, _ptr(self.workspace),
                                   wb, _stream(stream), ctypes.byref(h)), "recsa_tree_init")
        self.handle = h
        info = RecsaTreeInfoC()
        _check(lib.recsa_tree_info(h, ctypes.byref(info)), "recsa_tree_info")
        self.n_sel_levels = info.n_sel_levels
        self.splits, self.splits0 = info.splits, info.splits0
        self.tc_queries, self.tc_row_stride = info.tc_queries, info.tc_row_stride
        self.tc_logits_offset = info.tc_logits_offset

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            lib.recsa_tree_free(h)
            self.handle = None

    # --- the C-ABI calls -------------------------------------------------------
    def recsa_build(self, lengths, stream=None):
        arr = (ctypes.c_int64 * self.batch)(*[int(x) for x in lengths])
        _check(lib.recsa_build(self.handle, arr, _stream(stream)), "recsa_build")

    def recsa_append(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None):
        n = k_new.shape[2]
        assert k_new.is_contiguous() and v_new.is_contiguous() and k_new.shape == v_new.shape
        _check(lib.recsa_append(self.handle, _ptr(k_new), _ptr(v_new), n, _stream(stream)),
               "recsa_append")

    def recsa_append_decode(self, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor,
                            out: torch.Tensor, sel_out=None, counts_out=None, stream=None):
        assert k_new.is_contiguous() and v_new.is_contiguous() and k_new.shape == v_new.shape
        assert k_new.shape[2] == 1 and q.is_contiguous() and out.is_contiguous()
        _check(lib.recsa_append_decode(self.handle, _ptr(k_new), _ptr(v_new), _ptr(q), _ptr(out),
                                       _ptr(sel_out), _ptr(counts_out), _stream(stream)),
               "recsa_append_decode")

    def recsa_decode(self, q: torch.Tensor, out: torch.Tensor, sel_out=None, counts_out=None,
                     stream=None):
        assert q.is_contiguous() and out.is_contiguous()
        _check(lib.recsa_decode(self.handle, _ptr(q), _ptr(out), _ptr(sel_out), _ptr(counts_out),
                                _stream(stream)), "recsa_decode")

    def recsa_prefill_chunk(self, Q: torch.Tensor, pos0: int, O: torch.Tensor, sel_out=None,
                            counts_out=None, stream=None):
        assert Q.is_contiguous() and O.is_contiguous()
        n = Q.shape[1]
        _check(lib.recsa_prefill_chunk(self.handle, _ptr(Q), pos0, n, _ptr(O), _ptr(sel_out),
                                       _ptr(counts_out), _stream(stream)), "recsa_prefill_chunk")

    def recsa_tree_set_gated_pooler(self, params: dict | None):
        """Switch the tree's key pooler to Eq.5 (None: back to the stand-in).  params:
        hidden, tau, g, rho and fp64 device tensors w [d], W1t [2d][h], b1 [h],
        W2t [h][d]; they must outlive the tree's use of them (kept referenced here)."""
        if params is None:
            self._gated = None
            _check(lib.recsa_tree_set_gated_pooler(self.handle, None), "recsa_tree_set_gated_pooler")
            return
        for name in ("w", "W1t", "b1", "W2t"):
            t = params[name]
            assert t.dtype == torch.float64 and t.is_cuda and t.is_contiguous(), name
        p = RecsaGatedPoolerC()
        p.hidden, p.tau, p.g, p.rho = int(params["hidden"]), float(params["tau"]), \
            float(params["g"]), float(params["rho"])
        p.w, p.W1t = params["w"].data_ptr(), params["W1t"].data_ptr()
        p.b1, p.W2t = params["b1"].data_ptr(), params["W2t"].data_ptr()
        self._gated = params
        _check(lib.recsa_tree_set_gated_pooler(self.handle, ctypes.byref(p)),
               "recsa_tree_set_gated_pooler")

    def recsa_tree_set_offload_staging(self, staging: torch.Tensor | None = None):
        """Give a tree whose level 0 is in pinned host memory its device staging
        buffer (allocated here when not given; kept referenced)."""
        if staging is None:
            nb = ctypes.c_size_t()
            c = self.cfg.to_c()
            _check(lib.recsa_offload_staging_bytes(ctypes.byref(c), self.batch, ctypes.byref(nb)),
                   "recsa_offload_staging_bytes")
            staging = torch.empty(nb.value, dtype=torch.uint8, device="cuda")
        self._staging = staging
        _check(lib.recsa_tree_set_offload_staging(self.handle, _ptr(staging), staging.numel()),
               "recsa_tree_set_offload_staging")

    def recsa_get_status(self, stream=None) -> int:
        return lib.recsa_get_status(self.handle, _stream(stream))

    def recsa_set_profile_events(self, which: int, start=None, stop=None):
        """Record torch.cuda.Event start/stop around one kernel (see the header)."""
        s = ctypes.c_void_p(start.cuda_event) if start is not None else None
        e = ctypes.c_void_p(stop.cuda_event) if stop is not None else None
        _check(lib.recsa_set_profile_events(self.handle, which, s, e), "recsa_set_profile_events")

    def host_lengths(self):
        arr = (ctypes.c_int64 * self.batch)()
        _check(lib.recsa_host_lengths(self.handle, arr), "recsa_host_lengths")
        return list(arr)

    # --- conveniences (allocation + views only) -------------------------------
    def decode(self, q: torch.Tensor, with_sel: bool = False, stream=None):
        out = torch.empty_like(q)
        sel = cnt = None
        if with_sel:
            nl = max(self.n_sel_levels, 1)
            sel = torch.empty(q.shape[0], self.cfg.n_kv_heads, nl, self.cfg.k, dtype=torch.int32,
                              device=q.device)
            cnt = torch.empty(q.shape[0], self.cfg.n_kv_heads, self.n_sel_levels + 1,
                              dtype=torch.int32, device=q.device)
        self.recsa_decode(q, out, sel, cnt, stream)
        return out, sel, cnt

    def prefill(self, Q: torch.Tensor, pos0: int, with_sel: bool = False, stream=None):
        O = torch.empty_like(Q)
        sel = cnt = None
        if with_sel:
            nq = Q.shape[0] * Q.shape[1]
            nl = max(self.n_sel_levels, 1)
            sel = torch.empty(nq, self.cfg.n_kv_heads, nl, self.cfg.k, dtype=torch.int32,
                              device=Q.device)
            cnt = torch.empty(nq, self.cfg.n_kv_heads, self.n_sel_levels + 1, dtype=torch.int32,
                              device=Q.device)
        self.recsa_prefill_chunk(Q, pos0, O, sel, cnt, stream)
        return O, sel, cnt

    def level_tables(self, level: int):
        """(K, V) views [batch][Hkv][rows][d] of level `level` >= 1 in the levels buffer."""
        ko, vo, rows = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(lib.recsa_level_info(self.handle, level, ctypes.byref(ko), ctypes.byref(vo),
                                    ctypes.byref(rows)), "recsa_level_info")
        es = torch.empty((), dtype=self.cfg.torch_dtype).element_size()
        n = self.batch * self.cfg.n_kv_heads * rows.value * self.cfg.head_dim
        shape = (self.batch, self.cfg.n_kv_heads, rows.value, self.cfg.head_dim)
        K = self.levels[ko.value: ko.value + n * es].view(self.cfg.torch_dtype).view(shape)
        V = self.levels[vo.value: vo.value + n * es].view(self.cfg.torch_dtype).view(shape)
        return K, V
