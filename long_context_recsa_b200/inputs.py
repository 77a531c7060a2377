"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle side.

This module only draws random numbers and places them; it holds none of the
RecSA arithmetic.  Every tensor is drawn per (stream, sequence, KV head) slice
from its own seed, so any slice can be regenerated alone.

Recipe (stands in for Qwen3-4B attention inputs on RULER-style long contexts,
which are not available here):
  * K, V, q ~ N(0, 1), drawn in fp32 by ``torch.randn`` and rounded to the
    storage dtype (round to nearest even).
  * pooler logits w in R^C ~ N(0, 1) from the CPU generator, seed 7.
  * gated-pooler parameters (Eq.5, forward only): seeded stand-ins, seed 11.
  * needles: seeded positions whose keys are set to ``gain`` times the mean of
    the GQA group's query heads (before RoPE), so that selection is non-trivial.
  * seed of a slice = 1_000_000*config + 10_000*stream + 100*sequence + head;
    streams: K=1, V=2, q=3, needle positions=4, appended k=5, appended v=6,
    appended q=7.
"""
from __future__ import annotations

import torch

STREAM_K, STREAM_V, STREAM_Q, STREAM_NEEDLE = 1, 2, 3, 4
STREAM_KNEW, STREAM_VNEW, STREAM_QNEW = 5, 6, 7

_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def torch_dtype(name: str) -> torch.dtype:
    return _DT[name]


def slice_seed(config: int, stream: int, seq: int = 0, head: int = 0) -> int:
    return 1_000_000 * config + 10_000 * stream + 100 * seq + head


def randn(shape, seed: int, dtype: str = "f32", device="cpu") -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn(*shape, generator=g, dtype=torch.float32, device=device)
    return x.to(_DT[dtype])


def pooler_w(C: int, seed: int = 7) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return torch.randn(C, generator=g, dtype=torch.float32)


def gated_pooler_params(d: int, hidden: int | None = None, seed: int = 11) -> dict:
    """Seeded stand-in parameters of the gated pooler (trained values are not
    available): w, tau, g, rho and the MLP W1 [hidden][2d], b1 [hidden], W2
    [d][hidden], drawn on the CPU generator and returned as fp64 tensors/floats.
    Scales keep the pooled keys of N(0, 1) children O(1)."""
    h = d if hidden is None else hidden
    gen = torch.Generator().manual_seed(seed)
    def nrm(*shape, std):
        return (torch.randn(*shape, generator=gen, dtype=torch.float64) * std)
    return {
        "w": nrm(d, std=d ** -0.5),
        "tau": 2.0,
        "g": 0.75,
        "rho": float(d) ** 0.5,
        "W1": nrm(h, 2 * d, std=(2 * d) ** -0.5),
        "b1": nrm(h, std=0.1),
        "W2": nrm(d, h, std=0.1 * h ** -0.5),
    }


def kv_slice(config: int, seq: int, head: int, L: int, d: int, dtype: str, device="cpu"):
    """Level-0 keys and values of one (sequence, KV head): two [L, d] tensors."""
    K = randn((L, d), slice_seed(config, STREAM_K, seq, head), dtype, device)
    V = randn((L, d), slice_seed(config, STREAM_V, seq, head), dtype, device)
    return K, V


def q_rows(config: int, seq: int, n_rows: int, Hq: int, d: int, dtype: str,
           stream: int = STREAM_Q, device="cpu"):
    """Query rows of one sequence: [n_rows, Hq, d]."""
    return randn((n_rows, Hq, d), slice_seed(config, stream, seq, 0), dtype, device)


def needle_positions(config: int, seq: int, n_needles: int, L: int) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(slice_seed(config, STREAM_NEEDLE, seq, 0))
    return torch.randperm(L, generator=g)[:n_needles].sort().values


def needle_keys(q_group: torch.Tensor, gain: float, dtype: str) -> torch.Tensor:
    """Needle key of one KV head: gain * mean of its group's query heads."""
    return (gain * q_group.float().mean(dim=0)).to(_DT[dtype])
