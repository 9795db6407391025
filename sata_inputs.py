"""Seeded synthetic inputs for the SATA attention workloads.

This module only draws random numbers and names shapes. It holds none of the
method's arithmetic, so both the fp64 oracle (under ``oracle/``) and the CUDA
path may take their inputs from it without sharing any computation.

Recipe (every workload): a ``torch.Generator('cpu')`` seeded with
``SEED_BASE + workload_id`` draws q, then k, then v as i.i.d. N(0,1) fp32 in
``[B, H, N, d]`` order; workloads with bf16 inputs cast each tensor to bf16
(round to nearest even) and both sides consume those exact bf16 values.
Decode workloads draw their prefill with ``seed + 100`` and the single-token
steps sequentially from one generator seeded ``seed + 200``, each step drawing
q, k, v of shape ``[B, H, 1, d]`` in that order.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

SEED_BASE = 20261202


@dataclass(frozen=True)
class Workload:
    """Shape of one SATA workload: q,k ``[B,H,N,dK]``, v ``[B,H,N,dV]``."""

    wid: int
    B: int
    H: int
    N: int
    dK: int
    dV: int
    P: int
    dtype: str  # "f32" or "bf16": dtype of q, k, v
    decode_steps: int = 0
    note: str = ""

    @property
    def seed(self) -> int:
        return SEED_BASE + self.wid


# The five workloads the hot path is specified on (tiny reference, small fp32,
# mid bf16, long bf16 prefill, batched decode).
WORKLOADS = {
    1: Workload(1, 1, 1, 64, 8, 8, 4, "f32", note="tiny reference"),
    2: Workload(2, 2, 4, 1024, 16, 16, 4, "f32", note="fp32; also P=2,3 for error-vs-P"),
    3: Workload(3, 4, 8, 4096, 32, 32, 4, "bf16", note="bf16 prefill"),
    4: Workload(4, 1, 8, 16384, 64, 64, 4, "bf16", note="bf16 prefill on tensor cores"),
    5: Workload(5, 32, 8, 8192, 64, 64, 4, "bf16", decode_steps=1024,
                note="prefill N=8192 then 1024 single-token decode steps"),
}


def _draw(gen: torch.Generator, B: int, H: int, N: int, dK: int, dV: int, dtype: str):
    q = torch.randn(B, H, N, dK, generator=gen, dtype=torch.float32)
    k = torch.randn(B, H, N, dK, generator=gen, dtype=torch.float32)
    v = torch.randn(B, H, N, dV, generator=gen, dtype=torch.float32)
    if dtype == "bf16":
        q, k, v = q.bfloat16(), k.bfloat16(), v.bfloat16()
    elif dtype != "f32":
        raise ValueError(f"unknown dtype {dtype!r}")
    return q, k, v


def make_qkv(B: int, H: int, N: int, dK: int, dV: int, seed: int, dtype: str = "f32"):
    """q, k, v on the CPU, drawn from one generator seeded ``seed``.

    Returns tensors of dtype float32 or bfloat16 (as ``dtype`` says).
    """
    gen = torch.Generator("cpu").manual_seed(int(seed))
    return _draw(gen, B, H, N, dK, dV, dtype)


def workload_inputs(wid: int, N: int | None = None, P: int | None = None):
    """Prefill inputs of workload ``wid`` (optionally with another N)."""
    w = WORKLOADS[wid]
    seed = w.seed + (100 if w.decode_steps else 0)
    n = w.N if N is None else N
    return make_qkv(w.B, w.H, n, w.dK, w.dV, seed, w.dtype)


class DecodeStream:
    """Sequential single-token inputs of a decode workload: step t -> (q, k, v)."""

    def __init__(self, wid: int, B: int | None = None, H: int | None = None):
        w = WORKLOADS[wid]
        self.w = w
        self.B = w.B if B is None else B
        self.H = w.H if H is None else H
        self.gen = torch.Generator("cpu").manual_seed(w.seed + 200)

    def next(self):
        w = self.w
        return _draw(self.gen, self.B, self.H, 1, w.dK, w.dV, w.dtype)


def as_f64_numpy(t: torch.Tensor):
    """Exact widening of fp32/bf16 values to float64 numpy."""
    return t.detach().to("cpu").to(torch.float64).numpy()
