"""Seeded synthetic inputs for the RSM mixer workloads.

This module only draws random tensors; it holds none of the mixer's arithmetic. Both the CUDA
library's tests/benchmark and the CPU oracle receive the same tensors from here.

Input recipe (the pages run no public benchmark for this path, so all inputs are synthetic):
  q, k ~ N(0,1), each row L2-normalised over the M slots in fp32, then cast to the input dtype;
  v ~ N(0,1); router logits ~ N(0,1) in fp32;
  per-head (Mamba2-style) log-decay f = -softplus(N(0,1)), shape [B,T,H];
  per-slot (GLA-style) log-decay  f = -softplus(N(0,1)) / 16, shape [B,T,H,M];
  H0 = 0 unless a test asks for a random initial state (then N(0,1)).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    M: int
    K: int
    Dv: int
    dtype: str          # "f32" or "bf16" for q, k, v
    decay: str          # "head" (f [B,T,H]) or "slot" (f [B,T,H,M])
    seed: int
    T: int = 0          # prefill length (0 for pure decode)
    chunk: int = 64
    decode_prefill_T: int = 0
    decode_steps: int = 0
    notes: str = field(default="")

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# The five workloads: a tiny fp32 oracle check, the pages' small training shape, a mid-size
# per-slot-decay prefill, a 32K-token long-context prefill (16x a 2048 training length) and a
# 256-sequence decode after a 2048-token prefill.
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", B=1, T=128, H=2, M=64, K=16, Dv=64, dtype="f32",
                          decay="head", seed=0),
    "small_bf16": Workload("small_bf16", B=4, T=128, H=4, M=64, K=16, Dv=64, dtype="bf16",
                           decay="head", seed=1),
    "mid_gla_bf16": Workload("mid_gla_bf16", B=8, T=2048, H=8, M=128, K=16, Dv=128,
                             dtype="bf16", decay="slot", seed=2),
    "long_ctx_bf16": Workload("long_ctx_bf16", B=1, T=32768, H=16, M=128, K=16, Dv=128,
                              dtype="bf16", decay="head", seed=3),
    "decode_256x16": Workload("decode_256x16", B=256, H=16, M=128, K=16, Dv=128, dtype="bf16",
                              decay="head", seed=4, decode_prefill_T=2048, decode_steps=1024),
}


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def make_inputs(B: int, T: int, H: int, M: int, Dv: int, dtype: torch.dtype, decay: str,
                seed: int, device="cpu", h0: bool = False) -> dict:
    """Draws q, k, v, logits, f (and optionally H0) with the recipe above.

    Shapes: q, k, logits [B,T,H,M]; v [B,T,H,Dv]; f [B,T,H] or [B,T,H,M]; H0 [B,H,M,Dv] fp32.
    """
    g = _gen(device, seed)
    kw = dict(generator=g, device=device, dtype=torch.float32)
    q = _unit_rows(torch.randn(B, T, H, M, **kw)).to(dtype)
    k = _unit_rows(torch.randn(B, T, H, M, **kw)).to(dtype)
    v = torch.randn(B, T, H, Dv, **kw).to(dtype)
    logits = torch.randn(B, T, H, M, **kw)
    if decay == "head":
        f = -torch.nn.functional.softplus(torch.randn(B, T, H, **kw))
    elif decay == "slot":
        f = -torch.nn.functional.softplus(torch.randn(B, T, H, M, **kw)) / 16.0
    else:
        raise ValueError(decay)
    out = {"q": q, "k": k, "v": v, "logits": logits, "f": f}
    if h0:
        out["H0"] = torch.randn(B, H, M, Dv, **kw)
    return out


def make_workload_inputs(w: Workload, device="cpu", h0: bool = False) -> dict:
    return make_inputs(w.B, w.T, w.H, w.M, w.Dv, w.torch_dtype, w.decay, w.seed, device, h0)


# The generation-decode workload: its state comes from a prefill of `decode_prefill_T` random
# tokens for every sequence, drawn in groups of `DECODE_PREFILL_GROUP` sequences (bounded input
# memory), then `decode_steps` single-token steps. The benchmark and the tests draw the same
# tensors through these two functions.
DECODE_PREFILL_GROUP = 32


def decode_prefill_group(w: Workload, b0: int, rank: int = 0, device="cpu") -> dict:
    """Prefill inputs of sequences b0 .. b0 + DECODE_PREFILL_GROUP - 1 of a decode workload."""
    return make_inputs(DECODE_PREFILL_GROUP, w.decode_prefill_T, w.H, w.M, w.Dv, w.torch_dtype,
                       w.decay, seed=w.seed + b0 + 1000 * rank, device=device)


def decode_step_inputs(w: Workload, steps: int, rank: int = 0, device="cpu") -> dict:
    """Inputs of `steps` decode steps, stacked on a leading step axis: q, k, logits [S,B,H,M],
    v [S,B,H,Dv], f [S,B,H] or [S,B,H,M]."""
    return make_inputs(steps, w.B, w.H, w.M, w.Dv, w.torch_dtype, w.decay,
                       seed=w.seed + 7 + 1000 * rank, device=device)
