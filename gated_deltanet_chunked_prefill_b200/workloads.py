"""Seeded synthetic inputs for the Gated DeltaNet chunked-prefill operator.

This module only draws random numbers and rounds them to the I/O dtype; it holds
none of the operator's arithmetic. Both the CPU oracle tests and the CUDA path
(tests, bench, smoke) take their inputs from here, so that the two sides see the
same bits.

Value recipe (the operator's standard synthetic workload):
  q, k ~ N(0, 1), then L2-normalised per (token, head);
  v ~ N(0, 1);
  g = logsigmoid(N(0, 1))   (raw per-token log-decay, always <= 0), fp32;
  beta = sigmoid(N(0, 1))   in the I/O dtype;
  h0 ~ h0_std * N(0, 1)     fp32, or absent;
  dO ~ N(0, 1) in the I/O dtype, dhT ~ 0.01 * N(0, 1) fp32 (backward only).
Every array is drawn in fp64 from numpy.random.default_rng(seed), in the fixed
order lengths, q, k, v, g, beta, h0, dO, dhT, then rounded once.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

__all__ = ["Workload", "CONFIGS", "make_inputs", "varlen_lengths", "config_inputs"]


@dataclass
class Workload:
    """Shape and dtype of one synthetic operator call."""
    name: str
    B: int
    T: int
    Hqk: int
    Hv: int
    dk: int
    dv: int
    dtype: str                      # "f32" or "bf16": dtype of q, k, v, beta, o
    h0_std: Optional[float]         # None -> no initial state
    seed: int
    lengths: Optional[list] = None  # packed variable-length sequences (B must be 1)
    backward: bool = False
    description: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return len(self.lengths) if self.lengths is not None else self.B

    @property
    def tokens(self) -> int:
        return self.B * self.T


def varlen_lengths(rng: np.random.Generator, n: int, total: int, lo: int, hi: int) -> list:
    """n lengths drawn log-uniform on [lo, hi], rescaled to sum exactly to `total`.

    Floors the rescaled values and hands the remainder, one token each, to the
    largest fractional parts. Re-draws until at least one length is not a
    multiple of 64 (so that partial chunks are exercised).
    """
    while True:
        raw = np.exp(rng.uniform(math.log(lo), math.log(hi), size=n))
        x = raw * (total / raw.sum())
        base = np.floor(x).astype(np.int64)
        rem = int(total - base.sum())
        order = np.argsort(-(x - base), kind="stable")
        base[order[:rem]] += 1
        base = np.maximum(base, 1)
        # keep the exact total after the max(.,1) guard
        while base.sum() > total:
            base[int(np.argmax(base))] -= 1
        if np.any(base % 64 != 0):
            return [int(v) for v in base]


def _round(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype == "bf16":
        return t.to(torch.float32).to(torch.bfloat16)
    if dtype == "f32":
        return t.to(torch.float32)
    raise ValueError(dtype)


def _l2norm(x: np.ndarray) -> np.ndarray:
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True))


def make_inputs(B: int, T: int, Hqk: int, Hv: int, dk: int, dv: int, dtype: str,
                seed: int, h0_std: Optional[float] = None, lengths=None,
                backward: bool = False, g_scale: float = 1.0, qk_unit: bool = True) -> dict:
    """Draw one seeded input set (CPU tensors).

    Returns a dict with q, k [B,T,Hqk,dk], v [B,T,Hv,dv], beta [B,T,Hv] in the I/O
    dtype; g [B,T,Hv] fp32; h0 [N,Hv,dk,dv] fp32 or None; cu_seqlens int32 [N+1]
    or None; and, when backward, dO [B,T,Hv,dv] (I/O dtype) and dhT [N,Hv,dk,dv]
    fp32. `g_scale` multiplies the N(0,1) draw inside logsigmoid (1.0 = recipe).
    qk_unit=False leaves q and k as drawn, N(0, 1) (for the operator's own normalisation).
    """
    rng = np.random.default_rng(seed)
    if lengths is not None:
        if B != 1:
            raise ValueError("packed sequences need B == 1")
        lengths = [int(v) for v in lengths]
        T = int(sum(lengths))
        N = len(lengths)
        cu = np.zeros(N + 1, dtype=np.int32)
        cu[1:] = np.cumsum(lengths)
        cu_seqlens = torch.from_numpy(cu)
    else:
        N = B
        cu_seqlens = None
    unit = _l2norm if qk_unit else (lambda a: a)
    q = unit(rng.standard_normal((B, T, Hqk, dk)))
    k = unit(rng.standard_normal((B, T, Hqk, dk)))
    v = rng.standard_normal((B, T, Hv, dv))
    xg = rng.standard_normal((B, T, Hv)) * g_scale
    g = -np.logaddexp(0.0, -xg)                      # logsigmoid, <= 0
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, Hv))))
    h0 = None
    if h0_std is not None:
        h0 = torch.from_numpy(h0_std * rng.standard_normal((N, Hv, dk, dv))).to(torch.float32)
    out = dict(q=_round(q, dtype), k=_round(k, dtype), v=_round(v, dtype),
               g=torch.from_numpy(g).to(torch.float32), beta=_round(beta, dtype),
               h0=h0, cu_seqlens=cu_seqlens, scale=dk ** -0.5,
               shape=dict(B=B, T=T, Hqk=Hqk, Hv=Hv, dk=dk, dv=dv, N=N, dtype=dtype))
    if backward:
        out["dO"] = _round(rng.standard_normal((B, T, Hv, dv)), dtype)
        out["dhT"] = torch.from_numpy(0.01 * rng.standard_normal((N, Hv, dk, dv))).to(torch.float32)
    return out


def _varlen_c3() -> list:
    return varlen_lengths(np.random.default_rng(1003), 24, 65536, 256, 16384)


CONFIGS = {
    "tiny_fp32": Workload(
        "tiny_fp32", B=1, T=256, Hqk=2, Hv=2, dk=64, dv=64, dtype="f32", h0_std=None,
        seed=1000, description="tiny GDN forward, fp32: B=1 H=2 T=256 dk=dv=64"),
    "dense_bf16": Workload(
        "dense_bf16", B=4, T=4096, Hqk=16, Hv=16, dk=128, dv=128, dtype="bf16", h0_std=0.1,
        seed=1001, description="dense GDN forward, bf16: B=4 T=4096 H=16 dk=dv=128, h0~N(0,0.1)"),
    "long_gqa_bf16": Workload(
        "long_gqa_bf16", B=1, T=32768, Hqk=16, Hv=32, dk=128, dv=128, dtype="bf16", h0_std=None,
        seed=1002, description="long-context grouped-value GDN forward, bf16: T=32768 Hqk=16 Hv=32"),
    "varlen_bf16": Workload(
        "varlen_bf16", B=1, T=65536, Hqk=16, Hv=16, dk=128, dv=128, dtype="bf16", h0_std=0.1,
        seed=1003, lengths=_varlen_c3(),
        description="packed variable-length GDN forward, bf16: 24 seqs, 65536 tokens, H=16"),
    "bwd_bf16": Workload(
        "bwd_bf16", B=2, T=8192, Hqk=16, Hv=16, dk=128, dv=128, dtype="bf16", h0_std=0.1,
        seed=1004, backward=True,
        description="GDN backward, bf16: B=2 T=8192 H=16 dk=dv=128, dO~N(0,1), dhT~N(0,0.01)"),
}


def config_inputs(name: str) -> dict:
    """Inputs of one named workload (full size)."""
    w = CONFIGS[name]
    return make_inputs(w.B, w.T, w.Hqk, w.Hv, w.dk, w.dv, w.dtype, w.seed,
                       h0_std=w.h0_std, lengths=w.lengths, backward=w.backward)
