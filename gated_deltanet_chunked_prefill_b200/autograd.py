"""PyTorch autograd entry point with the flash-linear-attention call signature.

The pages describe the library as a drop-in GDN backend behind the usual flash-linear-attention
entry point ("FlashQLA resource", section 5, release table: v0.1.1 aligned the entry signatures
with that interface, v0.1.2 serves as its GDN backend; "Qwen's FlashQLA targets the expensive bit
of long-context AI", highlight "Plug-and-play integration"). `chunk_gated_delta_rule` takes the
same arguments in the same layout and returns (o, final_state).

Argument marshalling only: the forward is one gdn_chunk_fwd call through the C ABI and the
backward one gdn_chunk_bwd call. When gradients are needed the forward also fills the chunk-state
cache (gdn_options.states), which the backward reads instead of re-running the forward pass; it
is held between the two calls like any saved activation (56 KB per 64-token chunk and v-head).
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import chunk_states, gdn_chunk_bwd, gdn_chunk_fwd

__all__ = ["chunk_gated_delta_rule", "backward_supported"]


def backward_supported(q: torch.Tensor, v: torch.Tensor) -> bool:
    """The backward takes what the forward takes: bf16 or fp32 with dk, dv in {64, 128} (tensor cores
    for bf16 with dk = dv = 128, CUDA cores otherwise)."""
    return q.dtype in (torch.bfloat16, torch.float32) and q.shape[-1] in (64, 128) and v.shape[-1] in (64, 128)


def _tensor_core_path(q: torch.Tensor, v: torch.Tensor) -> bool:
    """bf16 with dk = dv = 128: the path whose forward can keep a chunk-state cache for its backward."""
    return q.dtype == torch.bfloat16 and q.shape[-1] == 128 and v.shape[-1] == 128


class _ChunkGatedDeltaRule(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, g, beta, scale, initial_state, output_final_state, cu_seqlens,
                cp_segment_chunks, needs_grad, qk_l2norm):
        states = chunk_states(q, v, cu_seqlens) if needs_grad and _tensor_core_path(q, v) else None
        o, hT = gdn_chunk_fwd(q, k, v, g, beta, scale, initial_state, cu_seqlens,
                              output_final_state=output_final_state,
                              cp_segment_chunks=cp_segment_chunks, states=states, qk_l2norm=qk_l2norm)
        ctx.set_materialize_grads(False)
        ctx.scale = scale
        ctx.qk_l2norm = qk_l2norm
        ctx.cp_segment_chunks = cp_segment_chunks
        ctx.want_dh0 = initial_state is not None and ctx.needs_input_grad[6]
        ctx.save_for_backward(q, k, v, g, beta, initial_state, cu_seqlens, states)
        return o, hT

    @staticmethod
    def backward(ctx, do, dht):
        q, k, v, g, beta, h0, cu_seqlens, states = ctx.saved_tensors
        if do is None:
            do = torch.zeros(q.shape[:2] + v.shape[2:], dtype=q.dtype, device=q.device)
        gr = gdn_chunk_bwd(q, k, v, g, beta, do.contiguous(), ctx.scale, h0,
                           None if dht is None else dht.contiguous(), cu_seqlens,
                           cp_segment_chunks=ctx.cp_segment_chunks, want_dh0=ctx.want_dh0,
                           states=states, qk_l2norm=ctx.qk_l2norm)
        return (gr["dq"], gr["dk"], gr["dv"], gr["dg"], gr["dbeta"], None, gr["dh0"], None, None,
                None, None, None)


def _host_cu_seqlens(cu: torch.Tensor, T: int) -> None:
    """Check a host-side cu_seqlens before it goes to the device: the kernels only report an
    inconsistent one through their status word, after the fact."""
    c = cu.tolist()
    if not c or c[0] != 0 or c[-1] != T or any(b < a for a, b in zip(c, c[1:])):
        raise ValueError(f"cu_seqlens must rise from 0 to T={T} without decreasing, got {c[:8]}...")


def chunk_gated_delta_rule(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                           beta: torch.Tensor, scale: Optional[float] = None,
                           initial_state: Optional[torch.Tensor] = None,
                           output_final_state: bool = False,
                           cu_seqlens: Optional[torch.Tensor] = None,
                           use_qk_l2norm_in_kernel: bool = False,
                           cp_segment_chunks: int = 0
                           ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Gated delta rule over 64-token chunks, differentiable.

    q, k [B,T,Hqk,dk] and v [B,T,Hv,dv], beta [B,T,Hv] in one dtype (bf16 or fp32); g [B,T,Hv]
    fp32, the raw per-token log-decay (the cumulative sum inside each chunk is part of the op);
    initial_state [N,Hv,dk,dv] fp32 (N = B, or the number of packed sequences); cu_seqlens
    [N+1] sequence starts of a packed batch (B = 1; int32 or int64). scale defaults to
    dk ** -0.5. Returns o [B,T,Hv,dv] and, if output_final_state, the final state
    [N,Hv,dk,dv] fp32, else None.

    Gradients flow to q, k, v, g, beta and initial_state, for bf16 and fp32 with dk, dv in
    {64, 128} (bf16 with dk = dv = 128 on tensor cores, the rest on CUDA cores).
    use_qk_l2norm_in_kernel: q and k rows are divided by sqrt(|x|^2 + 1e-6) inside the kernels
    (bf16, dk = dv = 128), and their gradients are taken through that normalisation. A cu_seqlens
    on the host is checked before it is copied to the device; one already on the device is not
    (the kernels report an inconsistent one only through their status word).
    """
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (g, "g"), (beta, "beta")):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
    q, k, v, g, beta = (t.contiguous() for t in (q, k, v, g, beta))
    if initial_state is not None:
        initial_state = initial_state.contiguous()
    if cu_seqlens is not None:
        if cu_seqlens.dtype not in (torch.int32, torch.int64):
            raise TypeError("cu_seqlens must be int32 or int64")
        if not cu_seqlens.is_cuda:
            _host_cu_seqlens(cu_seqlens, q.shape[1])
        cu_seqlens = cu_seqlens.to(device=q.device, dtype=torch.int32).contiguous()
    scale = q.shape[-1] ** -0.5 if scale is None else float(scale)
    needs_grad = torch.is_grad_enabled() and (
        any(t.requires_grad for t in (q, k, v, g, beta))
        or (initial_state is not None and initial_state.requires_grad))
    if needs_grad and not backward_supported(q, v):
        raise NotImplementedError("backward: bf16 or fp32 with dk, dv in {64, 128}")
    return _ChunkGatedDeltaRule.apply(q, k, v, g, beta, scale, initial_state, output_final_state,
                                      cu_seqlens, int(cp_segment_chunks), needs_grad,
                                      bool(use_qk_l2norm_in_kernel))
