"""The Ulysses attention layer under ``torch.autograd``.

Forward: mode-0 repack of the stacked Q/K/V(/G) input into the head-sharded
layout, attention keeping the base-2 log-sum-exp of every query row, mode-1
repack of the output.  Backward: ``ulysses_layer_bwd`` under the forward's
plan -- the rule of "hao-ai-lab FastVideo, compare main...perf/ulysses-h3-
adaptive" (docs, and ``_FusedUlyssesA2A.backward`` in ``ulysses_a2a.py``) that
the backward reuses the plan its forward saved.

Every arithmetic step runs in ``libulysses.so``; this module allocates the
tensors the C entry points write and passes their addresses.  The softmax
scale is 1/sqrt(D), as in ``ulysses_layer_fwd``.
"""
from __future__ import annotations

import math

import torch

from . import _lib as L


def _empty_like_layout(x: torch.Tensor) -> torch.Tensor:
    # same shape and strides as x (the plan's input layout)
    return torch.empty_strided(x.shape, x.stride(), dtype=x.dtype, device=x.device)


class UlyssesAttention(torch.autograd.Function):
    """``out = UlyssesAttention.apply(qkv_seq, plan)``.

    qkv_seq: bf16 CUDA tensor ``[Np, C, H, D]`` in the layout the plan was made
    for (token-interleaved by default, or a strided view of the stacked
    ``[C, Np, H, D]`` buffer).  Returns ``[Np, H, D]`` bf16.  The gradient has
    the input's layout; planes >= 3 (a gate) get zeros, since attention does
    not read them.
    """

    @staticmethod
    def forward(ctx, qkv_seq: torch.Tensor, plan: L.Plan) -> torch.Tensor:
        if not qkv_seq.is_cuda or qkv_seq.dtype != torch.bfloat16:
            raise TypeError("qkv_seq must be a bf16 CUDA tensor")
        Np, P, C, H, D = plan.padded_tokens, plan.P, plan.planes, plan.H, plan.D
        if tuple(qkv_seq.shape) != (Np, C, H, D):
            raise ValueError(f"qkv_seq shape {tuple(qkv_seq.shape)} != {(Np, C, H, D)}")
        Hl = H // P
        dev = qkv_seq.device
        stream = torch.cuda.current_stream(dev).cuda_stream
        T = torch.empty((P, C, Np, Hl, D), dtype=torch.bfloat16, device=dev)
        OT = torch.empty((P, Np, Hl, D), dtype=torch.bfloat16, device=dev)
        lse = torch.empty(plan.lse_bytes // 4, dtype=torch.float32, device=dev)
        out = torch.empty((Np, H, D), dtype=torch.bfloat16, device=dev)
        L.ulysses_repack_fwd(plan, qkv_seq, T, stream=stream)
        L.ulysses_attn_fwd_lse(plan, T, OT, lse, 1.0 / math.sqrt(D), stream=stream)
        L.ulysses_repack_bwd(plan, OT, out, 1, stream=stream)
        ctx.plan = plan
        ctx.save_for_backward(qkv_seq, T, OT, lse)
        return out

    @staticmethod
    def backward(ctx, dout: torch.Tensor):
        qkv_seq, T, OT, lse = ctx.saved_tensors
        plan = ctx.plan
        dev = qkv_seq.device
        stream = torch.cuda.current_stream(dev).cuda_stream
        dout = dout.to(torch.bfloat16).contiguous()
        dqkv = _empty_like_layout(qkv_seq)
        if plan.planes > 3:
            dqkv[:, 3:].zero_()
        ws = torch.empty(plan.layer_bwd_workspace_bytes, dtype=torch.uint8, device=dev)
        L.ulysses_layer_bwd(plan, T, OT, lse, dout, dqkv, ws, stream=stream)
        return dqkv, None


def ulysses_attention(qkv_seq: torch.Tensor, plan: L.Plan) -> torch.Tensor:
    """Functional form of :class:`UlyssesAttention`."""
    return UlyssesAttention.apply(qkv_seq, plan)
