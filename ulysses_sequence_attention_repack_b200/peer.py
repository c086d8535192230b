"""The Ulysses layer across P GPUs, one process per GPU, over peer memory.

Rank q holds the sequence rows [q*Nl, (q+1)*Nl) of the input as a shard
[Nl, C, H, D] (token-interleaved).  One forward is

  1. ``ulysses_repack_fwd_push``: rank q stores, for every rank r, its rows of
     r's heads into r's head slab T_r [C, Np, Hl, D] through a peer pointer
     (step 1, the all-to-all of the transport page, as a push);
  2. a stream-ordered barrier: every rank's stores into T_r have completed;
  3. ``ulysses_attn_fwd_push``: attention over T_r, whose epilogue stores each
     output row into its owning rank's output shard [Nl, H, D] (steps 2 and 3
     in one kernel);
  4. a barrier: every output shard is complete.

For training (``training=True``) step 3 keeps this rank's head-sharded
output and log-sum-exp (``ulysses_attn_fwd_lse_slab``, then
``ulysses_repack_bwd_push`` of the output), and the backward is

  5. ``ulysses_repack_fwd_push`` of the output gradient (one plane) into
     every rank's dO slab, a barrier;
  6. ``ulysses_attn_bwd_slab``: dQ, dK, dV of this rank's heads;
  7. ``ulysses_repack_bwd_push`` of the three gradient planes into their
     owners' gradient shards, a barrier.

The slabs and shards are allocated in PyTorch's symmetric memory, which maps
every rank's allocation into every peer (NVLink over NVSwitch) and provides
the barrier; every byte of the layer is moved and computed by this library's
kernels.  All ranks must build the plan with the same arguments; the
constructor checks that (``agree_plan``).

``exchange="ipc"`` maps the peers' buffers through CUDA IPC handles instead
(ordinary allocations; the handles cross in one all-gather over the group),
and each barrier becomes a host barrier: the stream is synchronised, then
``torch.distributed.barrier``.  It serves groups without symmetric memory,
gloo groups included, and processes that share one GPU: no kernel of one
rank then waits on another rank's kernel.
"""
from __future__ import annotations

import functools
import math
import os

from ._lib import (Plan, ulysses_a2a_pack, ulysses_a2a_unpack, ulysses_attn_bwd_slab, ulysses_attn_fwd_lse_slab,
                   ulysses_attn_fwd_push, ulysses_repack_bwd_push, ulysses_repack_fwd_push)


def plan_signature(plan: Plan) -> tuple:
    """What every rank's plan must agree on."""
    return (plan.N, plan.H, plan.D, plan.P, plan.planes,
            None if plan.cu_seqlens is None else tuple(plan.cu_seqlens), plan.causal)


def agree_plan(plan: Plan, group=None) -> None:
    """Raise ValueError on every rank unless the group has P ranks that all
    hold the same plan (a collective: every rank of the group must call it)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    sigs = [None] * world
    dist.all_gather_object(sigs, plan_signature(plan), group=group)
    if world != plan.P:
        raise ValueError(f"the plan has P={plan.P} ranks but the group has {world}")
    bad = [r for r, s in enumerate(sigs) if s != sigs[0]]
    if bad:
        raise ValueError(f"plans differ across ranks: ranks {bad} disagree with rank 0 ({sigs[0]} vs {sigs[bad[0]]})")


class PeerLayer:
    """One rank of the layer over P GPUs (softmax scale 1/sqrt(D) by default).

    ``forward(shard)`` returns this rank's output shard [Nl, H, D]; the tensor
    is reused by the next forward, so copy it to keep it.  Everything runs on
    the current CUDA stream.
    """

    def __init__(self, plan: Plan, group=None, device=None, softmax_scale: float | None = None,
                 training: bool = False, exchange: str = "symmetric"):
        import torch
        import torch.distributed as dist
        if exchange not in ("symmetric", "ipc"):
            raise ValueError("exchange must be 'symmetric' or 'ipc'")
        agree_plan(plan, group)
        self.plan = plan
        self.group = group if group is not None else dist.group.WORLD
        self.rank = dist.get_rank(self.group)
        self.device = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.scale = float(softmax_scale) if softmax_scale is not None else 1.0 / math.sqrt(plan.D)
        self.exchange = exchange
        self._ipc_keep = []   # peer tensors opened from IPC handles (keep the mappings alive)
        C, Np, Nl, H = plan.planes, plan.padded_tokens, plan.rows_per_rank, plan.H
        Hl = H // plan.P
        bf = dict(dtype=torch.bfloat16, device=self.device)
        # buffers the peers store into: (tensor, handle) pairs
        self.heads, self._heads_h = self._shared((C, Np, Hl, plan.D))
        self.out, self._out_h = self._shared((Nl, H, plan.D))
        self.heads_ptrs = self._peer_ptrs(self._heads_h, self.heads)
        self.out_ptrs = self._peer_ptrs(self._out_h, self.out)
        self.training = bool(training)
        if self.training:
            # this rank's output and lse for the backward, the dO slab and the
            # gradient shard the peers push into, and the backward's scratch
            self.out_heads = torch.empty(Np, Hl, plan.D, **bf)
            self.lse = torch.empty(plan.slab_lse_bytes // 4, dtype=torch.float32, device=self.device)
            self.dout_heads, self._dout_h = self._shared((1, Np, Hl, plan.D))
            self.dqkv_heads = torch.empty(3, Np, Hl, plan.D, **bf)
            self.grad, self._grad_h = self._shared((Nl, 3, H, plan.D))
            self.bwd_ws = torch.empty(plan.slab_attn_bwd_workspace_bytes, dtype=torch.uint8, device=self.device)
            self.dout_ptrs = self._peer_ptrs(self._dout_h, self.dout_heads)
            self.grad_ptrs = self._peer_ptrs(self._grad_h, self.grad)

    def _shared(self, shape):
        """A bf16 buffer the peers can store into, and its exchange handle."""
        import torch
        if self.exchange == "ipc":
            return torch.empty(shape, dtype=torch.bfloat16, device=self.device), None
        from torch.distributed import _symmetric_memory as symm
        # no NVLink multicast object is needed: the kernels use plain peer stores
        os.environ.setdefault("TORCH_SYMM_MEM_DISABLE_MULTICAST", "1")
        t = symm.empty(*shape, dtype=torch.bfloat16, device=self.device)
        return t, symm.rendezvous(t, self.group)

    def _peer_ptrs(self, handle, local) -> list[int]:
        """Every rank's address of the same tensor, as mapped on this device."""
        if self.exchange == "ipc":
            return self._ipc_ptrs(local)
        ptrs = [int(p) for p in handle.buffer_ptrs]
        off = local.data_ptr() - ptrs[self.rank]
        return [p + off for p in ptrs]

    def _ipc_ptrs(self, local) -> list[int]:
        """The peers' addresses of their copy of `local`, opened from the CUDA
        IPC handles every rank publishes in one all-gather (a collective)."""
        import torch.distributed as dist
        from torch.multiprocessing.reductions import reduce_tensor
        shared = [None] * dist.get_world_size(self.group)
        dist.all_gather_object(shared, reduce_tensor(local), group=self.group)
        ptrs = []
        for r, (rebuild, args) in enumerate(shared):
            if r == self.rank:
                ptrs.append(local.data_ptr())
                continue
            t = rebuild(*args)
            self._ipc_keep.append(t)
            ptrs.append(t.data_ptr())
        return ptrs

    def _barrier(self, handle, channel: int) -> None:
        """Every rank's stores issued so far are complete before any rank goes on."""
        if self.exchange == "ipc":
            import torch
            import torch.distributed as dist
            torch.cuda.current_stream(self.device).synchronize()
            dist.barrier(group=self.group)
        else:
            handle.barrier(channel=channel)

    def forward(self, shard):
        """shard: this rank's rows [Nl, C, H, D] (bf16, on this rank's device)."""
        ulysses_repack_fwd_push(self.plan, self.rank, shard, self.heads_ptrs)
        self._barrier(self._heads_h, 0)
        if self.training:
            ulysses_attn_fwd_lse_slab(self.plan, self.heads, self.out_heads, self.lse, self.scale)
            ulysses_repack_bwd_push(self.plan, self.rank, self.out_heads, self.out_ptrs, 1)
        else:
            ulysses_attn_fwd_push(self.plan, self.rank, self.heads, self.out_ptrs, self.scale)
        self._barrier(self._out_h, 1)
        return self.out

    __call__ = forward

    def backward(self, dout_shard):
        """dout_shard: the gradient of this rank's output rows [Nl, H, D].
        Returns this rank's (dQ, dK, dV) rows [Nl, 3, H, D] (reused by the
        next backward).  Needs ``training=True`` and the forward of the same
        input just before it on every rank."""
        if not self.training:
            raise RuntimeError("PeerLayer was built without training=True")
        ulysses_repack_fwd_push(self.plan, self.rank, dout_shard, self.dout_ptrs, 1)
        self._barrier(self._dout_h, 0)
        ulysses_attn_bwd_slab(self.plan, self.heads, self.out_heads, self.dout_heads, self.lse, self.dqkv_heads,
                              self.bwd_ws, self.scale)
        ulysses_repack_bwd_push(self.plan, self.rank, self.dqkv_heads, self.grad_ptrs, 3)
        self._barrier(self._grad_h, 1)
        return self.grad


class CollectiveLayer:
    """The same layer where ranks cannot map each other's memory: the bytes
    cross in ``torch.distributed.all_to_all_single`` (NCCL) and this library's
    kernels pack and unpack them (``ulysses_a2a_pack`` / ``ulysses_a2a_unpack``)
    around the one-slab attention.  One exchange per plane, as the transport
    page's fallback to a bulk all-to-all.  Same interface as ``PeerLayer``;
    the output and gradients are its bit for bit.
    """

    def __init__(self, plan: Plan, group=None, device=None, softmax_scale: float | None = None,
                 training: bool = False):
        import torch
        import torch.distributed as dist
        agree_plan(plan, group)
        self.plan = plan
        self.group = group
        self.rank = dist.get_rank(group)
        self.device = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.scale = float(softmax_scale) if softmax_scale is not None else 1.0 / math.sqrt(plan.D)
        self.training = bool(training)
        C, Np, Nl, H, D = plan.planes, plan.padded_tokens, plan.rows_per_rank, plan.H, plan.D
        Hl = H // plan.P
        bf = dict(dtype=torch.bfloat16, device=self.device)
        self.heads = torch.empty(C, Np, Hl, D, **bf)
        self.send = torch.empty(Np, Hl, D, **bf)          # [P, Nl, Hl, D] in destination order
        self.recv = torch.empty(Np, Hl, D, **bf)
        self.out = torch.empty(Nl, H, D, **bf)
        self.out_heads = torch.empty(Np, Hl, D, **bf)
        self.lse = torch.empty(plan.slab_lse_bytes // 4, dtype=torch.float32, device=self.device)
        if self.training:
            self.dout_heads = torch.empty(1, Np, Hl, D, **bf)
            self.dqkv_heads = torch.empty(3, Np, Hl, D, **bf)
            self.grad = torch.empty(Nl, 3, H, D, **bf)
            self.bwd_ws = torch.empty(plan.slab_attn_bwd_workspace_bytes, dtype=torch.uint8, device=self.device)

    def _exchange(self, dst, src):
        import torch.distributed as dist
        dist.all_to_all_single(dst, src, group=self.group)

    def forward(self, shard):
        p, C = self.plan, self.plan.planes
        for c in range(C):
            ulysses_a2a_pack(p, shard, C, c, self.send)
            self._exchange(self.heads[c], self.send)
        ulysses_attn_fwd_lse_slab(p, self.heads, self.out_heads, self.lse, self.scale)
        self._exchange(self.recv, self.out_heads)
        ulysses_a2a_unpack(p, self.recv, self.out, 1, 0)
        return self.out

    __call__ = forward

    def backward(self, dout_shard):
        if not self.training:
            raise RuntimeError("CollectiveLayer was built without training=True")
        p = self.plan
        ulysses_a2a_pack(p, dout_shard, 1, 0, self.send)
        self._exchange(self.dout_heads[0], self.send)
        ulysses_attn_bwd_slab(p, self.heads, self.out_heads, self.dout_heads, self.lse, self.dqkv_heads,
                              self.bwd_ws, self.scale)
        for c in range(3):
            self._exchange(self.recv, self.dqkv_heads[c])
            ulysses_a2a_unpack(p, self.recv, self.grad, 3, c)
        return self.grad


@functools.lru_cache(maxsize=None)
def _autograd():
    import torch

    class PeerUlyssesAttention(torch.autograd.Function):
        """``out = PeerUlyssesAttention.apply(shard, layer)`` on every rank, with
        ``layer`` a ``PeerLayer`` or ``CollectiveLayer`` built with
        ``training=True``: the rank's output rows
        [Nl, H, D] (a fresh tensor), and in the backward the gradient of its
        input rows [Nl, C, H, D] (planes >= 3, a gate, get zeros)."""

        @staticmethod
        def forward(ctx, shard, layer):
            ctx.layer = layer
            ctx.planes = shard.shape[1]
            return layer.forward(shard).clone()

        @staticmethod
        def backward(ctx, dout):
            layer = ctx.layer
            g = layer.backward(dout.to(torch.bfloat16).contiguous())
            if ctx.planes == 3:
                return g.clone(), None
            full = torch.zeros((g.shape[0], ctx.planes) + tuple(g.shape[2:]), dtype=g.dtype, device=g.device)
            full[:, :3].copy_(g)
            return full, None

    return PeerUlyssesAttention


def peer_ulysses_attention(shard, layer):
    """Functional form: this rank's output rows, differentiable through ``layer``."""
    return _autograd().apply(shard, layer)
