"""The repack index map against a real all-to-all between processes (gloo, CPU).

On P real GPUs each virtual rank is a process and step one of the layer is
one all-to-all that scatters heads and gathers the sequence (mode 0 of the
FastVideo Ulysses transport).  Here P CPU processes run that exchange with
torch.distributed.all_to_all_single; each rank's received slab must equal the
oracle's head-sharded slab for that rank bit for bit, and the inverse
exchange must restore the input.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import ulysses_oracle as orc


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, S_bits, result_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        Np, C, H, D = S_bits.shape
        Nl, Hl = Np // world, H // world
        # this rank's sequence shard; bit patterns widened to int32 (gloo has no 16-bit integers)
        x = torch.from_numpy(S_bits[rank * Nl:(rank + 1) * Nl].astype(np.int32))         # [Nl, C, H, D]
        # head block r goes to rank r: [P, C, Nl, Hl, D], split along dim 0
        send = x.reshape(Nl, C, world, Hl, D).permute(2, 1, 0, 3, 4).contiguous()
        recv = torch.empty_like(send)                                                   # [P(src), C, Nl, Hl, D]
        dist.all_to_all_single(recv, send)
        heads = recv.permute(1, 0, 2, 3, 4).reshape(C, world * Nl, Hl, D).contiguous()  # [C, Np, Hl, D]
        # inverse exchange (mode 1) restores the shard
        send_b = heads.reshape(C, world, Nl, Hl, D).permute(1, 0, 2, 3, 4).contiguous()
        recv_b = torch.empty_like(send_b)
        dist.all_to_all_single(recv_b, send_b)
        back = recv_b.permute(2, 1, 0, 3, 4).reshape(Nl, C, H, D)
        np.save(os.path.join(result_dir, f"heads{rank}.npy"), heads.numpy().astype(np.uint16))
        np.save(os.path.join(result_dir, f"back{rank}.npy"), back.numpy().astype(np.uint16))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,Nl,C,H", [(2, 5, 3, 4), (4, 3, 4, 8)])
def test_all_to_all_processes_match_oracle_repack(tmp_path, world, Nl, C, H):
    rng = np.random.default_rng(world)
    S = rng.integers(0, 1 << 16, size=(world * Nl, C, H, 4), dtype=np.uint16)
    mp.start_processes(_worker, args=(world, _free_port(), S, str(tmp_path)), nprocs=world, start_method="spawn")
    T = orc.repack_fwd(S, world)
    for r in range(world):
        assert np.array_equal(np.load(tmp_path / f"heads{r}.npy"), T[r])
        Nl_ = S.shape[0] // world
        assert np.array_equal(np.load(tmp_path / f"back{r}.npy"), S[r * Nl_:(r + 1) * Nl_])


def _agree_worker(rank, world, port, Ns, result_dir):
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import peer
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        plan = U.ulysses_plan(Ns[rank], 8, 128, world, 3)
        try:
            peer.agree_plan(plan)
            verdict = "ok"
        except ValueError as e:
            verdict = "refused: " + str(e)
        with open(os.path.join(result_dir, f"agree{rank}.txt"), "w") as f:
            f.write(verdict)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("Ns,expect_ok", [((1024, 1024), True), ((1024, 1000), False)])
def test_ranks_agree_on_the_plan(tmp_path, Ns, expect_ok):
    """Every rank of the multi-GPU layer checks that all ranks hold the same
    plan before any peer store; a mismatch is refused on every rank."""
    world = len(Ns)
    mp.start_processes(_agree_worker, args=(world, _free_port(), Ns, str(tmp_path)), nprocs=world,
                       start_method="spawn")
    verdicts = [(tmp_path / f"agree{r}.txt").read_text() for r in range(world)]
    if expect_ok:
        assert verdicts == ["ok"] * world
    else:
        assert all(v.startswith("refused: plans differ across ranks: ranks [1]") for v in verdicts), verdicts


def _world_mismatch_worker(rank, world, port, result_dir):
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import peer
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        plan = U.ulysses_plan(1024, 8, 128, 4, 3)   # four ranks planned, two present
        try:
            peer.agree_plan(plan)
            verdict = "ok"
        except ValueError as e:
            verdict = "refused: " + str(e)
        with open(os.path.join(result_dir, f"world{rank}.txt"), "w") as f:
            f.write(verdict)
    finally:
        dist.destroy_process_group()


def test_group_size_must_match_the_plan(tmp_path):
    mp.start_processes(_world_mismatch_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, start_method="spawn")
    for r in range(2):
        assert (tmp_path / f"world{r}.txt").read_text() == "refused: the plan has P=4 ranks but the group has 2"


# ---- CollectiveLayer's multi-rank orchestration on CPU processes (gloo).
# The CUDA kernels are replaced by CPU stand-ins that compute what the C ABI
# documents (pack / unpack index maps, fp64 attention and its gradient per
# head), so the test checks the host side that only several ranks exercise:
# buffer shapes, chunk order of the exchanges, the plane loops, and the
# backward's sequence.  The stand-ins and the reference share the same
# per-head arithmetic, so the exchanged results must match bit for bit.

def _attn_heads_f64(q, k, v, N, scale):
    """[Np, Hl, D] each -> [Np, Hl, D] fp64; keys >= N masked, pad rows zero."""
    Np = q.shape[0]
    s = torch.einsum("nhd,mhd->hnm", q, k) * scale
    s[:, :, N:] = -float("inf")
    p = torch.softmax(s, dim=-1)
    o = torch.einsum("hnm,mhd->nhd", p, v)
    o[N:] = 0
    return o


def _fake_kernels(N):
    def pack(plan, src, planes, plane, send, stream=None):
        P, Nl, H = plan.P, plan.rows_per_rank, plan.H
        Hl = H // P
        send.view(P, Nl, Hl, 128).copy_(src.view(Nl, planes, P, Hl, 128)[:, plane].permute(1, 0, 2, 3))

    def unpack(plan, recv, out, planes, plane, stream=None):
        P, Nl, H = plan.P, plan.rows_per_rank, plan.H
        Hl = H // P
        out.view(Nl, planes, P, Hl, 128)[:, plane] = recv.view(P, Nl, Hl, 128).permute(1, 0, 2, 3)

    def fwd(plan, heads, out_heads, lse, scale, stream=None):
        q, k, v = (heads[c].double() for c in range(3))
        out_heads.copy_(_attn_heads_f64(q, k, v, N, scale).to(torch.bfloat16))

    def bwd(plan, heads, out_heads, dout_heads, lse, dqkv, ws, scale, stream=None):
        q, k, v = (heads[c].double().requires_grad_(True) for c in range(3))
        o = _attn_heads_f64(q, k, v, N, scale)
        o.backward(dout_heads[0].double())
        for c, t in enumerate((q, k, v)):
            dqkv[c].copy_(t.grad.to(torch.bfloat16))

    return pack, unpack, fwd, bwd


def _collective_worker(rank, world, port, N, H, C, result_dir):
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import peer
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        plan = U.ulysses_plan(N, H, 128, world, C)
        pack, unpack, fwd, bwd = _fake_kernels(N)
        peer.ulysses_a2a_pack, peer.ulysses_a2a_unpack = pack, unpack
        peer.ulysses_attn_fwd_lse_slab, peer.ulysses_attn_bwd_slab = fwd, bwd
        S, dO = torch.load(os.path.join(result_dir, "inputs.pt"))
        Nl = plan.rows_per_rank
        layer = peer.CollectiveLayer(plan, device=torch.device("cpu"), training=True)
        out = layer(S[rank * Nl:(rank + 1) * Nl].contiguous()).clone()
        grad = layer.backward(dO[rank * Nl:(rank + 1) * Nl].contiguous()).clone()
        torch.save((out, grad), os.path.join(result_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,N,H,C", [(2, 300, 4, 3), (4, 257, 8, 4)])
def test_collective_layer_orchestration(tmp_path, world, N, H, C):
    """CollectiveLayer over `world` CPU processes: every rank's output rows and
    Q/K/V gradient rows equal the whole layer computed in one process."""
    Np = -(-N // world) * world
    g = torch.Generator().manual_seed(world * 100 + N)
    S = torch.randn((Np, C, H, 128), generator=g).to(torch.bfloat16)
    S[N:] = 0
    dO = torch.randn((Np, H, 128), generator=g).to(torch.bfloat16)
    dO[N:] = 0
    torch.save((S, dO), tmp_path / "inputs.pt")
    mp.start_processes(_collective_worker, args=(world, _free_port(), N, H, C, str(tmp_path)), nprocs=world,
                       start_method="spawn")
    # the reference: all heads over the whole sequence in one process
    scale = 1.0 / np.sqrt(128)
    q, k, v = (S[:, c].double().requires_grad_(True) for c in range(3))
    o = _attn_heads_f64(q, k, v, N, scale)
    o.backward(dO.double())
    out_ref = o.detach().to(torch.bfloat16)
    grad_ref = torch.stack([t.grad.to(torch.bfloat16) for t in (q, k, v)], 1)    # [Np, 3, H, D]
    Nl = Np // world
    for r in range(world):
        out, grad = torch.load(tmp_path / f"rank{r}.pt")
        assert torch.equal(out.view(torch.int16), out_ref[r * Nl:(r + 1) * Nl].view(torch.int16)), f"rank {r} output"
        assert torch.equal(grad.view(torch.int16), grad_ref[r * Nl:(r + 1) * Nl].view(torch.int16)), f"rank {r} grad"
