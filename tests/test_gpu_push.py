"""The multi-GPU push calls with the P ranks emulated on one GPU, through the C ABI.

Every rank's buffer is its own allocation and every pointer table holds those
buffers, so the kernels address P separate destinations exactly as they would
peer mappings; each rank's launch is independent (no launch waits for
another), and the results are read after all of them.  The exchange computes
the Ulysses map itself, so the pushed slabs must equal the oracle's mode 0 /
mode 1 bit for bit, and the fused attention-push must equal the one-GPU layer
bit for bit (same kernel, same tile order per work unit), which the parity
suite holds to the fp64 oracle; one case is also checked against the oracle
here.
"""
import math

import numpy as np
import pytest
from _parity import check_attention

from oracle import ulysses_oracle as orc

pytestmark = pytest.mark.gpu

# (P, N, H, C, cu_seqlens, causal, seed)
CASES = [
    pytest.param(2, 1024, 8, 3, None, False, 60, id="tiny-P2"),
    pytest.param(4, 1001, 8, 3, None, False, 61, id="ragged-P4-N1001"),
    pytest.param(4, 777, 8, 4, None, False, 62, id="qkvg-P4-N777"),
    pytest.param(8, 2048, 16, 3, [0, 1024, 1536, 2048], False, 63, id="varlen-P8"),
    pytest.param(2, 1000, 4, 3, [0, 300, 300, 777, 1000], True, 64, id="causal-varlen-P2"),
    pytest.param(4, 5, 4, 3, None, False, 65, id="N5-P4"),
    pytest.param(1, 300, 2, 3, None, False, 66, id="P1"),
    pytest.param(56, 1000, 56, 3, None, False, 76, id="P56-Hl1"),
]


def _bits(t):
    from ulysses_sequence_attention_repack_b200 import inputs
    return inputs.host_bits(t)


def _setup(gpu, P, N, H, C, cu, causal, seed, deterministic=False):
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    plan = U.ulysses_plan(N, H, 128, P, C, 0, 0, 0, cu, causal=causal, deterministic=deterministic)
    Np, Nl, Hl = plan.padded_tokens, plan.rows_per_rank, H // P
    S = inputs.qkv_seq(N, H, P, C, seed, gpu)
    shards = [S[q * Nl:(q + 1) * Nl].clone() for q in range(P)]
    T = [torch.empty((C, Np, Hl, 128), dtype=torch.bfloat16, device=gpu) for _ in range(P)]
    for t in T:
        t.fill_(float("nan"))
    return plan, S, shards, T


@pytest.mark.parametrize("P,N,H,C,cu,causal,seed", CASES)
def test_push_exchange_and_fused_attention(gpu, P, N, H, C, cu, causal, seed):
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    plan, S, shards, T = _setup(gpu, P, N, H, C, cu, causal, seed)
    Np, Nl, Hl = plan.padded_tokens, plan.rows_per_rank, H // P
    scale = 1.0 / math.sqrt(128)
    # step 1: every rank pushes its shard into every rank's head slab
    for q in range(P):
        U.ulysses_repack_fwd_push(plan, q, shards[q], T)
    # steps 2 + 3: each rank's attention stores its rows into the owners' shards
    O = [torch.full((Nl, H, 128), float("nan"), dtype=torch.bfloat16, device=gpu) for _ in range(P)]
    for r in range(P):
        U.ulysses_attn_fwd_push(plan, r, T[r], O, scale)
    # the one-GPU layer on the same input
    OS = torch.empty((Np, H, 128), dtype=torch.bfloat16, device=gpu)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=gpu)
    U.ulysses_layer_fwd(plan, S, OS, ws, fused=0)
    torch.cuda.synchronize()
    assert U.ulysses_last_device_error(plan) == 0
    T_ref = orc.repack_fwd(_bits(S), P)
    for r in range(P):
        assert np.array_equal(_bits(T[r]), T_ref[r]), f"head slab of rank {r}"
    got = np.concatenate([_bits(o) for o in O], axis=0)
    assert np.array_equal(got, _bits(OS))


@pytest.mark.parametrize("P,N,H,C,cu,causal,seed", CASES)
def test_push_inverse_round_trip(gpu, P, N, H, C, cu, causal, seed):
    """Mode 1 pushed by every rank: all C planes back restores the shards, and
    the attention output plane gives the layer's output."""
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    plan, S, shards, T = _setup(gpu, P, N, H, C, cu, causal, seed)
    Np, Nl, Hl = plan.padded_tokens, plan.rows_per_rank, H // P
    for q in range(P):
        U.ulysses_repack_fwd_push(plan, q, shards[q], T)
    back = [torch.full((Nl, C, H, 128), float("nan"), dtype=torch.bfloat16, device=gpu) for _ in range(P)]
    for r in range(P):
        U.ulysses_repack_bwd_push(plan, r, T[r], back, C)
    # one plane: the head-sharded attention output of the one-GPU path
    Tg = torch.empty((P, C, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_repack_fwd(plan, S, Tg)
    OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_attn_fwd(plan, Tg, OT, 1.0 / math.sqrt(128))
    O1 = [torch.full((Nl, 1, H, 128), float("nan"), dtype=torch.bfloat16, device=gpu) for _ in range(P)]
    for r in range(P):
        U.ulysses_repack_bwd_push(plan, r, OT[r], O1, 1)
    torch.cuda.synchronize()
    assert U.ulysses_last_device_error(plan) == 0
    for q in range(P):
        assert np.array_equal(_bits(back[q]), _bits(shards[q])), f"shard of rank {q}"
    got = np.concatenate([_bits(o)[:, 0] for o in O1], axis=0)
    assert np.array_equal(got, orc.repack_bwd(_bits(OT)[:, None])[:, 0])


def test_push_attention_against_oracle(gpu):
    """The fused attention-push output against the fp64 oracle (the layer's
    max-abs 2e-2 / mean-abs 2e-3), pad rows exactly zero."""
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    P, N, H, C = 4, 1001, 8, 3
    plan, S, shards, T = _setup(gpu, P, N, H, C, None, False, 67)
    Nl = plan.rows_per_rank
    scale = 1.0 / math.sqrt(128)
    for q in range(P):
        U.ulysses_repack_fwd_push(plan, q, shards[q], T)
    O = [torch.empty((Nl, H, 128), dtype=torch.bfloat16, device=gpu) for _ in range(P)]
    for r in range(P):
        U.ulysses_attn_fwd_push(plan, r, T[r], O, scale)
    torch.cuda.synchronize()
    got = torch.cat(O, 0).float().cpu().numpy().astype(np.float64)
    ref = orc.layer_fwd(_bits(S), P, N, scale)
    check_attention(f"push layer P={P} N={N} H={H}", got[:N], ref[:N])
    assert np.all(got[N:] == 0)


_PEER_SCRIPT = r"""
import math, os, sys
import torch, torch.distributed as dist
sys.path.insert(0, os.getcwd())
import ulysses_sequence_attention_repack_b200 as U
from ulysses_sequence_attention_repack_b200 import inputs, peer
dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % int(sys.argv[1]), rank=0, world_size=1)
dev = torch.device("cuda", 0)
torch.cuda.set_device(dev)
N, H, C = 1000, 4, 3
plan = U.ulysses_plan(N, H, 128, 1, C, deterministic=True)   # gradients compared bit for bit
layer = peer.PeerLayer(plan)
S = inputs.qkv_seq(N, H, 1, C, 68, dev)
out = layer(S).clone()
ref = torch.empty((plan.padded_tokens, H, 128), dtype=torch.bfloat16, device=dev)
U.ulysses_layer_fwd(plan, S, ref, torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=dev), fused=0)
torch.cuda.synchronize()
assert U.ulysses_last_device_error(plan) == 0
assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), "peer layer differs from the one-GPU layer"
del layer
# training through autograd, against the one-GPU autograd layer
from ulysses_sequence_attention_repack_b200 import autograd as A
tl = peer.PeerLayer(plan, training=True)
g = torch.Generator(device=dev)
g.manual_seed(69)
dOut = torch.randn((plan.padded_tokens, H, 128), generator=g, device=dev).to(torch.bfloat16)
x = S.clone().requires_grad_(True)
y = peer.peer_ulysses_attention(x, tl)
y.backward(dOut)
x2 = S.clone().requires_grad_(True)
y2 = A.ulysses_attention(x2, plan)
y2.backward(dOut)
torch.cuda.synchronize()
assert U.ulysses_last_device_error(plan) == 0
assert torch.equal(y.view(torch.int16), y2.view(torch.int16)), "training forward differs"
assert torch.equal(x.grad.view(torch.int16), x2.grad.view(torch.int16)), "gradient differs"
del tl
# the all-to-all fallback (NCCL moves the bytes): the same output and gradient
cl = peer.CollectiveLayer(plan, training=True)
x3 = S.clone().requires_grad_(True)
y3 = peer.peer_ulysses_attention(x3, cl)
y3.backward(dOut)
torch.cuda.synchronize()
assert U.ulysses_last_device_error(plan) == 0
assert torch.equal(y3.view(torch.int16), y2.view(torch.int16)), "collective forward differs"
assert torch.equal(x3.grad.view(torch.int16), x2.grad.view(torch.int16)), "collective gradient differs"
del cl
dist.destroy_process_group()
print("peer-layer-ok")
"""


def test_peer_layer_one_rank_through_symmetric_memory(gpu):
    """PeerLayer end to end on a one-rank group (the only multi-process shape a
    one-GPU machine can run): symmetric-memory slabs, the push kernels and the
    barriers, equal to the one-GPU layer bit for bit; then a training step
    through autograd, output and input gradient equal to the one-GPU
    autograd layer's bit for bit, with PeerLayer and with the all-to-all
    fallback (CollectiveLayer, NCCL)."""
    import os
    import socket
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    r = subprocess.run([sys.executable, "-c", _PEER_SCRIPT, str(port)], cwd=root, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and "peer-layer-ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]


TRAIN_CASES = [
    pytest.param(2, 1024, 8, 3, None, False, 70, id="train-P2"),
    pytest.param(4, 1001, 8, 4, None, False, 71, id="train-ragged-qkvg-P4"),
    pytest.param(2, 1000, 4, 3, [0, 300, 300, 777, 1000], True, 72, id="train-causal-varlen-P2"),
]


@pytest.mark.parametrize("deterministic", [pytest.param(True, id="two-pass"), pytest.param(False, id="one-pass")])
@pytest.mark.parametrize("P,N,H,C,cu,causal,seed", TRAIN_CASES)
def test_push_training_path_equals_one_gpu_backward(gpu, P, N, H, C, cu, causal, seed, deterministic):
    """The multi-GPU training path with the ranks emulated: per-slab attention
    with lse, output pushed back, dO pushed into the slabs, the per-slab
    backward, gradients pushed to their owners.  Output, lse and gradients
    equal the one-GPU layer and ulysses_layer_bwd bit for bit with the
    deterministic backward; with the one-pass backward dK and dV still do, and
    dQ (summed by L2 reductions in a varying order) agrees to within
    rounding."""
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    plan, S, shards, T = _setup(gpu, P, N, H, C, cu, causal, seed, deterministic=deterministic)
    Np, Nl, Hl = plan.padded_tokens, plan.rows_per_rank, H // P
    scale = 1.0 / math.sqrt(128)
    g = torch.Generator(device=gpu)
    g.manual_seed(seed + 1000)
    dOut = torch.randn((Np, H, 128), generator=g, device=gpu).to(torch.bfloat16)
    dOut[N:] = 0
    # forward
    for q in range(P):
        U.ulysses_repack_fwd_push(plan, q, shards[q], T)
    OTr = [torch.empty((Np, Hl, 128), dtype=torch.bfloat16, device=gpu) for _ in range(P)]
    lser = [torch.empty(plan.slab_lse_bytes // 4, dtype=torch.float32, device=gpu) for _ in range(P)]
    O = [torch.full((Nl, H, 128), float("nan"), dtype=torch.bfloat16, device=gpu) for _ in range(P)]
    for r in range(P):
        U.ulysses_attn_fwd_lse_slab(plan, T[r], OTr[r], lser[r], scale)
        U.ulysses_repack_bwd_push(plan, r, OTr[r], O, 1)
    # backward
    dOs = [dOut[q * Nl:(q + 1) * Nl].clone() for q in range(P)]
    dOT = [torch.full((1, Np, Hl, 128), float("nan"), dtype=torch.bfloat16, device=gpu) for _ in range(P)]
    for q in range(P):
        U.ulysses_repack_fwd_push(plan, q, dOs[q], dOT, 1)
    dq = [torch.empty((3, Np, Hl, 128), dtype=torch.bfloat16, device=gpu) for _ in range(P)]
    G = [torch.full((Nl, 3, H, 128), float("nan"), dtype=torch.bfloat16, device=gpu) for _ in range(P)]
    for r in range(P):
        ws = torch.empty(plan.slab_attn_bwd_workspace_bytes, dtype=torch.uint8, device=gpu)
        U.ulysses_attn_bwd_slab(plan, T[r], OTr[r], dOT[r], lser[r], dq[r], ws, scale)
        U.ulysses_repack_bwd_push(plan, r, dq[r], G, 3)
    # the one-GPU path
    Tg = torch.empty((P, C, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    lse = torch.empty(plan.lse_bytes // 4, dtype=torch.float32, device=gpu)
    U.ulysses_repack_fwd(plan, S, Tg)
    U.ulysses_attn_fwd_lse(plan, Tg, OT, lse, scale)
    OS = torch.empty((Np, H, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_repack_bwd(plan, OT, OS, 1)
    dS = torch.zeros_like(S)
    wsl = torch.empty(plan.layer_bwd_workspace_bytes, dtype=torch.uint8, device=gpu)
    U.ulysses_layer_bwd(plan, Tg, OT, lse, dOut, dS, wsl)
    torch.cuda.synchronize()
    assert U.ulysses_last_device_error(plan) == 0
    assert np.array_equal(np.concatenate([_bits(o) for o in O], 0), _bits(OS))
    stride = plan.lse_row_stride
    lse_h = lse.cpu().numpy().reshape(P, Hl, stride)[:, :, :Np]     # entries past Np are never written
    for r in range(P):
        mine = lser[r].cpu().numpy().reshape(Hl, stride)[:, :Np]
        assert np.array_equal(mine, lse_h[r]), f"lse of rank {r}"
        assert np.array_equal(_bits(OTr[r]), _bits(OT[r])), f"output slab of rank {r}"
    got = np.concatenate([_bits(x) for x in G], 0)
    want = _bits(dS)[:, :3]
    if deterministic:
        assert np.array_equal(got, want)
    else:
        assert np.array_equal(got[:, 1:], want[:, 1:])
        x = torch.cat(G, 0)[:, 0].double()
        y = dS[:, 0].double()
        tol = 2.0 ** -7 * torch.maximum(x.abs(), y.abs()) + 1e-6 * y.abs().max()
        assert ((x - y).abs() <= tol).all()


@pytest.mark.parametrize("P,N,H,C,seed", [pytest.param(4, 1001, 8, 3, 73, id="P4-N1001"),
                                          pytest.param(2, 777, 4, 4, 74, id="P2-qkvg"),
                                          pytest.param(8, 2048, 16, 3, 75, id="P8")])
def test_all_to_all_pack_unpack(gpu, P, N, H, C, seed):
    """The all-to-all fallback's kernels, with the collective emulated by
    moving the equal-split chunks between the ranks' buffers: the head slabs
    equal the oracle's mode 0 bit for bit, the unpacked output equals the
    one-GPU layer's rows, and a three-plane unpack lands in its plane."""
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    plan, S, shards, _ = _setup(gpu, P, N, H, C, None, False, seed)
    Np, Nl, Hl = plan.padded_tokens, plan.rows_per_rank, H // P
    send = [[torch.empty((P, Nl, Hl, 128), dtype=torch.bfloat16, device=gpu) for _ in range(C)] for _ in range(P)]
    for q in range(P):
        for c in range(C):
            U.ulysses_a2a_pack(plan, shards[q], C, c, send[q][c])
    # the exchange: rank r receives chunk r of every rank's send buffer, in rank order
    heads = [torch.stack([torch.cat([send[q][c][r] for q in range(P)], 0) for c in range(C)], 0) for r in range(P)]
    Tg = torch.empty((P, C, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_repack_fwd(plan, S, Tg)
    OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_attn_fwd(plan, Tg, OT, 1.0 / math.sqrt(128))
    OS = torch.empty((Np, H, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_repack_bwd(plan, OT, OS, 1)
    outs, three = [], []
    for q in range(P):
        recv = torch.stack([OT[r, q * Nl:(q + 1) * Nl] for r in range(P)], 0).contiguous()
        o = torch.full((Nl, H, 128), float("nan"), dtype=torch.bfloat16, device=gpu)
        U.ulysses_a2a_unpack(plan, recv, o, 1, 0)
        g = torch.zeros((Nl, 3, H, 128), dtype=torch.bfloat16, device=gpu)
        U.ulysses_a2a_unpack(plan, recv, g, 3, 1)
        outs.append(o)
        three.append(g)
    torch.cuda.synchronize()
    assert U.ulysses_last_device_error(plan) == 0
    T_ref = orc.repack_fwd(_bits(S), P)
    for r in range(P):
        assert np.array_equal(_bits(heads[r]), T_ref[r]), f"head slab of rank {r}"
    assert np.array_equal(np.concatenate([_bits(o) for o in outs], 0), _bits(OS))
    for q in range(P):
        g = _bits(three[q])
        assert np.array_equal(g[:, 1], _bits(outs[q])) and not g[:, 0].any() and not g[:, 2].any()
