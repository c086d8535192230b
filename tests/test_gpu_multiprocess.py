"""PeerLayer with its ranks as separate processes sharing one GPU.

Each rank is its own process with its own CUDA context, as on P GPUs: its
buffers are ordinary allocations, the peers' addresses come from CUDA IPC
handles exchanged over a gloo group (``PeerLayer(exchange="ipc")``), the
push kernels store through those mappings, and every barrier is a host
barrier after a stream synchronisation, so no kernel waits on another
process's kernel.  The gathered output shards (and, in training mode, the
input-gradient shards) must equal the one-GPU layer (and
``ulysses_layer_bwd``) bit for bit; the one-GPU layer is checked against the
oracle elsewhere.  This exercises the cross-process address exchange, the
ordering of the exchange and the per-rank launch sequence with P >= 2.
"""
import math
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_RANK = r"""
import datetime, math, os, sys
import numpy as np
import torch
import torch.distributed as dist
root, rank, world, port, out_path = sys.argv[1], int(sys.argv[2]), int(sys.argv[3]), int(sys.argv[4]), sys.argv[5]
N, H, C, seed, training = int(sys.argv[6]), int(sys.argv[7]), int(sys.argv[8]), int(sys.argv[9]), sys.argv[10] == "1"
sys.path.insert(0, root)
dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                        timeout=datetime.timedelta(seconds=120))
torch.cuda.set_device(0)
dev = torch.device("cuda", 0)
import ulysses_sequence_attention_repack_b200 as U
from ulysses_sequence_attention_repack_b200 import inputs, peer
plan = U.ulysses_plan(N, H, 128, world, C, deterministic=True)   # gradients compared bit for bit
Nl = plan.rows_per_rank
S = inputs.qkv_seq(N, H, world, C, seed, dev)
shard = S[rank * Nl:(rank + 1) * Nl].contiguous()
layer = peer.PeerLayer(plan, exchange="ipc", training=training)
res = {"out": layer(shard).clone().view(torch.int16).cpu().numpy()}
if training:
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 1000)
    dout = torch.randn((plan.padded_tokens, H, 128), generator=g, device=dev).to(torch.bfloat16)
    dout[N:] = 0
    res["grad"] = layer.backward(dout[rank * Nl:(rank + 1) * Nl].contiguous()).clone().view(torch.int16).cpu().numpy()
torch.cuda.synchronize()
res["err"] = np.array([U.ulysses_last_device_error(plan)])
np.savez(out_path, **res)
del layer                      # close the IPC mappings before any rank exits
torch.cuda.synchronize()
dist.barrier()
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_ranks(tmp_path, P, N, H, C, seed, training):
    script = tmp_path / "rank.py"
    script.write_text(_RANK)
    port = _free_port()
    env = dict(os.environ)
    env.pop("ULYSSES_LIBRARY", None)
    procs = []
    for r in range(P):
        procs.append(subprocess.Popen(
            [sys.executable, str(script), ROOT, str(r), str(P), str(port), str(tmp_path / f"r{r}.npz"), str(N),
             str(H), str(C), str(seed), "1" if training else "0"],
            env=env, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True))
    logs = []
    for pr in procs:
        try:
            out, _ = pr.communicate(timeout=300)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            raise
        logs.append(out)
    for r, pr in enumerate(procs):
        assert pr.returncode == 0, f"rank {r} failed:\n{logs[r][-3000:]}"
    return [dict(np.load(tmp_path / f"r{r}.npz")) for r in range(P)]


@pytest.mark.parametrize("P,N,H,C,seed", [pytest.param(2, 1001, 8, 3, 120, id="P2-ragged"),
                                          pytest.param(4, 2053, 8, 4, 121, id="P4-qkvg")])
def test_ranks_as_processes_equal_one_gpu_layer(gpu, tmp_path, P, N, H, C, seed):
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    ranks = _run_ranks(tmp_path, P, N, H, C, seed, training=False)
    plan = U.ulysses_plan(N, H, 128, P, C)
    S = inputs.qkv_seq(N, H, P, C, seed, gpu)
    OS = torch.empty((plan.padded_tokens, H, 128), dtype=torch.bfloat16, device=gpu)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=gpu)
    U.ulysses_layer_fwd(plan, S, OS, ws, fused=0)
    torch.cuda.synchronize()
    assert all(int(r["err"][0]) == 0 for r in ranks)
    got = np.concatenate([r["out"] for r in ranks], axis=0)
    assert np.array_equal(got, OS.view(torch.int16).cpu().numpy())


def test_training_ranks_as_processes_equal_one_gpu_backward(gpu, tmp_path):
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    P, N, H, C, seed = 2, 1001, 8, 3, 122
    ranks = _run_ranks(tmp_path, P, N, H, C, seed, training=True)
    plan = U.ulysses_plan(N, H, 128, P, C, deterministic=True)
    Np, Hl = plan.padded_tokens, H // P
    scale = 1.0 / math.sqrt(128)
    S = inputs.qkv_seq(N, H, P, C, seed, gpu)
    g = torch.Generator(device=gpu)
    g.manual_seed(seed + 1000)
    dout = torch.randn((Np, H, 128), generator=g, device=gpu).to(torch.bfloat16)
    dout[N:] = 0
    T = torch.empty((P, C, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    lse = torch.empty(plan.lse_bytes // 4, dtype=torch.float32, device=gpu)
    U.ulysses_repack_fwd(plan, S, T)
    U.ulysses_attn_fwd_lse(plan, T, OT, lse, scale)
    OS = torch.empty((Np, H, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_repack_bwd(plan, OT, OS, 1)
    dS = torch.zeros_like(S)
    ws = torch.empty(plan.layer_bwd_workspace_bytes, dtype=torch.uint8, device=gpu)
    U.ulysses_layer_bwd(plan, T, OT, lse, dout, dS, ws)
    torch.cuda.synchronize()
    assert all(int(r["err"][0]) == 0 for r in ranks)
    assert np.array_equal(np.concatenate([r["out"] for r in ranks], 0), OS.view(torch.int16).cpu().numpy())
    want = dS[:, :3].contiguous().view(torch.int16).cpu().numpy()
    assert np.array_equal(np.concatenate([r["grad"] for r in ranks], 0), want)
