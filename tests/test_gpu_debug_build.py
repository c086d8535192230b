"""The bounds-checked build (libulysses_debug.so, compiled with -DULYSSES_DEBUG).

In that build every global access of the repack, prologue and push kernels,
and every store of the attention epilogues and of the backward (its dK/dV
stores and dQ reduce-adds), checks that it lies inside the buffer the launch
geometry describes; an access outside is skipped and bit 4 of the device
error word is set.  It stands in for a memory checker on this GPU.  Here the
debug library runs the tiny and ragged workloads through every kernel family
with the error word staying zero and outputs equal, bit for bit, to the
default library's (for the one-pass backward, whose dQ is summed in a
varying order, dK and dV).  The check itself is exercised by a self-test hook
that touches no memory.
"""
import os
import subprocess
import sys

import _selftest_lib
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# Every kernel family on one geometry; prints nothing, saves the outputs and
# the error word of each call sequence to the .npz named on the command line.
_SCRIPT = r"""
import math, sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[3])
import ulysses_sequence_attention_repack_b200 as U
from ulysses_sequence_attention_repack_b200 import inputs
P, N, H, C = [int(x) for x in sys.argv[2].split(",")]
dev = torch.device("cuda", 0)
torch.cuda.set_device(dev)
plan = U.ulysses_plan(N, H, 128, P, C)
Np, Hl, Nl = plan.padded_tokens, H // P, plan.rows_per_rank
scale = 1.0 / math.sqrt(128)
S = inputs.qkv_seq(N, H, P, C, 90, dev)
out = {}
T = torch.empty((P, C, Np, Hl, 128), dtype=torch.bfloat16, device=dev)
OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=dev)
OS = torch.empty((Np, H, 128), dtype=torch.bfloat16, device=dev)
OSf = torch.empty_like(OS)
back = torch.empty_like(S)
U.ulysses_repack_fwd(plan, S, T)
U.ulysses_attn_fwd(plan, T, OT, scale)
U.ulysses_repack_bwd(plan, OT, OS, 1)
U.ulysses_repack_bwd(plan, T, back, C)
U.ulysses_layer_fwd(plan, S, OSf, None, fused=1)
T8 = torch.empty((P, C, Np, Hl, 128), dtype=torch.uint8, device=dev)
U.ulysses_repack_fwd_fp8(plan, S, T8)
g = torch.Generator(device=dev)
g.manual_seed(91)
wq = torch.randn(128, generator=g, device=dev).to(torch.bfloat16)
wk = torch.randn(128, generator=g, device=dev).to(torch.bfloat16)
ang = torch.rand((Np, 48), generator=g, device=dev)
cos_t = torch.cat([torch.cos(ang), torch.cos(ang)], 1).to(torch.bfloat16).contiguous()
sin_t = torch.cat([torch.sin(ang), torch.sin(ang)], 1).to(torch.bfloat16).contiguous()
Tp = torch.empty_like(T)
U.ulysses_prologue_repack_fwd(plan, S, Tp, wq, wk, cos_t, sin_t, 96, 1e-5)
slabs = [torch.empty((C, Np, Hl, 128), dtype=torch.bfloat16, device=dev) for _ in range(P)]
for q in range(P):
    U.ulysses_repack_fwd_push(plan, q, S[q * Nl:(q + 1) * Nl], slabs)
shards = [torch.empty((Nl, H, 128), dtype=torch.bfloat16, device=dev) for _ in range(P)]
for r in range(P):
    U.ulysses_attn_fwd_push(plan, r, slabs[r], shards, scale)
back_push = [torch.empty((Nl, 1, H, 128), dtype=torch.bfloat16, device=dev) for _ in range(P)]
for r in range(P):
    U.ulysses_repack_bwd_push(plan, r, OT[r], back_push, 1)
# attention backward in both forms (the one-pass dQ sums in a varying order:
# its dK and dV are compared, and all of the deterministic form's output)
lse = torch.empty(plan.lse_bytes // 4, dtype=torch.float32, device=dev)
U.ulysses_attn_fwd_lse(plan, T, OT, lse, scale)
g.manual_seed(92)
dO = torch.randn(OT.shape, generator=g, device=dev).to(torch.bfloat16)
dO[:, N:] = 0
dT = torch.empty((P, 3, Np, Hl, 128), dtype=torch.bfloat16, device=dev)
U.ulysses_attn_bwd(plan, T, OT, dO, lse, dT, torch.empty(plan.attn_bwd_workspace_bytes, dtype=torch.uint8,
                                                          device=dev), scale)
dplan = U.ulysses_plan(N, H, 128, P, C, deterministic=True)
dTd = torch.empty_like(dT)
U.ulysses_attn_bwd(dplan, T, OT, dO, lse, dTd, torch.empty(dplan.attn_bwd_workspace_bytes, dtype=torch.uint8,
                                                            device=dev), scale)
torch.cuda.synchronize()
out["err"] = np.array([U.ulysses_last_device_error(plan) | U.ulysses_last_device_error(dplan)])
for name, t in (("T", T), ("OT", OT), ("OS", OS), ("OSf", OSf), ("back", back), ("T8", T8), ("Tp", Tp),
                ("slabs", torch.stack(slabs)), ("shards", torch.cat(shards)), ("back_push", torch.cat(back_push)),
                ("dKV_one_pass", dT[:, 1:]), ("dQKV_two_pass", dTd)):
    out[name] = t.contiguous().view(torch.uint8).cpu().numpy()
np.savez(sys.argv[1], **out)
"""


def _run(tmp_path, lib, geom, tag):
    path = tmp_path / f"{tag}.npz"
    script = tmp_path / "run.py"
    script.write_text(_SCRIPT)
    env = dict(os.environ)
    if lib:
        env["ULYSSES_LIBRARY"] = lib
    else:
        env.pop("ULYSSES_LIBRARY", None)
    r = subprocess.run([sys.executable, str(script), str(path), ",".join(map(str, geom)), ROOT], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    return dict(np.load(path))


@pytest.mark.parametrize("geom", [pytest.param((2, 1024, 8, 3), id="tiny"),
                                  pytest.param((4, 1001, 8, 4), id="ragged-qkvg")])
def test_debug_build_runs_clean_and_matches(gpu, tmp_path, geom):
    from ulysses_sequence_attention_repack_b200 import build
    debug_lib = build.ensure_debug_built()
    got = _run(tmp_path, debug_lib, geom, "debug")
    want = _run(tmp_path, None, geom, "release")
    assert int(got["err"][0]) == 0, hex(int(got["err"][0]))      # no access fell outside its buffer
    assert int(want["err"][0]) == 0
    for name in want:
        assert np.array_equal(got[name], want[name]), name


def test_range_check_refuses_and_reports(gpu):
    import torch
    err = torch.zeros(4, dtype=torch.int32, device=gpu)
    lib = _selftest_lib.load()
    assert lib.ulysses_selftest_bounds_check(err.data_ptr(), torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert int(err[0].item()) == 4 | 0x10 | 0x20 | 0x40, hex(int(err[0].item()))
