"""NVTX ranges of the C ABI, recorded by a test-only NVTX injection library
(tests/nvtx_recorder.c) that NVTX loads through NVTX_INJECTION64_PATH.

On the CPU every launching entry point opens its range before it validates
its arguments, so calls refused for lack of a device still record their
names.  On the GPU the unfused layer call shows its three steps nested in
it: repack_fwd, attention, repack_bwd.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_SCRIPT = r"""
import ctypes, math, os, sys
sys.path.insert(0, sys.argv[1])
import ulysses_sequence_attention_repack_b200 as U
plan = U.ulysses_plan(1024, 8, 128, 2, 3)
gpu = sys.argv[2] == "gpu"
if gpu:
    import torch
    from ulysses_sequence_attention_repack_b200 import inputs
    dev = torch.device("cuda", 0)
    S = inputs.qkv_seq(1024, 8, 2, 3, 0, dev)
    out = torch.empty((1024, 8, 128), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=dev)
    U.ulysses_layer_fwd(plan, S, out, ws, fused=0)
    U.ulysses_layer_fwd(plan, S, out, None, fused=1)
    torch.cuda.synchronize()
else:
    for call in (lambda: U.ulysses_repack_fwd(plan, None, None), lambda: U.ulysses_attn_fwd(plan, None, None, 0.1),
                 lambda: U.ulysses_repack_bwd(plan, None, None, 1), lambda: U.ulysses_layer_fwd(plan, None, None, None)):
        try:
            call()
        except U.UlyssesError:
            pass
rec = ctypes.CDLL(os.environ["NVTX_INJECTION64_PATH"])
rec.nvtx_recorded.restype = ctypes.c_char_p
sys.stdout.write(rec.nvtx_recorded().decode())
"""


def _recorder(tmp_path):
    gcc = shutil.which("gcc") or shutil.which("cc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib = tmp_path / "libnvtx_recorder.so"
    subprocess.run([gcc, "-shared", "-fPIC", "-O1", "-I", "/usr/local/cuda/include",
                    os.path.join(ROOT, "tests", "nvtx_recorder.c"), "-o", str(lib)], check=True)
    return str(lib)


def _record(tmp_path, mode):
    env = dict(os.environ, NVTX_INJECTION64_PATH=_recorder(tmp_path))
    env.pop("ULYSSES_LIBRARY", None)
    r = subprocess.run([sys.executable, "-c", _SCRIPT, ROOT, mode], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return r.stdout.splitlines()


def test_entry_points_open_named_ranges(tmp_path):
    lines = _record(tmp_path, "cpu")
    for name in ("ulysses_repack_fwd", "ulysses_attn_fwd", "ulysses_repack_bwd", "ulysses_layer_fwd"):
        assert f"ulysses/{name}" in lines, (name, lines)


@pytest.mark.gpu
def test_layer_steps_nest_inside_the_layer_range(gpu, tmp_path):
    lines = _record(tmp_path, "gpu")
    i = lines.index("ulysses/ulysses_layer_fwd")
    assert lines[i + 1:i + 4] == ["ulysses/repack_fwd", "ulysses/attention", "ulysses/repack_bwd"], lines
    j = lines.index("ulysses/ulysses_layer_fwd", i + 1)
    assert lines[j + 1] == "ulysses/fused attention", lines
