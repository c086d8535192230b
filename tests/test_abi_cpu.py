"""Host-side tests of the C ABI (no GPU needed: nothing here launches a kernel)."""
import os
import re

import pytest

import ulysses_sequence_attention_repack_b200 as U
from oracle import ulysses_oracle as orc
from ulysses_sequence_attention_repack_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols(header="ulysses.h"):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ulysses_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = U.load()
    syms = declared_symbols()
    assert len(syms) >= 14
    for name in syms:
        assert hasattr(lib, name), name
    assert set(syms) == set(U.EXPORTS)


def test_test_hooks_live_outside_the_product_library():
    """include/ulysses_selftest.h is served by libulysses_selftest.so alone."""
    import ctypes

    import _selftest_lib
    hooks = declared_symbols("ulysses_selftest.h")
    assert set(hooks) == set(_selftest_lib.SELFTEST_EXPORTS)
    lib = U.load()
    test_lib = _selftest_lib.load()
    for name in hooks:
        assert hasattr(test_lib, name), name
        with pytest.raises(AttributeError):
            getattr(ctypes.CDLL(U.library_path()), name)
    assert not set(hooks) & set(U.EXPORTS)
    assert lib is not None


def test_library_built_for_sm100a():
    # the build passes exactly one gencode target: sm_100a
    from ulysses_sequence_attention_repack_b200 import build
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert os.path.exists(U.library_path())


def _code(**kw):
    args = dict(N=1024, H=8, D=128, P=2, planes=3, token_stride=0, plane_stride=0, plane_chunk=0, cu_seqlens=None)
    args.update(kw)
    try:
        U.ulysses_plan(**args)
        return 0
    except U.UlyssesError as e:
        return e.code


def test_plan_flags():
    import ctypes
    lib = U.load()
    h = ctypes.c_void_p()
    for flags, want in ((0, 0), (_lib.ULYSSES_PLAN_CAUSAL, 0), (_lib.ULYSSES_PLAN_PAIR_ATTENTION, 0),
                        (_lib.ULYSSES_PLAN_CAUSAL | _lib.ULYSSES_PLAN_PAIR_ATTENTION, 0),
                        (_lib.ULYSSES_PLAN_DETERMINISTIC, 0), (7, 0), (8, _lib.ULYSSES_ERR_ARG)):
        code = lib.ulysses_plan_ex(ctypes.byref(h), 1024, 8, 128, 2, 3, 0, 0, 0, None, 0, flags)
        assert code == want, (flags, code)
        if code == 0:
            lib.ulysses_plan_destroy(h)


def test_plan_validation_codes():
    assert _code() == _lib.ULYSSES_OK
    assert _code(D=64) == _lib.ULYSSES_ERR_UNSUPPORTED
    assert _code(H=6, P=4) == _lib.ULYSSES_ERR_DIVISIBILITY
    assert _code(P=16) == _lib.ULYSSES_ERR_DIVISIBILITY          # more ranks than heads
    assert _code(P=0) == _lib.ULYSSES_ERR_ARG
    assert _code(N=0) == _lib.ULYSSES_ERR_ARG
    assert _code(planes=0) == _lib.ULYSSES_ERR_ARG
    assert _code(planes=9) == _lib.ULYSSES_ERR_ARG
    assert _code(token_stride=3 * 8 * 128 + 4, plane_stride=8 * 128) == _lib.ULYSSES_ERR_ALIGN
    assert _code(token_stride=8 * 128, plane_stride=8 * 128) == _lib.ULYSSES_ERR_ARG   # planes overlap
    # one plane per rank above 1 GiB: 400,000 tokens x 56 heads at SP 4
    assert _code(N=400_000, H=56, P=4) == _lib.ULYSSES_ERR_WINDOW
    # a chunk of two 896,000,000-byte planes exceeds the window
    assert _code(N=250_000, H=56, P=4, planes=4, plane_chunk=2) == _lib.ULYSSES_ERR_WINDOW
    assert _code(plane_chunk=4) == _lib.ULYSSES_ERR_ARG
    # cu_seqlens: must start at 0, end at N, never decrease
    assert _code(N=10, P=2, H=2, cu_seqlens=[0, 5, 10]) == _lib.ULYSSES_OK
    assert _code(N=10, P=2, H=2, cu_seqlens=[1, 5, 10]) == _lib.ULYSSES_ERR_ARG
    assert _code(N=10, P=2, H=2, cu_seqlens=[0, 5, 9]) == _lib.ULYSSES_ERR_ARG
    assert _code(N=10, P=2, H=2, cu_seqlens=[0, 6, 5, 10]) == _lib.ULYSSES_ERR_ARG
    assert _code(N=65, P=1, H=1, cu_seqlens=list(range(66))) == _lib.ULYSSES_ERR_UNSUPPORTED


@pytest.mark.parametrize("N,H,P,C", [(19_394, 56, 4, 3), (38_912, 56, 4, 4), (104_448, 56, 8, 3),
                                     (250_000, 56, 4, 4), (32_000, 56, 4, 4), (1024, 8, 2, 3), (5, 4, 4, 3)])
def test_plan_sizes_agree_with_oracle(N, H, P, C):
    plan = U.ulysses_plan(N, H, 128, P, C)
    assert plan.padded_tokens == orc.padded_tokens(N, P)
    assert plan.window_bytes_per_plane == orc.plane_bytes_per_rank(N, H, 128, P)
    assert plan.plane_chunk == orc.auto_plane_chunk(N, H, 128, P, C)
    Np, Hl = orc.padded_tokens(N, P), H // P

    def up(x):
        return (x + 255) // 256 * 256
    assert plan.workspace_bytes == up(P * C * Np * Hl * 128 * 2) + up(P * Np * Hl * 128 * 2)


@pytest.mark.parametrize("N,H,P", [(19_394, 56, 4), (104_448, 56, 8), (1024, 8, 2), (5, 4, 4), (300, 2, 1),
                                   (4, 56, 56)])
def test_backward_workspace_sizes(N, H, P):
    """The deterministic backward needs the two row-term arrays; the one-pass
    form adds the fp32 dQ accumulator [P*Hl][Np][D] after them, placed so that
    a rank's slab workspace (ulysses_attn_bwd_slab) is exactly 1/P of the
    whole; the layer backward's workspace grows by the same amount."""
    det = U.ulysses_plan(N, H, 128, P, 3, deterministic=True)
    one = U.ulysses_plan(N, H, 128, P, 3)
    Np, Hl = orc.padded_tokens(N, P), H // P
    rows = 2 * det.lse_bytes
    assert det.attn_bwd_workspace_bytes == rows
    acc = P * Hl * Np * 128 * 4
    want = (rows + 256 * P - 1) // (256 * P) * (256 * P) + acc
    assert one.attn_bwd_workspace_bytes == want
    assert want % P == 0 and (want // P) % 256 == 0
    # a rank's slab is the same problem on one rank with Hl heads
    slab_rows = 2 * (det.lse_bytes // P)
    assert one.slab_attn_bwd_workspace_bytes == (slab_rows + 255) // 256 * 256 + Hl * Np * 128 * 4

    def up(x):
        return (x + 255) // 256 * 256
    for plan in (det, one):
        assert plan.layer_bwd_workspace_bytes == (up(P * Np * Hl * 128 * 2) + up(3 * P * Np * Hl * 128 * 2) +
                                                  up(plan.attn_bwd_workspace_bytes))


def test_window_bytes_printed_on_the_pages():
    # 250,000 tokens, 56 heads, head dim 128, SP 4: 896,000,000 bytes per plane, one plane per launch
    plan = U.ulysses_plan(250_000, 56, 128, 4, 4)
    assert plan.window_bytes_per_plane == 896_000_000
    assert plan.plane_chunk == 1


def test_launch_argument_checks_before_any_device_work():
    plan = U.ulysses_plan(1024, 8, 128, 2, 3)
    lib = U.load()
    h = plan.handle
    # null pointers
    assert lib.ulysses_repack_fwd(h, None, 0x10000, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_attn_fwd(h, 0x10000, None, 0.1, None) == _lib.ULYSSES_ERR_ARG
    # misaligned pointers
    assert lib.ulysses_repack_fwd(h, 0x10008, 0x90000000, None) == _lib.ULYSSES_ERR_ALIGN
    assert lib.ulysses_repack_bwd(h, 0x10000, 0x90000004, 1, None) == _lib.ULYSSES_ERR_ALIGN
    # overlapping input and output
    assert lib.ulysses_repack_fwd(h, 0x10000, 0x10000 + 4096, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_attn_fwd(h, 0x10000, 0x10000, 0.1, None) == _lib.ULYSSES_ERR_ARG
    # bad scale and plane count
    assert lib.ulysses_attn_fwd(h, 0x10000, 0x90000000, -1.0, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_repack_bwd(h, 0x10000, 0x90000000, 4, None) == _lib.ULYSSES_ERR_ARG
    # layer: missing or short workspace, bad fused flag
    assert lib.ulysses_layer_fwd(h, 0x10000, 0x90000000, None, 0, 0, None) == _lib.ULYSSES_ERR_WORKSPACE
    assert lib.ulysses_layer_fwd(h, 0x10000, 0x90000000, 0xA0000000, 16, 0, None) == _lib.ULYSSES_ERR_WORKSPACE
    assert lib.ulysses_layer_fwd(h, 0x10000, 0x90000000, None, 0, 2, None) == _lib.ULYSSES_ERR_ARG
    # host-buffer layer: same checks, made before any stream or copy is created
    hl = lib.ulysses_layer_fwd_host
    assert hl(h, None, 0x20000000, 0x10000, 0x90000000, None, 0, 1, None) == _lib.ULYSSES_ERR_ARG
    assert hl(h, 0x30000000, 0x20000000, 0x10000, 0x90000000, None, 0, 0, None) == _lib.ULYSSES_ERR_WORKSPACE
    assert hl(h, 0x30000000, 0x20000000, 0x10008, 0x90000000, None, 0, 1, None) == _lib.ULYSSES_ERR_ALIGN
    assert hl(h, 0x30000000, 0x30000000, 0x10000, 0x90000000, None, 0, 1, None) == _lib.ULYSSES_ERR_ARG
    assert hl(h, 0x30000000, 0x20000000, 0x10000, 0x10000, None, 0, 1, None) == _lib.ULYSSES_ERR_ARG
    assert hl(h, 0x30000000, 0x20000000, 0x10000, 0x90000000, None, 0, 3, None) == _lib.ULYSSES_ERR_ARG
    # FP8 variant
    assert lib.ulysses_repack_fwd_fp8(h, None, 0x10000, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_repack_fwd_fp8(h, 0x10008, 0x90000000, None) == _lib.ULYSSES_ERR_ALIGN
    assert lib.ulysses_repack_fwd_fp8(h, 0x10000, 0x10000 + 4096, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_attn_fwd_fp8(h, 0x10000, 0x10000, 0.1, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_attn_fwd_fp8(h, 0x10000, 0x90000000, 0.0, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_layer_fwd_fp8(h, 0x10000, 0x90000000, None, 0, None) == _lib.ULYSSES_ERR_WORKSPACE
    fh = lib.ulysses_layer_fwd_fp8_host
    assert fh(h, 0x30000000, 0x20000000, 0x10000, 0x90000000, None, 0, None) == _lib.ULYSSES_ERR_WORKSPACE
    assert fh(h, 0x30000000, 0x20000000, 0x10008, 0x90000000, None, 0, None) == _lib.ULYSSES_ERR_ALIGN
    assert fh(h, None, 0x20000000, 0x10000, 0x90000000, None, 0, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_workspace_bytes_fp8(h) == ((1024 * 3 * 8 * 128 + 255) // 256 * 256 + 1024 * 8 * 128 * 2)
    # a gate-less plan cannot run attention
    p2 = U.ulysses_plan(1024, 8, 128, 2, 2)
    assert lib.ulysses_attn_fwd(p2.handle, 0x10000, 0x90000000, 0.1, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_attn_fwd_fp8(p2.handle, 0x10000, 0x90000000, 0.1, None) == _lib.ULYSSES_ERR_ARG


def test_push_argument_checks_before_any_device_work():
    """The multi-GPU push calls validate rank, pointer tables, alignment,
    overlap and the shard layout before touching a device; a valid call on a
    machine without a GPU reports ULYSSES_ERR_CUDA."""
    import ctypes
    lib = U.load()
    plan = U.ulysses_plan(1024, 8, 128, 2, 3)
    h = plan.handle
    assert plan.rows_per_rank == 512

    def table(*ptrs):
        return (ctypes.c_void_p * len(ptrs))(*ptrs)

    good = table(0x40000000, 0x50000000)
    ok_codes = (_lib.ULYSSES_ERR_CUDA,)
    assert lib.ulysses_repack_fwd_push(h, 0, 0x10000, good, 3, None) in ok_codes
    assert lib.ulysses_repack_fwd_push(h, 2, 0x10000, good, 3, None) == _lib.ULYSSES_ERR_ARG       # rank >= P
    assert lib.ulysses_repack_fwd_push(h, -1, 0x10000, good, 3, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_repack_fwd_push(h, 0, None, good, 3, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_repack_fwd_push(h, 0, 0x10000, None, 3, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_repack_fwd_push(h, 0, 0x10000, good, 0, None) == _lib.ULYSSES_ERR_ARG       # planes < 1
    assert lib.ulysses_repack_fwd_push(h, 0, 0x10000, good, 4, None) == _lib.ULYSSES_ERR_ARG       # planes > C
    assert lib.ulysses_repack_fwd_push(h, 0, 0x10000, good, 1, None) in ok_codes
    assert lib.ulysses_repack_fwd_push(h, 0, 0x10000, table(0x40000000, 0), 3, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_repack_fwd_push(h, 0, 0x10008, good, 3, None) == _lib.ULYSSES_ERR_ALIGN
    assert lib.ulysses_repack_fwd_push(h, 0, 0x10000, table(0x40000000, 0x50000004), 3, None) == _lib.ULYSSES_ERR_ALIGN
    # two ranks' destinations overlapping each other
    assert lib.ulysses_repack_fwd_push(h, 0, 0x10000, table(0x40000000, 0x40000000 + 4096), 3, None) == _lib.ULYSSES_ERR_ARG
    # a destination slab overlapping the source shard
    assert lib.ulysses_repack_fwd_push(h, 1, 0x10000, table(0x40000000, 0x10000 + 4096), 3, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_attn_fwd_push(h, 1, 0x10000, good, 0.1, None) in ok_codes
    assert lib.ulysses_attn_fwd_push(h, 1, 0x10000, good, 0.0, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_attn_fwd_push(h, 3, 0x10000, good, 0.1, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_attn_fwd_push(h, 0, 0x10000, table(0x40000000, 0x10000), 0.1, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_repack_bwd_push(h, 0, 0x10000, good, 1, None) in ok_codes
    assert lib.ulysses_repack_bwd_push(h, 0, 0x10000, good, 0, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_repack_bwd_push(h, 0, 0x10000, good, 4, None) == _lib.ULYSSES_ERR_ARG
    # shards use the token-interleaved layout only
    pm = U.ulysses_plan(1024, 8, 128, 2, 3, 8 * 128, 1024 * 8 * 128)
    assert lib.ulysses_repack_fwd_push(pm.handle, 0, 0x10000, good, 3, None) == _lib.ULYSSES_ERR_UNSUPPORTED
    assert lib.ulysses_attn_fwd_push(pm.handle, 0, 0x10000, good, 0.1, None) == _lib.ULYSSES_ERR_UNSUPPORTED
    # the all-to-all fallback's pack and unpack
    assert lib.ulysses_a2a_pack(h, 0x10000, 3, 2, 0x40000000, None) in ok_codes
    assert lib.ulysses_a2a_pack(h, 0x10000, 3, 3, 0x40000000, None) == _lib.ULYSSES_ERR_ARG      # plane >= planes
    assert lib.ulysses_a2a_pack(h, 0x10000, 0, 0, 0x40000000, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_a2a_pack(h, 0x10000, 9, 0, 0x40000000, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_a2a_pack(h, 0x10008, 3, 0, 0x40000000, None) == _lib.ULYSSES_ERR_ALIGN
    assert lib.ulysses_a2a_pack(h, 0x10000, 3, 0, 0x10000 + 512, None) == _lib.ULYSSES_ERR_ARG   # overlap
    assert lib.ulysses_a2a_unpack(h, 0x10000, 0x40000000, 3, 1, None) in ok_codes
    assert lib.ulysses_a2a_unpack(h, 0x10000, 0x40000000, 1, 1, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_a2a_unpack(h, 0x10000, 0x10000, 1, 0, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_a2a_pack(pm.handle, 0x10000, 3, 0, 0x40000000, None) == _lib.ULYSSES_ERR_UNSUPPORTED
    # one rank's slab: the one-GPU checks on the slab's sizes
    assert lib.ulysses_attn_fwd_lse_slab(h, 0x10000, 0x40000000, 0x50000000, 0.1, None) in ok_codes
    assert lib.ulysses_attn_fwd_lse_slab(h, 0x10000, 0x10000, 0x50000000, 0.1, None) == _lib.ULYSSES_ERR_ARG
    assert lib.ulysses_attn_fwd_lse_slab(None, 0x10000, 0x40000000, 0x50000000, 0.1, None) == _lib.ULYSSES_ERR_ARG
    small = plan.slab_attn_bwd_workspace_bytes
    assert small * 2 == plan.attn_bwd_workspace_bytes
    assert lib.ulysses_attn_bwd_slab(h, 0x10000, 0x20000000, 0x30000000, 0x40000000, 0x50000000, 0x60000000,
                                     small - 16, 0.1, None) == _lib.ULYSSES_ERR_WORKSPACE
    assert lib.ulysses_attn_bwd_slab(h, 0x10000, 0x20000000, 0x30000000, 0x40000000, 0x50000000, 0x60000000,
                                     small, 0.1, None) in ok_codes
    # the binding wants one destination per rank
    with pytest.raises(U.UlyssesError):
        U.ulysses_repack_fwd_push(plan, 0, 0x10000, [0x40000000], stream=0)
    with pytest.raises(U.UlyssesError):
        U.ulysses_attn_fwd_push(plan, 0, 0x10000, [0x40000000, 0x50000000, 0x60000000], 0.1, stream=0)


def test_strerror_covers_every_code():
    for code in range(9):
        assert U.strerror(code) != "unknown error code"
    assert U.strerror(99) == "unknown error code"


def test_a_plain_c_program_links_the_library(tmp_path):
    """The boundary is a C ABI: a C99 program that includes only
    include/ulysses.h links libulysses.so, creates a plan and reads its sizes
    (no GPU needed: launches would return ULYSSES_ERR_CUDA)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib = U.library_path()
    U.load()   # builds the library if the sources are newer
    src = tmp_path / "probe.c"
    src.write_text(r'''
#include <stdio.h>
#include "ulysses.h"
int main(void) {
  ulysses_plan_t* p = NULL;
  int s = ulysses_plan(&p, 19394, 56, 128, 4, 3, 0, 0, 0, NULL, 0);
  if (s != ULYSSES_OK) return 10 + s;
  printf("%lld %lld %zu %s\n", (long long)ulysses_plan_padded_tokens(p),
         (long long)ulysses_plan_window_bytes_per_plane(p), ulysses_workspace_bytes(p), ulysses_strerror(ULYSSES_ERR_ALIGN));
  int bad = ulysses_repack_fwd(p, NULL, NULL, NULL);
  ulysses_plan_destroy(p);
  return bad == ULYSSES_ERR_ARG ? 0 : 20;
}
''')
    exe = tmp_path / "probe"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    "-L", os.path.dirname(lib), "-l:" + os.path.basename(lib),
                    "-Wl,-rpath," + os.path.dirname(lib), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out
    Np, window, ws = out.stdout.split()[:3]
    assert int(Np) == 19396
    assert int(window) == 4849 * 56 * 128 * 2
    assert int(ws) > 0 and "16-byte" in out.stdout
