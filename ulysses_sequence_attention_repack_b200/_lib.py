"""ctypes binding of libulysses.so: argument marshalling only.

Every function has the name of the C entry point it calls and takes torch
tensors (device memory), plain ints and an optional CUDA stream; all work
happens in the library's kernels.  There is no fallback: if the library
cannot be loaded, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build


# return codes, as in include/ulysses.h
ULYSSES_OK = 0
ULYSSES_ERR_ARG = 1
ULYSSES_ERR_DIVISIBILITY = 2
ULYSSES_ERR_ALIGN = 3
ULYSSES_ERR_WINDOW = 4
ULYSSES_ERR_WORKSPACE = 5
ULYSSES_ERR_CUDA = 6
ULYSSES_ERR_DEVICE = 7
ULYSSES_ERR_UNSUPPORTED = 8
ULYSSES_PLAN_CAUSAL = 1
ULYSSES_PLAN_PAIR_ATTENTION = 2
ULYSSES_PLAN_DETERMINISTIC = 4
MAX_SEQS = 64
MAX_WINDOW_BYTES = 1024 ** 3

EXPORTS = (
    "ulysses_plan", "ulysses_plan_ex", "ulysses_plan_destroy", "ulysses_plan_padded_tokens", "ulysses_plan_plane_chunk",
    "ulysses_plan_window_bytes_per_plane", "ulysses_workspace_bytes", "ulysses_repack_fwd",
    "ulysses_repack_bwd", "ulysses_attn_fwd", "ulysses_layer_fwd", "ulysses_layer_fwd_host",
    "ulysses_last_device_error", "ulysses_strerror",
    "ulysses_layer_fwd_fused_noalloc", "ulysses_prologue_repack_fwd",
    "ulysses_lse_bytes", "ulysses_attn_fwd_lse", "ulysses_attn_bwd_workspace_bytes", "ulysses_attn_bwd",
    "ulysses_layer_bwd_workspace_bytes", "ulysses_layer_bwd", "ulysses_repack_fwd_fp8", "ulysses_attn_fwd_fp8",
    "ulysses_workspace_bytes_fp8", "ulysses_layer_fwd_fp8", "ulysses_repack_fwd_push", "ulysses_attn_fwd_push",
    "ulysses_repack_bwd_push", "ulysses_attn_fwd_lse_slab", "ulysses_attn_bwd_slab", "ulysses_a2a_pack",
    "ulysses_a2a_unpack", "ulysses_layer_fwd_fp8_host",
)


class UlyssesError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: error {code}: {strerror(code)}")


_lock = threading.Lock()
_handle: ctypes.CDLL | None = None


def library_path() -> str:
    """The library this process loads: $ULYSSES_LIBRARY when set (for
    example the bounds-checked libulysses_debug.so), else the in-tree
    libulysses.so."""
    return os.environ.get("ULYSSES_LIBRARY") or _build.LIB


def load() -> ctypes.CDLL:
    """Load (building first if the sources are newer) and type the library."""
    global _handle
    with _lock:
        if _handle is not None:
            return _handle
        path = os.environ.get("ULYSSES_LIBRARY") or _build.ensure_built()
        if not os.path.exists(path):
            raise ImportError(f"libulysses library missing at {path}")
        lib = ctypes.CDLL(path)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        lib.ulysses_plan.argtypes = [ctypes.POINTER(vp), i64, i32, i32, i32, i32, i64, i64, i64,
                                     ctypes.POINTER(ctypes.c_int32), i32]
        lib.ulysses_plan.restype = ctypes.c_int
        lib.ulysses_plan_ex.argtypes = [ctypes.POINTER(vp), i64, i32, i32, i32, i32, i64, i64, i64,
                                        ctypes.POINTER(ctypes.c_int32), i32, ctypes.c_uint32]
        lib.ulysses_plan_ex.restype = ctypes.c_int
        lib.ulysses_plan_destroy.argtypes = [vp]
        lib.ulysses_plan_destroy.restype = None
        lib.ulysses_plan_padded_tokens.argtypes = [vp]
        lib.ulysses_plan_padded_tokens.restype = i64
        lib.ulysses_plan_plane_chunk.argtypes = [vp]
        lib.ulysses_plan_plane_chunk.restype = i32
        lib.ulysses_plan_window_bytes_per_plane.argtypes = [vp]
        lib.ulysses_plan_window_bytes_per_plane.restype = i64
        lib.ulysses_workspace_bytes.argtypes = [vp]
        lib.ulysses_workspace_bytes.restype = sz
        lib.ulysses_repack_fwd.argtypes = [vp, vp, vp, vp]
        lib.ulysses_repack_fwd.restype = ctypes.c_int
        lib.ulysses_prologue_repack_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, ctypes.c_float, vp]
        lib.ulysses_prologue_repack_fwd.restype = ctypes.c_int
        lib.ulysses_lse_bytes.argtypes = [vp]
        lib.ulysses_lse_bytes.restype = sz
        lib.ulysses_attn_fwd_lse.argtypes = [vp, vp, vp, vp, ctypes.c_float, vp]
        lib.ulysses_attn_fwd_lse.restype = ctypes.c_int
        lib.ulysses_attn_bwd_workspace_bytes.argtypes = [vp]
        lib.ulysses_attn_bwd_workspace_bytes.restype = sz
        lib.ulysses_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, sz, ctypes.c_float, vp]
        lib.ulysses_attn_bwd.restype = ctypes.c_int
        lib.ulysses_layer_bwd_workspace_bytes.argtypes = [vp]
        lib.ulysses_layer_bwd_workspace_bytes.restype = sz
        lib.ulysses_layer_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.ulysses_layer_bwd.restype = ctypes.c_int
        lib.ulysses_repack_bwd.argtypes = [vp, vp, vp, i32, vp]
        lib.ulysses_repack_bwd.restype = ctypes.c_int
        lib.ulysses_attn_fwd.argtypes = [vp, vp, vp, ctypes.c_float, vp]
        lib.ulysses_attn_fwd.restype = ctypes.c_int
        lib.ulysses_layer_fwd.argtypes = [vp, vp, vp, vp, sz, i32, vp]
        lib.ulysses_layer_fwd.restype = ctypes.c_int
        lib.ulysses_layer_fwd_host.argtypes = [vp, vp, vp, vp, vp, vp, sz, i32, vp]
        lib.ulysses_layer_fwd_host.restype = ctypes.c_int
        lib.ulysses_last_device_error.argtypes = [vp, vp]
        lib.ulysses_last_device_error.restype = ctypes.c_int
        lib.ulysses_strerror.argtypes = [ctypes.c_int]
        lib.ulysses_strerror.restype = ctypes.c_char_p
        lib.ulysses_layer_fwd_fused_noalloc.argtypes = [vp, vp, i64, i32, i32, i32, i32, i64, i64,
                                                        ctypes.POINTER(ctypes.c_int32), i32,
                                                        ctypes.POINTER(ctypes.c_int32), vp]
        lib.ulysses_layer_fwd_fused_noalloc.restype = ctypes.c_int
        lib.ulysses_repack_fwd_fp8.argtypes = [vp, vp, vp, vp]
        lib.ulysses_repack_fwd_fp8.restype = ctypes.c_int
        lib.ulysses_attn_fwd_fp8.argtypes = [vp, vp, vp, ctypes.c_float, vp]
        lib.ulysses_attn_fwd_fp8.restype = ctypes.c_int
        lib.ulysses_workspace_bytes_fp8.argtypes = [vp]
        lib.ulysses_workspace_bytes_fp8.restype = sz
        lib.ulysses_layer_fwd_fp8.argtypes = [vp, vp, vp, vp, sz, vp]
        lib.ulysses_layer_fwd_fp8.restype = ctypes.c_int
        lib.ulysses_repack_fwd_push.argtypes = [vp, i32, vp, ctypes.POINTER(vp), i32, vp]
        lib.ulysses_repack_fwd_push.restype = ctypes.c_int
        lib.ulysses_attn_fwd_push.argtypes = [vp, i32, vp, ctypes.POINTER(vp), ctypes.c_float, vp]
        lib.ulysses_attn_fwd_push.restype = ctypes.c_int
        lib.ulysses_repack_bwd_push.argtypes = [vp, i32, vp, ctypes.POINTER(vp), i32, vp]
        lib.ulysses_repack_bwd_push.restype = ctypes.c_int
        lib.ulysses_layer_fwd_fp8_host.argtypes = [vp, vp, vp, vp, vp, vp, sz, vp]
        lib.ulysses_layer_fwd_fp8_host.restype = ctypes.c_int
        lib.ulysses_a2a_pack.argtypes = [vp, vp, i32, i32, vp, vp]
        lib.ulysses_a2a_pack.restype = ctypes.c_int
        lib.ulysses_a2a_unpack.argtypes = [vp, vp, vp, i32, i32, vp]
        lib.ulysses_a2a_unpack.restype = ctypes.c_int
        lib.ulysses_attn_fwd_lse_slab.argtypes = [vp, vp, vp, vp, ctypes.c_float, vp]
        lib.ulysses_attn_fwd_lse_slab.restype = ctypes.c_int
        lib.ulysses_attn_bwd_slab.argtypes = [vp, vp, vp, vp, vp, vp, vp, sz, ctypes.c_float, vp]
        lib.ulysses_attn_bwd_slab.restype = ctypes.c_int
        _handle = lib
        return lib


def strerror(code: int) -> str:
    return load().ulysses_strerror(int(code)).decode()


def _check(code: int, where: str) -> None:
    if code != ULYSSES_OK:
        raise UlyssesError(code, where)


def _ptr(t) -> int | None:
    """Device (or host) address of a tensor, or an int address as given."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class Plan:
    """Owner of a ulysses_plan_t*; destroyed with the object."""

    def __init__(self, handle: int, N: int, H: int, D: int, P: int, planes: int, cu_seqlens, causal: bool = False):
        self._h = ctypes.c_void_p(handle)
        self.N, self.H, self.D, self.P, self.planes = N, H, D, P, planes
        self.causal = bool(causal)
        self.cu_seqlens = None if cu_seqlens is None else [int(x) for x in cu_seqlens]

    @property
    def handle(self) -> ctypes.c_void_p:
        if not self._h:
            raise ValueError("plan destroyed")
        return self._h

    @property
    def padded_tokens(self) -> int:
        return load().ulysses_plan_padded_tokens(self.handle)

    @property
    def rows_per_rank(self) -> int:
        """Nl = Np / P: the sequence rows each rank owns."""
        return self.padded_tokens // self.P

    @property
    def plane_chunk(self) -> int:
        return load().ulysses_plan_plane_chunk(self.handle)

    @property
    def window_bytes_per_plane(self) -> int:
        return load().ulysses_plan_window_bytes_per_plane(self.handle)

    @property
    def workspace_bytes(self) -> int:
        return load().ulysses_workspace_bytes(self.handle)

    @property
    def workspace_bytes_fp8(self) -> int:
        return load().ulysses_workspace_bytes_fp8(self.handle)

    @property
    def lse_bytes(self) -> int:
        return load().ulysses_lse_bytes(self.handle)

    @property
    def lse_row_stride(self) -> int:
        """Floats between the lse rows of consecutive (rank, local head) pairs."""
        return self.lse_bytes // 4 // self.H

    @property
    def attn_bwd_workspace_bytes(self) -> int:
        return load().ulysses_attn_bwd_workspace_bytes(self.handle)

    @property
    def slab_lse_bytes(self) -> int:
        """lse bytes of one rank's slab (ulysses_attn_fwd_lse_slab)."""
        return self.lse_bytes // self.P

    @property
    def slab_attn_bwd_workspace_bytes(self) -> int:
        """Workspace of ulysses_attn_bwd_slab."""
        return self.attn_bwd_workspace_bytes // self.P

    @property
    def layer_bwd_workspace_bytes(self) -> int:
        return load().ulysses_layer_bwd_workspace_bytes(self.handle)

    def destroy(self) -> None:
        if self._h:
            load().ulysses_plan_destroy(self._h)
            self._h = ctypes.c_void_p(None)

    def __del__(self):
        try:
            self.destroy()
        except Exception:  # noqa: BLE001 - interpreter shutdown
            pass


def ulysses_plan(N: int, H: int, D: int, P: int, planes: int, token_stride: int = 0, plane_stride: int = 0,
                 plane_chunk: int = 0, cu_seqlens=None, causal: bool = False, pair_cta: bool = False,
                 deterministic: bool = False) -> Plan:
    """ulysses_plan (or ulysses_plan_ex with ULYSSES_PLAN_CAUSAL when causal,
    ULYSSES_PLAN_PAIR_ATTENTION when pair_cta, ULYSSES_PLAN_DETERMINISTIC when
    deterministic)."""
    lib = load()
    h = ctypes.c_void_p()
    if cu_seqlens is None:
        arr, ns = None, 0
    else:
        vals = [int(x) for x in cu_seqlens]
        arr = (ctypes.c_int32 * len(vals))(*vals)
        ns = len(vals) - 1
    flags = ((ULYSSES_PLAN_CAUSAL if causal else 0) | (ULYSSES_PLAN_PAIR_ATTENTION if pair_cta else 0)
             | (ULYSSES_PLAN_DETERMINISTIC if deterministic else 0))
    if flags:
        code = lib.ulysses_plan_ex(ctypes.byref(h), int(N), int(H), int(D), int(P), int(planes), int(token_stride),
                                   int(plane_stride), int(plane_chunk), arr, ns, flags)
    else:
        code = lib.ulysses_plan(ctypes.byref(h), int(N), int(H), int(D), int(P), int(planes), int(token_stride),
                                int(plane_stride), int(plane_chunk), arr, ns)
    _check(code, "ulysses_plan")
    return Plan(h.value, N, H, D, P, planes, cu_seqlens, causal)


def ulysses_repack_fwd(plan: Plan, src_seq, dst_heads, stream=None) -> None:
    _check(load().ulysses_repack_fwd(plan.handle, _ptr(src_seq), _ptr(dst_heads), _stream(stream)),
           "ulysses_repack_fwd")


def ulysses_prologue_repack_fwd(plan: Plan, src_seq, dst_heads, norm_q_weight, norm_k_weight, cos, sin,
                                rotary_dim: int, eps: float = 1e-5, stream=None) -> None:
    _check(load().ulysses_prologue_repack_fwd(plan.handle, _ptr(src_seq), _ptr(dst_heads), _ptr(norm_q_weight),
                                              _ptr(norm_k_weight), _ptr(cos), _ptr(sin), int(rotary_dim),
                                              float(eps), _stream(stream)), "ulysses_prologue_repack_fwd")


def ulysses_attn_fwd_lse(plan: Plan, qkv_heads, out_heads, lse, softmax_scale: float, stream=None) -> None:
    _check(load().ulysses_attn_fwd_lse(plan.handle, _ptr(qkv_heads), _ptr(out_heads), _ptr(lse),
                                       float(softmax_scale), _stream(stream)), "ulysses_attn_fwd_lse")


def ulysses_attn_bwd(plan: Plan, qkv_heads, out_heads, dout_heads, lse, dqkv_heads, workspace,
                     softmax_scale: float, workspace_bytes: int | None = None, stream=None) -> None:
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(load().ulysses_attn_bwd(plan.handle, _ptr(qkv_heads), _ptr(out_heads), _ptr(dout_heads), _ptr(lse),
                                   _ptr(dqkv_heads), _ptr(workspace), int(workspace_bytes), float(softmax_scale),
                                   _stream(stream)), "ulysses_attn_bwd")


def ulysses_a2a_pack(plan: Plan, src_shard, planes: int, plane: int, send, stream=None) -> None:
    """Plane `plane` of a shard [Nl, planes, H, D] -> all-to-all send buffer [P, Nl, Hl, D]."""
    _check(load().ulysses_a2a_pack(plan.handle, _ptr(src_shard), int(planes), int(plane), _ptr(send),
                                   _stream(stream)), "ulysses_a2a_pack")


def ulysses_a2a_unpack(plan: Plan, recv, out_shard, planes: int, plane: int, stream=None) -> None:
    """All-to-all receive buffer [P, Nl, Hl, D] -> plane `plane` of a shard [Nl, planes, H, D]."""
    _check(load().ulysses_a2a_unpack(plan.handle, _ptr(recv), _ptr(out_shard), int(planes), int(plane),
                                     _stream(stream)), "ulysses_a2a_unpack")


def ulysses_attn_fwd_lse_slab(plan: Plan, heads, out_heads, lse, softmax_scale: float, stream=None) -> None:
    """Attention over one rank's head slab [C, Np, Hl, D] with its lse."""
    _check(load().ulysses_attn_fwd_lse_slab(plan.handle, _ptr(heads), _ptr(out_heads), _ptr(lse),
                                            float(softmax_scale), _stream(stream)), "ulysses_attn_fwd_lse_slab")


def ulysses_attn_bwd_slab(plan: Plan, heads, out_heads, dout_heads, lse, dqkv_heads, workspace,
                          softmax_scale: float, workspace_bytes: int | None = None, stream=None) -> None:
    """The attention backward of one rank's head slab: dqkv_heads [3, Np, Hl, D]."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(load().ulysses_attn_bwd_slab(plan.handle, _ptr(heads), _ptr(out_heads), _ptr(dout_heads), _ptr(lse),
                                        _ptr(dqkv_heads), _ptr(workspace), int(workspace_bytes),
                                        float(softmax_scale), _stream(stream)), "ulysses_attn_bwd_slab")


def ulysses_layer_bwd(plan: Plan, qkv_heads, out_heads, lse, dout_seq, dqkv_seq, workspace,
                      workspace_bytes: int | None = None, stream=None) -> None:
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(load().ulysses_layer_bwd(plan.handle, _ptr(qkv_heads), _ptr(out_heads), _ptr(lse), _ptr(dout_seq),
                                    _ptr(dqkv_seq), _ptr(workspace), int(workspace_bytes), _stream(stream)),
           "ulysses_layer_bwd")


def ulysses_repack_bwd(plan: Plan, src_heads, dst_seq, planes: int, stream=None) -> None:
    _check(load().ulysses_repack_bwd(plan.handle, _ptr(src_heads), _ptr(dst_seq), int(planes), _stream(stream)),
           "ulysses_repack_bwd")


def ulysses_attn_fwd(plan: Plan, qkv_heads, out_heads, softmax_scale: float, stream=None) -> None:
    _check(load().ulysses_attn_fwd(plan.handle, _ptr(qkv_heads), _ptr(out_heads), float(softmax_scale),
                                   _stream(stream)), "ulysses_attn_fwd")


def _ptr_table(ptrs):
    """Host array of device pointers (tensors or int addresses), indexed by rank."""
    if ptrs is None:
        return None
    vals = [_ptr(t) for t in ptrs]
    return (ctypes.c_void_p * max(1, len(vals)))(*vals)


def ulysses_repack_fwd_push(plan: Plan, rank: int, src_shard, dst_heads, planes: int | None = None,
                            stream=None) -> None:
    """Rank `rank` pushes its shard [Nl, planes, H, D] into every rank's head
    slab dst_heads[r] = T_r [planes, Np, Hl, D] (device pointers, one per
    rank); planes defaults to the plan's C."""
    if dst_heads is not None and len(dst_heads) != plan.P:
        raise UlyssesError(ULYSSES_ERR_ARG, "ulysses_repack_fwd_push: one destination per rank")
    planes = plan.planes if planes is None else int(planes)
    _check(load().ulysses_repack_fwd_push(plan.handle, int(rank), _ptr(src_shard), _ptr_table(dst_heads), planes,
                                          _stream(stream)), "ulysses_repack_fwd_push")


def ulysses_attn_fwd_push(plan: Plan, rank: int, heads, dst_seq, softmax_scale: float, stream=None) -> None:
    """Attention over rank `rank`'s head slab T_r with each output row stored
    into its owning rank's shard dst_seq[q] = O_q [Nl, H, D]."""
    if dst_seq is not None and len(dst_seq) != plan.P:
        raise UlyssesError(ULYSSES_ERR_ARG, "ulysses_attn_fwd_push: one destination per rank")
    _check(load().ulysses_attn_fwd_push(plan.handle, int(rank), _ptr(heads), _ptr_table(dst_seq),
                                        float(softmax_scale), _stream(stream)), "ulysses_attn_fwd_push")


def ulysses_repack_bwd_push(plan: Plan, rank: int, src_heads, dst_seq, planes: int, stream=None) -> None:
    """Rank `rank` pushes its head rows [planes, Np, Hl, D] into every rank's
    shard dst_seq[q] = [Nl, planes, H, D]."""
    if dst_seq is not None and len(dst_seq) != plan.P:
        raise UlyssesError(ULYSSES_ERR_ARG, "ulysses_repack_bwd_push: one destination per rank")
    _check(load().ulysses_repack_bwd_push(plan.handle, int(rank), _ptr(src_heads), _ptr_table(dst_seq), int(planes),
                                          _stream(stream)), "ulysses_repack_bwd_push")


def ulysses_repack_fwd_fp8(plan: Plan, src_seq, dst_heads_fp8, stream=None) -> None:
    _check(load().ulysses_repack_fwd_fp8(plan.handle, _ptr(src_seq), _ptr(dst_heads_fp8), _stream(stream)),
           "ulysses_repack_fwd_fp8")


def ulysses_attn_fwd_fp8(plan: Plan, qkv_heads_fp8, out_heads, softmax_scale: float, stream=None) -> None:
    _check(load().ulysses_attn_fwd_fp8(plan.handle, _ptr(qkv_heads_fp8), _ptr(out_heads), float(softmax_scale),
                                       _stream(stream)), "ulysses_attn_fwd_fp8")


def ulysses_layer_fwd_fp8(plan: Plan, qkv_seq, out_seq, workspace, workspace_bytes: int | None = None,
                          stream=None) -> None:
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().ulysses_layer_fwd_fp8(plan.handle, _ptr(qkv_seq), _ptr(out_seq), _ptr(workspace),
                                        int(workspace_bytes), _stream(stream)), "ulysses_layer_fwd_fp8")


def ulysses_layer_fwd(plan: Plan, qkv_seq, out_seq, workspace=None, workspace_bytes: int | None = None,
                      fused: int = 0, stream=None) -> None:
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().ulysses_layer_fwd(plan.handle, _ptr(qkv_seq), _ptr(out_seq), _ptr(workspace),
                                    int(workspace_bytes), int(fused), _stream(stream)), "ulysses_layer_fwd")


def ulysses_layer_fwd_host(plan: Plan, host_qkv_seq, host_out_seq, dev_qkv_seq, dev_out_seq, workspace=None,
                           workspace_bytes: int | None = None, fused: int = 0, stream=None) -> None:
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().ulysses_layer_fwd_host(plan.handle, _ptr(host_qkv_seq), _ptr(host_out_seq), _ptr(dev_qkv_seq),
                                         _ptr(dev_out_seq), _ptr(workspace), int(workspace_bytes), int(fused),
                                         _stream(stream)), "ulysses_layer_fwd_host")


def ulysses_layer_fwd_fp8_host(plan: Plan, host_qkv_seq, host_out_seq, dev_qkv_seq, dev_out_seq, workspace,
                               workspace_bytes: int | None = None, stream=None) -> None:
    """The FP8 layer from host buffers, streamed by head groups (workspace_bytes_fp8)."""
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().ulysses_layer_fwd_fp8_host(plan.handle, _ptr(host_qkv_seq), _ptr(host_out_seq), _ptr(dev_qkv_seq),
                                             _ptr(dev_out_seq), _ptr(workspace), int(workspace_bytes),
                                             _stream(stream)), "ulysses_layer_fwd_fp8_host")


def ulysses_last_device_error(plan: Plan, stream=None) -> int:
    return load().ulysses_last_device_error(plan.handle, _stream(stream))


def ulysses_layer_fwd_fused_noalloc(qkv_seq, out_seq, N: int, H: int, D: int, P: int, planes: int,
                                    token_stride: int = 0, plane_stride: int = 0, cu_seqlens=None,
                                    check: bool = False, stream=None) -> int:
    """The fused layer without a plan and without any device allocation.

    Returns the kernel's error bits when ``check`` is true (the call then
    synchronises the stream; non-zero bits are returned, not raised), else 0.
    Argument and CUDA errors raise UlyssesError.
    """
    if cu_seqlens is None:
        arr, ns = None, 0
    else:
        vals = [int(x) for x in cu_seqlens]
        arr = (ctypes.c_int32 * len(vals))(*vals)
        ns = len(vals) - 1
    status = ctypes.c_int32(0)
    code = load().ulysses_layer_fwd_fused_noalloc(_ptr(qkv_seq), _ptr(out_seq), int(N), int(H), int(D), int(P),
                                                  int(planes), int(token_stride), int(plane_stride), arr, ns,
                                                  ctypes.byref(status) if check else None, _stream(stream))
    if check and code == ULYSSES_ERR_DEVICE:
        return status.value
    _check(code, "ulysses_layer_fwd_fused_noalloc")
    return status.value
