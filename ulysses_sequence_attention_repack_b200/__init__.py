"""One-GPU Ulysses sequence-parallel attention layer for NVIDIA B200 (sm_100a).

The layer (repack -> attention -> inverse repack) runs in the kernels of
``libulysses.so``; this package is its Python binding.  Entry points keep the
names of the C ABI declared in ``include/ulysses.h``.
"""
from ._lib import (  # noqa: F401
    EXPORTS,
    MAX_SEQS,
    MAX_WINDOW_BYTES,
    Plan,
    UlyssesError,
    library_path,
    load,
    strerror,
    ulysses_a2a_pack,
    ulysses_a2a_unpack,
    ulysses_attn_bwd,
    ulysses_attn_bwd_slab,
    ulysses_attn_fwd,
    ulysses_attn_fwd_fp8,
    ulysses_attn_fwd_lse,
    ulysses_attn_fwd_lse_slab,
    ulysses_attn_fwd_push,
    ulysses_last_device_error,
    ulysses_layer_bwd,
    ulysses_layer_fwd,
    ulysses_layer_fwd_fp8,
    ulysses_layer_fwd_fp8_host,
    ulysses_layer_fwd_fused_noalloc,
    ulysses_layer_fwd_host,
    ulysses_plan,
    ulysses_prologue_repack_fwd,
    ulysses_repack_bwd,
    ulysses_repack_bwd_push,
    ulysses_repack_fwd,
    ulysses_repack_fwd_fp8,
    ulysses_repack_fwd_push,
)
