"""Plain CPU oracle for the Ulysses sequence-parallel attention layer (fp64).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
use it.  It shares no code with the CUDA library; both sides see the same
seeded inputs and nothing else.

Sources (web pages, cited by title and section):

* "hao-ai-lab FastVideo, compare main...perf/ulysses-h3-adaptive" -- the fused
  Ulysses all-to-all.  The shape comment above ``ulysses_a2a_tuned`` in
  ``csrc/comm/ulysses_all_to_all.cu`` fixes the two modes:
  mode 0 maps ``[B, S_local, H, D]`` to ``[B, S_global, H_local, D]`` and mode 1
  is its inverse, with ``H_local = H / world``.  ``docs/contributing/
  ulysses_performance.md`` ("Ulysses performance on GB200") fixes the 1 GiB
  per-rank window and the per-plane exchange (896,000,000 bytes per plane at
  250,000 tokens, 56 heads, head dim 128, sequence parallelism 4).
  ``ulysses_a2a.py`` (``MAX_WINDOW_BYTES``, ``_call_signature``, ``run_armed``)
  gives the window arithmetic and the one-launch-per-plane loop.
* "hao-ai-lab FastVideo, compare aryan/h3-nvfp4-stack-speedups...main" --
  ``DistributedAttention.forward_stacked`` in ``fastvideo/attention/layer.py``
  (stack Q/K/V, all-to-all with scatter_dim=2 / gather_dim=1, backend
  attention, inverse all-to-all) and the FA4 wrappers in
  ``flash_attn_cute.py`` (softmax attention with ``softmax_scale``, non-causal,
  varlen through ``cu_seqlens``).

Readings where the pages leave a step open (each one is also listed in the
design notes of the repository):

* The all-to-all body is not printed.  We take the standard reading of the
  mode-0 shape map: source rank q contributes its local tokens as global rows
  ``q*Nl + i`` (rank order), and destination rank r receives heads
  ``[r*Hl, (r+1)*Hl)``.
* N not divisible by P is padded to ``Np = P*ceil(N/P)`` rows; pad rows are
  moved by the repack like any other row, never attended to as keys, and
  produce zero output rows.
* Sequence-sharded layout is token-interleaved ``[Np, C, H, D]`` (planes Q, K,
  V[, G]); head-sharded layout is ``[P, C, Np, Hl, D]``.

Everything here is written for clarity, not speed.
"""
from __future__ import annotations

import math

import numpy as np

# 1 GiB registered window per rank ("Ulysses performance on GB200": each rank
# keeps at most 1 GiB of registered window storage; ``MAX_WINDOW_BYTES`` in
# ulysses_a2a.py).
MAX_WINDOW_BYTES = 1024 ** 3
BF16_BYTES = 2


# ---------------------------------------------------------------------------
# Sizes and window arithmetic
# ---------------------------------------------------------------------------

def local_tokens(N: int, P: int) -> int:
    """Nl = ceil(N / P): tokens owned by each virtual rank before the repack."""
    if P < 1 or N < 0:
        raise ValueError("need P >= 1 and N >= 0")
    return -(-N // P)


def padded_tokens(N: int, P: int) -> int:
    """Np = P * Nl: the padded global sequence length every buffer is sized for."""
    return P * local_tokens(N, P)


def plane_bytes_per_rank(N: int, H: int, D: int, P: int, elem_bytes: int = BF16_BYTES) -> int:
    """Bytes one virtual rank sends (and receives) for ONE plane.

    Sequence side: Nl tokens x H heads x D; head side: Np tokens x H/P heads x D.
    Both are equal.  ulysses_a2a.py sizes the chunked window as
    ``nbytes // planes`` for an operand ``[planes, S_local, H, D]``.
    """
    return local_tokens(N, P) * H * D * elem_bytes


def auto_plane_chunk(N: int, H: int, D: int, P: int, planes: int,
                     window_bytes: int = MAX_WINDOW_BYTES) -> int:
    """Largest number of planes per launch whose per-rank bytes fit the window.

    Returns 0 when a single plane already exceeds the window (the call must be
    refused, as ulysses_a2a.py declines operands whose window exceeds the cap).
    """
    per_plane = plane_bytes_per_rank(N, H, D, P)
    if per_plane > window_bytes:
        return 0
    if per_plane == 0:
        return planes
    return min(planes, window_bytes // per_plane)


# ---------------------------------------------------------------------------
# bf16 helpers (bit patterns held as uint16)
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening: a bf16 pattern is the top half of an IEEE binary32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 -> fp32 (round to nearest even) -> bf16 (round to nearest even).

    Used only to build bf16 inputs for closed-form tests; NaN maps to the
    canonical quiet NaN 0x7FC0.
    """
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    rounded = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(f)
    rounded[nan] = 0x7FC0
    return rounded


# ---------------------------------------------------------------------------
# Repack (the all-to-all index map), exact on bit patterns
# ---------------------------------------------------------------------------

def repack_fwd(S: np.ndarray, P: int) -> np.ndarray:
    """Ulysses mode 0 on one GPU: sequence-sharded -> head-sharded.

    S: ``[Np, C, H, D]`` uint16 (bf16 bits).  Rank q owns rows ``[q*Nl, (q+1)*Nl)``.
    Returns T: ``[P, C, Np, Hl, D]`` with ``T[r, c, n, j, d] = S[n, c, r*Hl + j, d]``.

    Written as the reshape/transpose of the mode-0 shape comment in
    ``ulysses_all_to_all.cu``: every source rank's ``[Nl, H, D]`` block is split
    along heads into P pieces; piece r goes to rank r, where the pieces from
    all source ranks are stacked in source-rank order along the sequence.
    """
    Np, C, H, D = S.shape
    if Np % P or H % P:
        raise ValueError("Np and H must be divisible by P")
    Nl, Hl = Np // P, H // P
    # [src rank q, local token i, plane c, dest rank r, local head j, d]
    x = S.reshape(P, Nl, C, P, Hl, D)
    # -> [dest rank r, plane c, src rank q, local token i, local head j, d]
    x = x.transpose(3, 2, 0, 1, 4, 5)
    return np.ascontiguousarray(x).reshape(P, C, Np, Hl, D)


def repack_bwd(T: np.ndarray) -> np.ndarray:
    """Ulysses mode 1: head-sharded ``[P, C, Np, Hl, D]`` -> ``[Np, C, P*Hl, D]``.

    ``S[n, c, r*Hl + j, d] = T[r, c, n, j, d]``: the inverse of :func:`repack_fwd`.
    """
    P, C, Np, Hl, D = T.shape
    Nl = Np // P
    x = T.reshape(P, C, P, Nl, Hl, D)           # [r, c, q, i, j, d]
    x = x.transpose(2, 3, 1, 0, 4, 5)            # [q, i, c, r, j, d]
    return np.ascontiguousarray(x).reshape(Np, C, P * Hl, D)


# ---------------------------------------------------------------------------
# Attention (fp64 definition)
# ---------------------------------------------------------------------------

def segments_from_cu_seqlens(cu_seqlens, N: int) -> list[tuple[int, int]]:
    """Turn ``cu_seqlens`` prefix sums into ``[(start, end), ...]``.

    ``cu_seqlens`` is the varlen metadata of the FA4 wrappers (int32 prefix sums
    of packed sequence lengths, first entry 0, last entry the total).  None
    means one sequence of length N.
    """
    if cu_seqlens is None:
        return [(0, N)]
    cu = [int(v) for v in cu_seqlens]
    if len(cu) < 2 or cu[0] != 0 or cu[-1] != N or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("cu_seqlens must start at 0, be non-decreasing and end at N")
    return [(a, b) for a, b in zip(cu, cu[1:])]


def attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """Softmax attention of query rows ``q [R, D]`` over keys ``k, v [M, D]`` in fp64.

    ``o = softmax(scale * q k^T) v`` row by row (non-causal: every key counts).
    The row maximum is subtracted before ``exp``; this changes nothing
    mathematically and keeps fp64 finite.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if k.shape[0] == 0:
        return np.zeros((q.shape[0], v.shape[1]), dtype=np.float64)
    z = scale * (q @ k.T)                        # [R, M] logits
    z = z - z.max(axis=1, keepdims=True)
    p = np.exp(z)
    return (p @ v) / p.sum(axis=1, keepdims=True)


def attention_heads(T: np.ndarray, N: int, scale: float, cu_seqlens=None,
                    rows: np.ndarray | None = None, workers: int = 1,
                    row_block: int = 256, causal: bool = False, decode=None) -> np.ndarray:
    """Step two of the layer: attention on every head-sharded slab.

    T: head-sharded ``[P, C, Np, Hl, D]`` uint16; planes 0, 1, 2 are Q, K, V
    (a fourth plane, the gate, is ignored).  Query row n attends to the keys of
    its own segment (all keys ``< N`` without ``cu_seqlens``).  Rows ``n >= N``
    are padding and give zero.

    With ``causal``, query row n attends only to keys m <= n of its segment
    (the causal attention of the trainer's Ulysses flash wrapper in "Ulysses
    context parallelism" of the prime-rl pull request).

    Returns fp64 ``[P, R, Hl, D]`` for the selected rows (all ``Np`` rows when
    ``rows`` is None).  Query rows are independent, so they are evaluated
    ``row_block`` at a time to bound memory, and ``workers`` threads may take
    different (rank, head) slabs; neither changes any arithmetic.

    ``decode`` maps the stored codes to fp64: bf16 bit patterns by default,
    :func:`e4m3_bits_to_f64` for the FP8 variant.
    """
    if decode is None:
        decode = bf16_bits_to_f64
    P, C, Np, Hl, D = T.shape
    if C < 3:
        raise ValueError("need Q, K and V planes")
    segs = segments_from_cu_seqlens(cu_seqlens, N)
    rows = np.arange(Np) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((P, rows.size, Hl, D), dtype=np.float64)
    seg_of = np.full(rows.size, -1, dtype=np.int64)
    for s, (a, b) in enumerate(segs):
        seg_of[(rows >= a) & (rows < b)] = s

    def one_slab(rj):
        r, j = rj
        for s, (a, b) in enumerate(segs):
            sel = np.nonzero(seg_of == s)[0]
            if sel.size == 0:
                continue
            k = decode(T[r, 1, a:b, j, :])
            v = decode(T[r, 2, a:b, j, :])
            if causal:
                for i in sel:
                    n = int(rows[i])
                    q = decode(T[r, 0, n:n + 1, j, :])
                    out[r, i, j, :] = attention_rows(q, k[:n + 1 - a], v[:n + 1 - a], scale)[0]
                continue
            for i0 in range(0, sel.size, row_block):
                part = sel[i0:i0 + row_block]
                q = decode(T[r, 0, rows[part], j, :])
                out[r, part, j, :] = attention_rows(q, k, v, scale)

    slabs = [(r, j) for r in range(P) for j in range(Hl)]
    if workers > 1:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=workers) as ex:
            list(ex.map(one_slab, slabs))
    else:
        for rj in slabs:
            one_slab(rj)
    return out


def output_repack_bwd(O_heads: np.ndarray) -> np.ndarray:
    """Step three on the attention output: ``[P, R, Hl, D] -> [R, P*Hl, D]``.

    The same index map as :func:`repack_bwd` with one plane, applied to fp64
    values (row selection already done).
    """
    P, R, Hl, D = O_heads.shape
    return np.ascontiguousarray(O_heads.transpose(1, 0, 2, 3)).reshape(R, P * Hl, D)


def layer_fwd(S: np.ndarray, P: int, N: int, scale: float, cu_seqlens=None,
              rows: np.ndarray | None = None, workers: int = 1, causal: bool = False) -> np.ndarray:
    """The whole layer: repack -> attention per slab -> inverse repack.

    S: sequence-sharded ``[Np, C, H, D]`` uint16.  Returns fp64 ``[R, H, D]``
    (sequence-sharded output rows, all ``Np`` rows when ``rows`` is None).
    """
    T = repack_fwd(S, P)
    O = attention_heads(T, N, scale, cu_seqlens=cu_seqlens, rows=rows, workers=workers, causal=causal)
    return output_repack_bwd(O)


def sample_rows(N: int, count: int, seed: int, cu_seqlens=None) -> np.ndarray:
    """The seeded subset of query rows checked on large N.

    ``count`` rows drawn without replacement from ``[0, N)`` with
    ``numpy.random.default_rng(seed + 10_000)``; rows 0 and N-1 and the first
    and last row of every segment are always included.  Sorted.
    """
    if count >= N:
        return np.arange(N)
    rng = np.random.default_rng(seed + 10_000)
    chosen = set(int(x) for x in rng.choice(N, size=count, replace=False))
    forced = {0, N - 1}
    for a, b in segments_from_cu_seqlens(cu_seqlens, N):
        if b > a:
            forced.update((a, b - 1))
    return np.array(sorted(chosen | forced), dtype=np.int64)


def attention_flops(N: int, H: int, D: int, cu_seqlens=None, causal: bool = False) -> float:
    """Algorithmic attention FLOPs: 4 * L^2 * H * D summed over sequences.

    Causal: each query row n of a segment starting at a uses n - a + 1 keys,
    i.e. 4 * H * D * L (L + 1) / 2 per segment.
    """
    segs = segments_from_cu_seqlens(cu_seqlens, N)
    if causal:
        return float(sum(4 * H * D * (b - a) * (b - a + 1) // 2 for a, b in segs))
    return float(sum(4 * (b - a) ** 2 * H * D for a, b in segs))


def softmax_scale(D: int) -> float:
    """1/sqrt(D): the scale of the Ulysses layer (1/sqrt(128) for D = 128)."""
    return 1.0 / math.sqrt(D)


# ---------------------------------------------------------------------------
# FP8 variant: Q, K and V cast to E4M3 before attention
# ---------------------------------------------------------------------------
#
# The MiniMax-H3 recipe branch described on "Request FA4's 2-CTA kernel for
# MiniMax-H3 on SM103 and SM107" (NVIDIA TensorRT-LLM pull request 21275, its
# commit merging the recipe branches) runs cuDNN FP8 attention with Q and K
# cast to FP8 in a fused step, and FA4 has an FP8 P V path
# (FA4_FP8_PV_USE_FUSED_PACK in the FA4 JIT-cache test of "hao-ai-lab
# FastVideo, compare aryan/h3-nvfp4-stack-speedups...main").  The pages fix no
# scaling recipe; the plainest reading of "cast" is a direct conversion of each
# bf16 value to the nearest E4M3 value (no scale factor), which the N(0,1)
# inputs fit comfortably.  The attention is then the same softmax attention on
# the cast values.
#
# E4M3 (the OCP 8-bit floating-point format "E4M3"): 1 sign bit, 4 exponent
# bits with bias 7, 3 mantissa bits; exponent field 0 encodes subnormals
# m/8 * 2^-6; exponent 15 with mantissa 7 is NaN (no infinities), so the
# largest finite magnitude is 1.75 * 2^8 = 448.

E4M3_MAX = 448.0


def e4m3_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode E4M3 codes (uint8) to fp64, from the format's definition."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 0xF) & ((b & 7) == 7), np.nan, mag)
    return sign * mag


def _e4m3_table():
    codes = np.arange(0x7F, dtype=np.uint8)          # non-negative finite codes, increasing value
    return codes, e4m3_bits_to_f64(codes)


def f64_to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """Round to the nearest E4M3 value, ties to the even code, saturating.

    Magnitudes above 448 become 448 (the "satfinite" conversion); the sign is
    kept, so negative values that round to zero give the code 0x80.  NaN maps
    to 0x7F.
    """
    x = np.asarray(x, dtype=np.float64)
    codes, vals = _e4m3_table()
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(vals, a, side="left"), 0, vals.size - 1)   # first value >= a
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - vals[lo], vals[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (codes[hi] % 2 == 0))
    c = np.where(pick_hi, codes[hi], codes[lo]).astype(np.uint8)
    c = np.where(np.signbit(x), c | np.uint8(0x80), c).astype(np.uint8)
    return np.where(np.isnan(x), np.uint8(0x7F), c).astype(np.uint8)


def repack_fwd_fp8(S: np.ndarray, P: int) -> np.ndarray:
    """Mode 0 with the cast: ``[Np, C, H, D]`` bf16 bits -> ``[P, C, Np, Hl, D]`` E4M3 codes.

    The cast is elementwise, so it commutes with the index map: this is the
    bf16 repack followed by the conversion of every element.
    """
    return f64_to_e4m3_bits(bf16_bits_to_f64(repack_fwd(S, P)))


def layer_fwd_fp8(S: np.ndarray, P: int, N: int, scale: float, cu_seqlens=None,
                  rows: np.ndarray | None = None, workers: int = 1, causal: bool = False) -> np.ndarray:
    """The FP8 layer: repack with the E4M3 cast, attention on the cast values
    (exact, fp64), inverse repack of the output."""
    T8 = repack_fwd_fp8(S, P)
    O = attention_heads(T8, N, scale, cu_seqlens=cu_seqlens, rows=rows, workers=workers, causal=causal,
                        decode=e4m3_bits_to_f64)
    return output_repack_bwd(O)


# ---------------------------------------------------------------------------
# QKV prologue (per-head RMSNorm + partial rotate-half RoPE), fused before the
# repack.  Source: "hao-ai-lab FastVideo, compare aryan/h3-nvfp4-stack-speedups
# ...main", fastvideo/models/dits/minimax_h3_fusions/mk/qkv_prologue.py (module
# docstring and kernel): per 128-wide (token, head) row of Q and of K,
#   y = x / sqrt(mean(x^2) + eps) * w        (eps = 1e-5, w the per-channel norm weight)
#   y'[i] = y[i] cos[i] + rot(y)[i] sin[i]   for i < rotary_dim, where
#   rot(y)[i] = -y[i + rotary_dim/2] (i < rotary_dim/2), y[i - rotary_dim/2] otherwise,
#   channels i >= rotary_dim unchanged; V (and any further plane) copied verbatim.
# cos / sin are per-token tables [S, rotary_dim].
# ---------------------------------------------------------------------------

PROLOGUE_EPS = 1e-5


def rms_norm_rows(x: np.ndarray, w: np.ndarray, eps: float = PROLOGUE_EPS) -> np.ndarray:
    """RMSNorm over the last axis in fp64: x / sqrt(mean(x^2) + eps) * w."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(w, dtype=np.float64)


def rope_rotate_half(y: np.ndarray, cos: np.ndarray, sin: np.ndarray, rotary_dim: int) -> np.ndarray:
    """Partial rotate-half RoPE on the first rotary_dim channels of the last axis.

    y: [..., D]; cos, sin: broadcastable to [..., rotary_dim].
    """
    y = np.asarray(y, dtype=np.float64)
    half = rotary_dim // 2
    out = y.copy()
    a, b = y[..., :half], y[..., half:rotary_dim]
    c = np.asarray(cos, dtype=np.float64)
    s = np.asarray(sin, dtype=np.float64)
    out[..., :half] = a * c[..., :half] - b * s[..., :half]
    out[..., half:rotary_dim] = b * c[..., half:rotary_dim] + a * s[..., half:rotary_dim]
    return out


def qkv_prologue(S: np.ndarray, wq: np.ndarray, wk: np.ndarray, cos: np.ndarray, sin: np.ndarray,
                 rotary_dim: int, eps: float = PROLOGUE_EPS) -> np.ndarray:
    """The prologue on the sequence-sharded pack, in fp64.

    S: ``[Np, C, H, D]`` uint16 bf16 bits (planes Q, K, V[, G]); wq, wk: ``[D]``
    bf16 bits; cos, sin: ``[Np, rotary_dim]`` bf16 bits.  Returns fp64
    ``[Np, C, H, D]``: planes 0 and 1 normalised and rotated, the others the
    exact input values.
    """
    x = bf16_bits_to_f64(S).reshape(S.shape)
    c = bf16_bits_to_f64(cos).reshape(cos.shape)[:, None, :]       # [Np, 1, rd] broadcast over heads
    s = bf16_bits_to_f64(sin).reshape(sin.shape)[:, None, :]
    out = x.copy()
    for plane, w in ((0, wq), (1, wk)):
        y = rms_norm_rows(x[:, plane], bf16_bits_to_f64(w), eps)
        out[:, plane] = rope_rotate_half(y, c, s, rotary_dim)
    return out


def prologue_repack_fwd(S: np.ndarray, P: int, wq, wk, cos, sin, rotary_dim: int,
                        eps: float = PROLOGUE_EPS) -> np.ndarray:
    """Prologue, then the mode-0 index map: fp64 ``[P, C, Np, Hl, D]``."""
    y = qkv_prologue(S, wq, wk, cos, sin, rotary_dim, eps)
    Np, C, H, D = y.shape
    Nl, Hl = Np // P, H // P
    return np.ascontiguousarray(y.reshape(P, Nl, C, P, Hl, D).transpose(3, 2, 0, 1, 4, 5)).reshape(P, C, Np, Hl, D)


# ---------------------------------------------------------------------------
# Attention backward (the gradient the Ulysses transport carries back under
# the forward's plan: _FusedUlyssesA2A.backward runs the inverse map on the
# incoming gradient).  Written from the definition O = softmax(s Q K^T) V:
#   P = softmax(s Q K^T), dV = P^T dO, dP = dO V^T,
#   dS = P o (dP - rowsum(dP o P)),  dQ = s dS K,  dK = s dS^T Q.
# rowsum(dP o P) equals rowsum(dO o O) (both are sum_m P_nm (dO_n . V_m)).
# ---------------------------------------------------------------------------

def attention_rows_bwd(q, k, v, do, scale: float, causal_offset: int | None = None):
    """fp64 gradients of O = softmax(scale q k^T) v for query rows q [R, D].

    With causal_offset = a, query row i (global index a + i... relative to the
    key block start) sees keys 0..i only.  Returns (dq [R, D], dk [M, D], dv [M, D]).
    """
    q, k, v, do = (np.asarray(t, dtype=np.float64) for t in (q, k, v, do))
    z = scale * (q @ k.T)
    if causal_offset is not None:
        R, M = z.shape
        mask = np.arange(M)[None, :] > (np.arange(R)[:, None] + causal_offset)
        z = np.where(mask, -np.inf, z)
    z = z - z.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    dv = p.T @ do
    dp = do @ v.T
    ds = p * (dp - (dp * p).sum(axis=1, keepdims=True))
    return scale * (ds @ k), scale * (ds.T @ q), dv


def attention_bwd_sampled(q, k, v, do, scale: float, q_rows, k_rows, causal: bool = False, block: int = 512):
    """dQ at query rows ``q_rows`` and dK, dV at key rows ``k_rows`` of one
    (head, segment) block, fp64, from the same definition as
    ``attention_rows_bwd``: every query row's softmax row, dP row and
    rowsum(dP o P) are formed in full.  Query rows are visited ``block`` at a
    time only to bound memory (each row's terms are independent of the
    others).  Causal: query n sees keys m <= n (indices within the segment).
    Returns (dq [len(q_rows), D], dk [len(k_rows), D], dv [len(k_rows), D]).
    """
    q, k, v, do = (np.asarray(t, dtype=np.float64) for t in (q, k, v, do))
    R, M = q.shape[0], k.shape[0]
    qr = np.asarray(q_rows, dtype=np.int64)
    kr = np.asarray(k_rows, dtype=np.int64)

    def row_terms(idx):
        z = scale * (q[idx] @ k.T)
        if causal:
            z = np.where(np.arange(M)[None, :] > idx[:, None], -np.inf, z)
        z = z - z.max(axis=1, keepdims=True)
        p = np.exp(z)
        p /= p.sum(axis=1, keepdims=True)
        dp = do[idx] @ v.T
        return p, p * (dp - (dp * p).sum(axis=1, keepdims=True))

    _, ds = row_terms(qr)
    dq = scale * (ds @ k)
    dk = np.zeros((kr.size, q.shape[1]))
    dv = np.zeros((kr.size, v.shape[1]))
    for i0 in range(0, R if kr.size else 0, block):
        idx = np.arange(i0, min(R, i0 + block))
        p, ds = row_terms(idx)
        dk += scale * (ds[:, kr].T @ q[idx])
        dv += p[:, kr].T @ do[idx]
    return dq, dk, dv


def attention_heads_bwd(T: np.ndarray, dO: np.ndarray, N: int, scale: float, cu_seqlens=None,
                        causal: bool = False) -> np.ndarray:
    """Gradients of step two for every head-sharded slab.

    T: head-sharded ``[P, C, Np, Hl, D]`` uint16 (Q, K, V planes); dO: fp64 or
    uint16 ``[P, Np, Hl, D]``.  Returns fp64 ``[P, 3, Np, Hl, D]`` (dQ, dK, dV);
    pad rows and the gate plane get no gradient (zeros).
    """
    P, C, Np, Hl, D = T.shape
    g = dO if dO.dtype != np.uint16 else bf16_bits_to_f64(dO)
    out = np.zeros((P, 3, Np, Hl, D), dtype=np.float64)
    for r in range(P):
        for j in range(Hl):
            for a, b in segments_from_cu_seqlens(cu_seqlens, N):
                if b <= a:
                    continue
                q = bf16_bits_to_f64(T[r, 0, a:b, j])
                k = bf16_bits_to_f64(T[r, 1, a:b, j])
                v = bf16_bits_to_f64(T[r, 2, a:b, j])
                dq, dk, dv = attention_rows_bwd(q, k, v, g[r, a:b, j], scale, 0 if causal else None)
                out[r, 0, a:b, j], out[r, 1, a:b, j], out[r, 2, a:b, j] = dq, dk, dv
    return out


def layer_bwd(S: np.ndarray, dOut: np.ndarray, P: int, N: int, scale: float, cu_seqlens=None,
              causal: bool = False) -> np.ndarray:
    """Backward of the whole layer: dOut ``[Np, H, D]`` -> d(S) ``[Np, 3, H, D]`` fp64.

    Mode 0 on the output gradient, attention backward per slab, mode 1 on the
    three input gradients (the transport's backward runs the inverse map).
    """
    T = repack_fwd(S, P)
    Np, H, D = dOut.shape
    g = dOut if dOut.dtype != np.uint16 else bf16_bits_to_f64(dOut)
    dO_T = np.ascontiguousarray(g.reshape(P, Np // P, 1, P, H // P, D).transpose(3, 2, 0, 1, 4, 5)).reshape(
        P, Np, H // P, D)
    dT = attention_heads_bwd(T, dO_T, N, scale, cu_seqlens, causal)
    return np.ascontiguousarray(dT.reshape(P, 3, P, Np // P, H // P, D).transpose(2, 3, 1, 0, 4, 5)).reshape(
        Np, 3, H, D)
