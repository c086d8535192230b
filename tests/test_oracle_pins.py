"""Pins for the CPU oracle: facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: byte counts
the pages print, the inverse/identity properties of the all-to-all, a
brute-force index loop, closed-form softmax results, and the Ulysses
invariant that the whole layer equals plain multi-head attention on the
unsharded sequence.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import ulysses_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(rng, shape):
    # arbitrary 16-bit patterns, NaN/Inf/denormal included: the repack is a bit copy
    return rng.integers(0, 1 << 16, size=shape, dtype=np.uint16)


def _bf16_normal(rng, shape, scale=1.0):
    return orc.f64_to_bf16_bits(rng.standard_normal(shape) * scale)


# ---------------------------------------------------------------- window bytes

def test_window_bytes_match_printed_values():
    g = json.load(open(os.path.join(GOLDEN, "window_bytes.json")))
    for case in g["per_plane"]:
        assert orc.plane_bytes_per_rank(case["tokens"], case["heads"], case["head_dim"], case["sp"]) == case["bytes"]
    for case in g["whole_operand"]:
        per_plane = orc.plane_bytes_per_rank(case["tokens"], case["heads"], case["head_dim"], case["sp"])
        assert per_plane * case["planes"] == case["bytes"]
    b = g["half_gib_boundary"]
    lim = b["limit_bytes"]
    lo, hi = b["below"], b["above"]
    assert orc.plane_bytes_per_rank(lo["tokens"], lo["heads"], lo["head_dim"], lo["sp"]) <= lim
    assert orc.plane_bytes_per_rank(hi["tokens"], hi["heads"], hi["head_dim"], hi["sp"]) > lim
    assert orc.MAX_WINDOW_BYTES == g["window_cap_bytes"]["value"]


def test_auto_plane_chunk_one_plane_per_launch_at_250k():
    # 896,000,000 B per plane: two planes exceed 1 GiB, so one plane per launch
    assert orc.auto_plane_chunk(250_000, 56, 128, 4, planes=4) == 1
    # 32,000 tokens: all four planes (458,752,000 B) fit in one window
    assert orc.auto_plane_chunk(32_000, 56, 128, 4, planes=4) == 4
    # a plane larger than the window cannot be exchanged at all
    assert orc.auto_plane_chunk(400_000, 56, 128, 4, planes=3) == 0


def test_padding_sizes():
    assert orc.padded_tokens(19_394, 4) == 19_396
    assert orc.padded_tokens(1024, 2) == 1024
    assert orc.padded_tokens(104_448, 8) == 104_448
    assert orc.local_tokens(19_394, 4) == 4849


# ---------------------------------------------------------------- repack

@pytest.mark.parametrize("P,C,Nl,H,D", [(1, 3, 5, 4, 8), (2, 3, 4, 8, 4), (4, 4, 3, 8, 2), (8, 3, 2, 56, 2)])
def test_repack_round_trip_is_identity(P, C, Nl, H, D):
    rng = np.random.default_rng(P * 100 + C)
    S = _bits(rng, (P * Nl, C, H, D))
    T = orc.repack_fwd(S, P)
    assert T.shape == (P, C, P * Nl, H // P, D)
    assert np.array_equal(orc.repack_bwd(T), S)
    # and the other way round
    T2 = _bits(rng, T.shape)
    assert np.array_equal(orc.repack_fwd(orc.repack_bwd(T2), P), T2)


def test_repack_p1_is_identity():
    rng = np.random.default_rng(7)
    S = _bits(rng, (9, 4, 6, 8))
    T = orc.repack_fwd(S, 1)
    assert np.array_equal(T[0].transpose(1, 0, 2, 3), S)


def _brute_force_fwd(S, P):
    # literal per-element loop over the destination index set
    Np, C, H, D = S.shape
    Hl = H // P
    T = np.zeros((P, C, Np, Hl, D), dtype=S.dtype)
    for r in range(P):
        for c in range(C):
            for n in range(Np):
                for j in range(Hl):
                    for d in range(D):
                        T[r, c, n, j, d] = S[n, c, r * Hl + j, d]
    return T


def _per_rank_all_to_all(S, P):
    # the mode-0 shape map as P separate ranks: rank q holds x_q [C, Nl, H, D]
    # (sequence shard); it sends head block r to rank r, which concatenates the
    # blocks it receives in source-rank order along the sequence
    Np, C, H, D = S.shape
    Nl, Hl = Np // P, H // P
    local = [S[q * Nl:(q + 1) * Nl].transpose(1, 0, 2, 3) for q in range(P)]
    out = []
    for r in range(P):
        recv = [local[q][:, :, r * Hl:(r + 1) * Hl, :] for q in range(P)]
        out.append(np.concatenate(recv, axis=1))   # [C, Np, Hl, D]
    return np.stack(out)


def test_repack_matches_brute_force_loop_and_per_rank_exchange():
    rng = np.random.default_rng(11)
    for P, C, Nl, H, D in [(2, 3, 3, 4, 2), (4, 4, 2, 8, 3), (3, 3, 2, 6, 2)]:
        S = _bits(rng, (P * Nl, C, H, D))
        T = orc.repack_fwd(S, P)
        assert np.array_equal(T, _brute_force_fwd(S, P))
        assert np.array_equal(T, _per_rank_all_to_all(S, P))


def test_repack_rejects_indivisible_heads():
    with pytest.raises(ValueError):
        orc.repack_fwd(np.zeros((4, 3, 6, 2), np.uint16), 4)


# ---------------------------------------------------------------- bf16 helpers

def test_bf16_widening_known_patterns():
    bits = np.array([0x3F80, 0xC000, 0x0000, 0x8000, 0x3F81, 0x7F80, 0x0001], dtype=np.uint16)
    f = orc.bf16_bits_to_f64(bits)
    assert f[0] == 1.0 and f[1] == -2.0 and f[2] == 0.0 and math.copysign(1, f[3]) == -1
    assert f[4] == 1.0 + 2.0 ** -7
    assert math.isinf(f[5])
    assert f[6] == 2.0 ** -133


def test_bf16_rounding_ties_to_even():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to the even pattern 0x3F80
    assert orc.f64_to_bf16_bits(np.array([1.0 + 2.0 ** -8]))[0] == 0x3F80
    # 1 + 3*2^-8 is halfway between 1+2^-7 (odd, 0x3F81) and 1+2^-6 (even, 0x3F82)
    assert orc.f64_to_bf16_bits(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 0x3F82
    assert orc.f64_to_bf16_bits(np.array([-2.0]))[0] == 0xC000
    assert orc.f64_to_bf16_bits(np.array([float("nan")]))[0] == 0x7FC0


# ---------------------------------------------------------------- attention closed forms

S128 = 1.0 / math.sqrt(128.0)


def test_scale_is_one_over_sqrt_128():
    assert orc.softmax_scale(128) == S128


def test_two_keys_weights_three_to_one():
    # logits differ by ln 3 after scaling => weights exactly 3/4 and 1/4
    D = 128
    q = np.zeros((1, D)); q[0, 0] = 1.0
    k = np.zeros((2, D)); k[0, 0] = math.log(3.0) * math.sqrt(128.0)
    v = np.zeros((2, D)); v[0, :] = 4.0; v[1, :] = -8.0
    o = orc.attention_rows(q, k, v, S128)
    assert np.allclose(o, 0.75 * 4.0 + 0.25 * -8.0, rtol=0, atol=1e-13)


def test_uniform_keys_give_mean_of_v():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((5, 16))
    k = np.tile(rng.standard_normal((1, 16)), (9, 1))
    v = rng.standard_normal((9, 16))
    o = orc.attention_rows(q, k, v, 0.3)
    assert np.allclose(o, np.tile(v.mean(axis=0), (5, 1)), rtol=0, atol=1e-13)


def test_single_key_returns_its_value():
    rng = np.random.default_rng(4)
    v = rng.standard_normal((1, 8))
    o = orc.attention_rows(rng.standard_normal((3, 8)), rng.standard_normal((1, 8)), v, 1.0)
    assert np.allclose(o, np.tile(v, (3, 1)), rtol=0, atol=1e-15)


def test_key_permutation_invariance():
    rng = np.random.default_rng(5)
    q, k, v = rng.standard_normal((4, 8)), rng.standard_normal((12, 8)), rng.standard_normal((12, 8))
    perm = rng.permutation(12)
    assert np.allclose(orc.attention_rows(q, k, v, 0.5), orc.attention_rows(q, k[perm], v[perm], 0.5),
                       rtol=0, atol=1e-13)


def _brute_force_softmax(q, k, v, scale):
    out = []
    for qi in q:
        logits = [scale * math.fsum(float(a) * float(b) for a, b in zip(qi, kj)) for kj in k]
        m = max(logits)
        w = [math.exp(z - m) for z in logits]
        tot = math.fsum(w)
        out.append([math.fsum(wj * float(vj[d]) for wj, vj in zip(w, v)) / tot for d in range(v.shape[1])])
    return np.array(out)


@pytest.mark.parametrize("M", [1, 7, 64])
def test_matches_brute_force_softmax(M):
    rng = np.random.default_rng(M)
    q, k, v = rng.standard_normal((6, 16)), rng.standard_normal((M, 16)), rng.standard_normal((M, 16))
    assert np.allclose(orc.attention_rows(q, k, v, 0.25), _brute_force_softmax(q, k, v, 0.25),
                       rtol=0, atol=1e-12)


# ---------------------------------------------------------------- layer invariants

def _plain_mha(S, N, scale, segs):
    # multi-head attention on the unsharded sequence, head by head (no repack)
    Np, C, H, D = S.shape
    out = np.zeros((Np, H, D))
    for h in range(H):
        for a, b in segs:
            q = orc.bf16_bits_to_f64(S[a:b, 0, h])
            k = orc.bf16_bits_to_f64(S[a:b, 1, h])
            v = orc.bf16_bits_to_f64(S[a:b, 2, h])
            out[a:b, h] = _brute_force_softmax(q, k, v, scale) if b - a <= 8 else orc.attention_rows(q, k, v, scale)
    return out


@pytest.mark.parametrize("P,N,H,C", [(2, 16, 4, 3), (4, 14, 8, 4), (1, 9, 2, 3), (3, 10, 6, 3)])
def test_layer_equals_plain_multi_head_attention(P, N, H, C):
    rng = np.random.default_rng(P * 31 + N)
    D = 8
    Np = orc.padded_tokens(N, P)
    S = _bf16_normal(rng, (Np, C, H, D))
    S[N:] = 0                                      # pad rows are zero in the input
    got = orc.layer_fwd(S, P, N, 0.35)
    want = _plain_mha(S, N, 0.35, [(0, N)])
    assert np.allclose(got, want, rtol=0, atol=1e-12)
    assert np.all(got[N:] == 0.0)                   # pad query rows give zero


def test_varlen_equals_independent_segments():
    rng = np.random.default_rng(21)
    P, H, D, C = 2, 4, 8, 3
    cu = [0, 5, 6, 13, 16]
    N = cu[-1]
    S = _bf16_normal(rng, (N, C, H, D))
    got = orc.layer_fwd(S, P, N, 0.5, cu_seqlens=cu)
    want = _plain_mha(S, N, 0.5, list(zip(cu, cu[1:])))
    assert np.allclose(got, want, rtol=0, atol=1e-12)
    # a segment of length one returns its own value row
    assert np.allclose(got[5], orc.bf16_bits_to_f64(S[5, 2]), atol=1e-15)


def test_padding_keys_never_attended():
    # padded rows hold large values; results must not change
    rng = np.random.default_rng(22)
    P, N, H, D = 4, 10, 4, 8
    Np = orc.padded_tokens(N, P)
    S = _bf16_normal(rng, (Np, 3, H, D))
    S[N:] = 0
    base = orc.layer_fwd(S, P, N, 0.4)
    S2 = S.copy()
    S2[N:] = orc.f64_to_bf16_bits(np.full((Np - N, 3, H, D), 50.0))
    got = orc.layer_fwd(S2, P, N, 0.4)
    assert np.array_equal(got[:N], base[:N]) and np.all(got[N:] == 0)


def test_row_sampling_matches_full_rows():
    rng = np.random.default_rng(23)
    P, N, H, D = 2, 40, 4, 8
    S = _bf16_normal(rng, (N, 3, H, D))
    rows = orc.sample_rows(N, 9, seed=1, cu_seqlens=[0, 17, 40])
    assert {0, 16, 17, 39} <= set(rows.tolist())
    full = orc.layer_fwd(S, P, N, 0.3, cu_seqlens=[0, 17, 40])
    part = orc.layer_fwd(S, P, N, 0.3, cu_seqlens=[0, 17, 40], rows=rows)
    assert np.array_equal(part, full[rows])


def test_flop_count():
    assert orc.attention_flops(1024, 8, 128) == 4 * 1024 ** 2 * 8 * 128
    cu = [0, 52224, 83456, 104448]
    assert orc.attention_flops(104448, 56, 128, cu) == sum(4 * L ** 2 * 56 * 128 for L in (52224, 31232, 20992))


# ---------------------------------------------------------------- causal variant

def _plain_causal_mha(S, segs, scale):
    Np, C, H, D = S.shape
    out = np.zeros((Np, H, D))
    for h in range(H):
        for a, b in segs:
            for n in range(a, b):
                q = orc.bf16_bits_to_f64(S[n:n + 1, 0, h])
                k = orc.bf16_bits_to_f64(S[a:n + 1, 1, h])
                v = orc.bf16_bits_to_f64(S[a:n + 1, 2, h])
                out[n, h] = _brute_force_softmax(q, k, v, scale)[0]
    return out


@pytest.mark.parametrize("P,N,H,cu", [(2, 12, 4, None), (4, 10, 8, None), (2, 14, 4, [0, 5, 6, 14])])
def test_causal_layer_equals_plain_causal_attention(P, N, H, cu):
    rng = np.random.default_rng(40 + N)
    D = 8
    Np = orc.padded_tokens(N, P)
    S = _bf16_normal(rng, (Np, 3, H, D))
    S[N:] = 0
    got = orc.layer_fwd(S, P, N, 0.4, cu_seqlens=cu, causal=True)
    segs = [(0, N)] if cu is None else list(zip(cu, cu[1:]))
    want = _plain_causal_mha(S, segs, 0.4)
    assert np.allclose(got[:N], want[:N], rtol=0, atol=1e-12)
    assert np.all(got[N:] == 0)


def test_causal_first_row_of_each_segment_is_its_value():
    # the first query of a segment sees exactly one key: its own
    rng = np.random.default_rng(41)
    cu = [0, 4, 9]
    S = _bf16_normal(rng, (9, 3, 2, 8))
    got = orc.layer_fwd(S, 1, 9, 0.7, cu_seqlens=cu, causal=True)
    for a in cu[:-1]:
        assert np.array_equal(got[a], orc.bf16_bits_to_f64(S[a, 2]))


def test_causal_last_row_equals_non_causal_last_row():
    rng = np.random.default_rng(42)
    S = _bf16_normal(rng, (8, 3, 2, 8))
    full = orc.layer_fwd(S, 2, 8, 0.3)
    causal = orc.layer_fwd(S, 2, 8, 0.3, causal=True)
    assert np.allclose(full[7], causal[7], rtol=0, atol=1e-12)
    assert not np.allclose(full[0], causal[0])


def test_causal_flop_count():
    assert orc.attention_flops(4, 1, 1, causal=True) == 4 * (1 + 2 + 3 + 4)
    assert orc.attention_flops(6, 2, 8, [0, 2, 6], causal=True) == 4 * 2 * 8 * ((1 + 2) + (1 + 2 + 3 + 4))


# ---------------------------------------------------------------- QKV prologue (RMSNorm + partial RoPE)

def test_rms_norm_closed_forms():
    # a constant row c: x / sqrt(c^2 + eps) -> c / sqrt(c^2 + eps) in every channel
    x = np.full((1, 128), 3.0)
    y = orc.rms_norm_rows(x, np.ones(128), 1e-5)
    assert np.allclose(y, 3.0 / math.sqrt(9.0 + 1e-5), rtol=0, atol=1e-15)
    # the weight scales channel by channel; the output's rms is 1 (up to eps) for unit weight
    rng = np.random.default_rng(50)
    x = rng.standard_normal((7, 128)) * 5
    y = orc.rms_norm_rows(x, np.ones(128), 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=0, atol=1e-13)
    w = rng.standard_normal(128)
    assert np.allclose(orc.rms_norm_rows(x, w, 0.0), y * w, rtol=0, atol=1e-13)


def test_rope_identity_quarter_turn_and_pair_norms():
    rng = np.random.default_rng(51)
    y = rng.standard_normal((5, 128))
    rd = 96
    one, zero = np.ones((5, rd)), np.zeros((5, rd))
    assert np.array_equal(orc.rope_rotate_half(y, one, zero, rd), y)
    # cos 0, sin 1: a quarter turn of every (i, i + 48) pair
    q = orc.rope_rotate_half(y, zero, one, rd)
    assert np.array_equal(q[:, :48], -y[:, 48:96]) and np.array_equal(q[:, 48:96], y[:, :48])
    assert np.array_equal(q[:, 96:], y[:, 96:])        # channels past rotary_dim untouched
    # any angle (same angle for i and i + 48) keeps each pair's length
    th = rng.uniform(-3, 3, (5, 48))
    c = np.concatenate([np.cos(th), np.cos(th)], axis=1)
    s = np.concatenate([np.sin(th), np.sin(th)], axis=1)
    r = orc.rope_rotate_half(y, c, s, rd)
    assert np.allclose(r[:, :48] ** 2 + r[:, 48:96] ** 2, y[:, :48] ** 2 + y[:, 48:96] ** 2, rtol=0, atol=1e-12)
    # rotating by th then by -th restores the input
    back = orc.rope_rotate_half(r, c, -s, rd)
    assert np.allclose(back, y, rtol=0, atol=1e-12)


def test_prologue_then_repack_commutes_and_copies_v():
    rng = np.random.default_rng(52)
    P, N, C, H, D, rd = 2, 6, 4, 4, 128, 96
    S = _bf16_normal(rng, (N, C, H, D))
    wq, wk = _bf16_normal(rng, (D,)), _bf16_normal(rng, (D,))
    cos, sin = _bf16_normal(rng, (N, rd)), _bf16_normal(rng, (N, rd))
    T = orc.prologue_repack_fwd(S, P, wq, wk, cos, sin, rd)
    # equals repack of the prologue output (per-row ops commute with the index map)
    y = orc.qkv_prologue(S, wq, wk, cos, sin, rd)
    assert np.array_equal(orc.repack_fwd(orc.f64_to_bf16_bits(y), P), orc.f64_to_bf16_bits(T))
    # planes 2 and 3 are the input, exactly
    assert np.array_equal(T[:, 2:], orc.bf16_bits_to_f64(orc.repack_fwd(S, P)[:, 2:]).reshape(T[:, 2:].shape))
    # head-by-head against a direct per-row formula for one element
    n, h = 3, 2
    x = orc.bf16_bits_to_f64(S[n, 1, h])
    yk = x / math.sqrt(np.mean(x * x) + 1e-5) * orc.bf16_bits_to_f64(wk)
    cc, ss = orc.bf16_bits_to_f64(cos[n]), orc.bf16_bits_to_f64(sin[n])
    i = 10
    want = yk[i] * cc[i] - yk[i + 48] * ss[i]
    r, j = h // (H // P), h % (H // P)
    assert abs(T[r, 1, n, j, i] - want) < 1e-12


# ---------------------------------------------------------------- attention backward

def _loss(q, k, v, g, scale, causal):
    z = scale * (q @ k.T)
    if causal:
        z = np.where(np.arange(k.shape[0])[None, :] > np.arange(q.shape[0])[:, None], -np.inf, z)
    z = z - z.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    return float(np.sum((p @ v) * g))


@pytest.mark.parametrize("causal", [False, True])
def test_attention_backward_matches_finite_differences(causal):
    # central differences of L = sum(O * G) pin every gradient independently of the formulas
    rng = np.random.default_rng(60 + causal)
    R, D = 5, 6
    q, k, v, g = (rng.standard_normal((R, D)) for _ in range(4))
    dq, dk, dv = orc.attention_rows_bwd(q, k, v, g, 0.7, 0 if causal else None)
    h = 1e-6
    for X, dX in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            old = X[idx]
            X[idx] = old + h
            lp = _loss(q, k, v, g, 0.7, causal)
            X[idx] = old - h
            lm = _loss(q, k, v, g, 0.7, causal)
            X[idx] = old
            num[idx] = (lp - lm) / (2 * h)
        assert np.allclose(dX, num, rtol=1e-6, atol=1e-8), np.abs(dX - num).max()


def test_backward_row_term_identity():
    # rowsum(dP o P) == rowsum(dO o O)
    rng = np.random.default_rng(62)
    q, k, v, g = (rng.standard_normal((7, 8)) for _ in range(4))
    z = 0.5 * q @ k.T
    p = np.exp(z - z.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    assert np.allclose(((g @ v.T) * p).sum(1), (g * (p @ v)).sum(1), rtol=0, atol=1e-12)


def test_layer_backward_is_transposed_repack_of_head_gradients():
    # sum over all gradients of the layer equals the per-head plain MHA gradients, regrouped
    rng = np.random.default_rng(63)
    P, N, H, D = 2, 6, 4, 8
    S = _bf16_normal(rng, (N, 3, H, D))
    G = rng.standard_normal((N, H, D))
    dS = orc.layer_bwd(S, G, P, N, 0.4)
    for h in range(H):
        q, k, v = (orc.bf16_bits_to_f64(S[:, c, h]) for c in range(3))
        dq, dk, dv = orc.attention_rows_bwd(q, k, v, G[:, h], 0.4)
        assert np.allclose(dS[:, 0, h], dq, atol=1e-12) and np.allclose(dS[:, 1, h], dk, atol=1e-12)
        assert np.allclose(dS[:, 2, h], dv, atol=1e-12)
    # varlen: cross-segment gradients vanish
    dS2 = orc.layer_bwd(S, G, P, N, 0.4, cu_seqlens=[0, 3, 6])
    q, k, v = (orc.bf16_bits_to_f64(S[:3, c, 0]) for c in range(3))
    dq, dk, dv = orc.attention_rows_bwd(q, k, v, G[:3, 0], 0.4)
    assert np.allclose(dS2[:3, 1, 0], dk, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_backward_equals_full_rows(causal):
    # the row-sampled backward reduces to the full one (pinned above by finite differences)
    rng = np.random.default_rng(64 + causal)
    R, D = 37, 8
    q, k, v, g = (rng.standard_normal((R, D)) for _ in range(4))
    dq, dk, dv = orc.attention_rows_bwd(q, k, v, g, 0.6, 0 if causal else None)
    qr, kr = np.array([0, 5, 36, 17]), np.array([36, 0, 11])
    sq, sk, sv = orc.attention_bwd_sampled(q, k, v, g, 0.6, qr, kr, causal, block=5)
    assert np.allclose(sq, dq[qr], rtol=0, atol=1e-12)
    assert np.allclose(sk, dk[kr], rtol=0, atol=1e-12)
    assert np.allclose(sv, dv[kr], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- FP8 (E4M3) cast

def test_e4m3_decode_known_codes():
    # values fixed by the format: bias 7, 3 mantissa bits, subnormals below 2^-6, max 448
    table = {0x00: 0.0, 0x38: 1.0, 0x40: 2.0, 0x3C: 1.5, 0x7E: 448.0, 0x08: 2.0 ** -6, 0x01: 2.0 ** -9,
             0x07: 7 * 2.0 ** -9, 0x0F: 1.875 * 2.0 ** -6, 0xB8: -1.0, 0xFE: -448.0, 0x30: 0.5}
    codes = np.array(list(table), dtype=np.uint8)
    np.testing.assert_array_equal(orc.e4m3_bits_to_f64(codes), np.array(list(table.values())))
    assert np.isnan(orc.e4m3_bits_to_f64(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def test_e4m3_encode_rounding_ties_and_saturation():
    cases = [
        (1.0625, 0x38),        # halfway 1 / 1.125: even code (mantissa 0)
        (1.1875, 0x3A),        # halfway 1.125 / 1.25: even code 1.25
        (1.0624, 0x38), (1.0626, 0x39),
        (2.0 ** -10, 0x00),    # halfway 0 / 2^-9: even code 0
        (3 * 2.0 ** -10, 0x02),  # halfway 2^-9 / 2^-8: even code 2^-8
        (464.0, 0x7E), (1e6, 0x7E), (-1e6, 0xFE),   # saturation to +-448
        (-2.0 ** -11, 0x80),   # negative underflow keeps the sign
        (240.0, 0x77), (0.3, 0x2A),
    ]
    x = np.array([c[0] for c in cases])
    np.testing.assert_array_equal(orc.f64_to_e4m3_bits(x), np.array([c[1] for c in cases], dtype=np.uint8))
    assert orc.f64_to_e4m3_bits(np.array([np.nan]))[0] == 0x7F


def test_e4m3_round_trip_every_code_and_monotone():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = orc.e4m3_bits_to_f64(codes)
    back = orc.f64_to_e4m3_bits(vals)
    np.testing.assert_array_equal(orc.e4m3_bits_to_f64(back), vals)
    np.testing.assert_array_equal(back[codes != 0x80], codes[codes != 0x80])
    xs = np.linspace(-500, 500, 20001)
    dec = orc.e4m3_bits_to_f64(orc.f64_to_e4m3_bits(xs))
    assert np.all(np.diff(dec) >= 0)
    # nearest: no representable value is closer than the chosen one
    allv = orc.e4m3_bits_to_f64(np.arange(0x7F, dtype=np.uint8))
    a = np.abs(xs[np.abs(xs) <= 448])
    chosen = np.abs(orc.e4m3_bits_to_f64(orc.f64_to_e4m3_bits(a)))
    best = np.min(np.abs(allv[None, :] - a[:, None]), axis=1)
    np.testing.assert_allclose(np.abs(chosen - a), best, rtol=0, atol=0)


def test_e4m3_cast_of_bf16_values_matches_torch():
    torch = pytest.importorskip("torch")
    if not hasattr(torch, "float8_e4m3fn"):
        pytest.skip("torch without float8_e4m3fn")
    rng = np.random.default_rng(11)
    bits = _bf16_normal(rng, (4096,), scale=3.0)
    x = orc.bf16_bits_to_f64(bits)
    x = x[np.abs(x) <= 448]
    want = torch.tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(orc.f64_to_e4m3_bits(x), want)


def test_fp8_layer_is_exact_attention_on_cast_values():
    # the FP8 layer equals the bf16 layer's oracle run on inputs that are already
    # E4M3 values (the cast is then the identity), and the cast commutes with mode 0
    rng = np.random.default_rng(12)
    P, N, H, C = 2, 200, 4, 3
    S = _bf16_normal(rng, (N, C, H, 128))
    S8 = orc.f64_to_e4m3_bits(orc.bf16_bits_to_f64(S))
    S_exact = orc.f64_to_bf16_bits(orc.e4m3_bits_to_f64(S8))       # E4M3 values are bf16 values
    np.testing.assert_array_equal(orc.e4m3_bits_to_f64(S8), orc.bf16_bits_to_f64(S_exact))
    scale = 1.0 / math.sqrt(128)
    np.testing.assert_allclose(orc.layer_fwd_fp8(S, P, N, scale), orc.layer_fwd(S_exact, P, N, scale),
                               rtol=0, atol=1e-12)
    np.testing.assert_array_equal(orc.repack_fwd_fp8(S, P), orc.repack_fwd(S8.view(np.uint8), P))
