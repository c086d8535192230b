"""Attention backward and layer backward against the fp64 oracle.

Both forms of the backward are checked: the default one pass over the keys
(dQ added into an fp32 accumulator through L2 reductions) and the two-pass
deterministic form (plan flag ULYSSES_PLAN_DETERMINISTIC).

The GPU path rounds P and dS to bf16 for its tensor-core products (as the
forward rounds P), accumulates in fp32 and rounds the gradients to bf16 once.
Each bf16 rounding is a relative error of at most 2^-8 (RMS 1.66e-3, see
tests/_parity.py); summed over a 128-wide contraction with random signs they
stay well under 1% of the gradient's magnitude.  The bounds used: per
gradient tensor, max|gpu - ref| <= 2e-2 * max|ref|, mean|gpu - ref| <=
5e-3 * mean|ref| and rel-L2 <= 1e-2 (two roundings in quadrature, ~2.4e-3,
as for the forward output).
"""
import math

import numpy as np
import pytest
from _parity import check_attention

from oracle import ulysses_oracle as orc

pytestmark = pytest.mark.gpu

MAX_REL = 2e-2
MEAN_REL = 5e-3

CASES = [
    pytest.param(2, 1024, 8, None, False, 0, id="tiny"),
    pytest.param(4, 1001, 8, None, False, 1, id="ragged"),
    pytest.param(1, 300, 2, None, False, 2, id="P1"),
    pytest.param(2, 1000, 4, [0, 300, 301, 777, 1000], False, 3, id="varlen"),
    pytest.param(2, 1024, 8, None, True, 4, id="causal"),
    pytest.param(2, 700, 4, [0, 256, 300, 700], True, 5, id="causal-varlen"),
    pytest.param(2, 1000, 4, [0, 0, 300, 300, 1000], False, 6, id="varlen-empty-segments"),
    pytest.param(4, 5, 4, None, False, 7, id="N5"),
    pytest.param(56, 1000, 56, None, False, 8, id="P56-Hl1"),
    pytest.param(1, 129, 2, None, True, 9, id="causal-N129"),
]


def _grad(gpu, shape, seed):
    import torch
    g = torch.Generator(device=gpu)
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device=gpu).to(torch.bfloat16)


def _close(got, ref, what, record=True):
    err = np.abs(got - ref)
    mx, mn = np.abs(ref).max(), np.abs(ref).mean()
    assert err.max() <= MAX_REL * mx, (what, float(err.max()), float(mx))
    assert err.mean() <= MEAN_REL * mn, (what, float(err.mean()), float(mn))
    if record:
        check_attention(f"backward {what}", got, ref, max_abs=None, mean_abs=None)


FORMS = [pytest.param(False, id="one-pass"), pytest.param(True, id="two-pass")]


@pytest.mark.parametrize("deterministic", FORMS)
@pytest.mark.parametrize("P,N,H,cu,causal,seed", CASES)
def test_attention_backward_against_oracle(gpu, P, N, H, cu, causal, seed, deterministic):
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    plan = U.ulysses_plan(N, H, 128, P, 3, 0, 0, 0, cu, causal=causal, deterministic=deterministic)
    Np, Hl = plan.padded_tokens, H // P
    scale = 1.0 / math.sqrt(128)
    S = inputs.qkv_seq(N, H, P, 3, 100 + seed, gpu)
    T = torch.empty((P, 3, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_repack_fwd(plan, S, T)
    OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    lse = torch.empty(plan.lse_bytes // 4, dtype=torch.float32, device=gpu)
    U.ulysses_attn_fwd_lse(plan, T, OT, lse, scale)
    dO = _grad(gpu, (P, Np, Hl, 128), 200 + seed)
    dO[:, N:] = 0
    dT = torch.full((P, 3, Np, Hl, 128), float("nan"), dtype=torch.bfloat16, device=gpu)
    ws = torch.empty(plan.attn_bwd_workspace_bytes, dtype=torch.uint8, device=gpu)
    U.ulysses_attn_bwd(plan, T, OT, dO, lse, dT, ws, scale)
    torch.cuda.synchronize()
    assert U.ulysses_last_device_error(plan) == 0
    # the forward's lse: m + log2 l of every real row, against fp64
    T_bits = inputs.host_bits(T)
    ls = plan.lse_row_stride
    got_lse = lse.view(P * Hl, ls)[:, :N].cpu().numpy().astype(np.float64)
    ref = orc.attention_heads_bwd(T_bits, inputs.host_bits(dO), N, scale, cu, causal)
    got = dT.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    form = "two-pass" if deterministic else "one-pass"
    for c, name in enumerate(("dQ", "dK", "dV")):
        _close(got[:, c, :N], ref[:, c, :N], f"{name} {form}")
    assert np.all(got[:, :, N:] == 0)               # pad rows get no gradient
    # lse check: log2 of sum_m exp2(s log2e q.k) per row, fp64
    q = orc.bf16_bits_to_f64(T_bits[:, 0])
    k = orc.bf16_bits_to_f64(T_bits[:, 1])
    segs = orc.segments_from_cu_seqlens(cu, N)
    for r in range(P):
        for j in range(Hl):
            for a, b in segs:
                if b == a:
                    continue
                z = scale * (q[r, a:b, j] @ k[r, a:b, j].T) / math.log(2.0)
                if causal:
                    z = np.where(np.arange(b - a)[None, :] > np.arange(b - a)[:, None], -np.inf, z)
                mz = z.max(1, keepdims=True)
                want = (mz + np.log2(np.exp2(z - mz).sum(1, keepdims=True)))[:, 0]
                assert np.abs(got_lse[r * Hl + j, a:b] - want).max() < 1e-3


@pytest.mark.parametrize("deterministic", FORMS)
@pytest.mark.parametrize("P,N,H,cu,causal", [(2, 1024, 8, None, False), (4, 1001, 8, [0, 500, 1001], True)])
def test_layer_backward_against_oracle(gpu, P, N, H, cu, causal, deterministic):
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    plan = U.ulysses_plan(N, H, 128, P, 3, 0, 0, 0, cu, causal=causal, deterministic=deterministic)
    Np, Hl = plan.padded_tokens, H // P
    scale = 1.0 / math.sqrt(128)
    S = inputs.qkv_seq(N, H, P, 3, 300, gpu)
    # forward, keeping what the backward needs
    T = torch.empty((P, 3, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    lse = torch.empty(plan.lse_bytes // 4, dtype=torch.float32, device=gpu)
    U.ulysses_repack_fwd(plan, S, T)
    U.ulysses_attn_fwd_lse(plan, T, OT, lse, scale)
    dOut = _grad(gpu, (Np, H, 128), 301)
    dOut[N:] = 0
    dS = torch.full_like(S, float("nan"))
    ws = torch.empty(plan.layer_bwd_workspace_bytes, dtype=torch.uint8, device=gpu)
    U.ulysses_layer_bwd(plan, T, OT, lse, dOut, dS, ws)
    torch.cuda.synchronize()
    assert U.ulysses_last_device_error(plan) == 0
    ref = orc.layer_bwd(inputs.host_bits(S), inputs.host_bits(dOut), P, N, scale, cu, causal)
    got = dS.float().cpu().numpy().astype(np.float64)
    for c, name in enumerate(("dQ", "dK", "dV")):
        _close(got[:N, c], ref[:N, c], name)
    assert np.all(got[N:] == 0)


@pytest.mark.slow
@pytest.mark.parametrize("deterministic", FORMS)
@pytest.mark.parametrize("causal", [False, True])
def test_attention_backward_dit19k(gpu, causal, deterministic):
    """Video-DiT size (P=4, N=19,394, H=56), as the benchmark times it.

    Every head: sum_k dK[k] = 0 (each row of dS sums to zero) and
    sum_k dV[k] = sum_q dO[q] (each row of P sums to one).  Sampled rows against
    fp64: dQ at 256 queries of every head, dK / dV at 256 keys of two heads.
    """
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    P, N, H = 4, 19_394, 56
    plan = U.ulysses_plan(N, H, 128, P, 3, causal=causal, deterministic=deterministic)
    Np, Hl = plan.padded_tokens, H // P
    scale = 1.0 / math.sqrt(128)
    S = inputs.qkv_seq(N, H, P, 3, 1, gpu)
    T = torch.empty((P, 3, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_repack_fwd(plan, S, T)
    del S
    OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    lse = torch.empty(plan.lse_bytes // 4, dtype=torch.float32, device=gpu)
    U.ulysses_attn_fwd_lse(plan, T, OT, lse, scale)
    dO = _grad(gpu, (P, Np, Hl, 128), 210 + causal)
    dO[:, N:] = 0
    dT = torch.empty((P, 3, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    ws = torch.empty(plan.attn_bwd_workspace_bytes, dtype=torch.uint8, device=gpu)
    U.ulysses_attn_bwd(plan, T, OT, dO, lse, dT, ws, scale)
    torch.cuda.synchronize()
    assert U.ulysses_last_device_error(plan) == 0
    assert not dT[:, :, N:].any()
    # invariants on every head, fp64 sums of the bf16 gradients
    dK = dT[:, 1, :N].double()
    dV = dT[:, 2, :N].double()
    g = dO[:, :N].double()
    assert (dK.sum(1).abs() <= 1e-3 * dK.abs().sum(1) + 1e-6).all()
    assert ((dV.sum(1) - g.sum(1)).abs() <= 1e-3 * g.abs().sum(1) + 1e-6).all()
    del dK, dV, g
    # sampled rows
    rng = np.random.default_rng(7 + causal)
    qr = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 254, replace=False)]))
    kr = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 254, replace=False)]))
    iq, ik = torch.from_numpy(qr).to(gpu), torch.from_numpy(kr).to(gpu)
    got_q = dT[:, 0].index_select(1, iq).double().cpu().numpy()          # [P, R, Hl, D]
    got_k = dT[:, 1].index_select(1, ik).double().cpu().numpy()
    got_v = dT[:, 2].index_select(1, ik).double().cpu().numpy()
    T_bits = inputs.host_bits(T)
    dO_bits = inputs.host_bits(dO)
    full_heads = {(0, 0), (P - 1, Hl - 1)}
    pairs = {"dQ": ([], []), "dK": ([], []), "dV": ([], [])}
    for r in range(P):
        for j in range(Hl):
            q, k, v = (orc.bf16_bits_to_f64(T_bits[r, c, :N, j]) for c in range(3))
            g_h = orc.bf16_bits_to_f64(dO_bits[r, :N, j])
            sel = kr if (r, j) in full_heads else kr[:0]
            dq, dk, dv = orc.attention_bwd_sampled(q, k, v, g_h, scale, qr, sel, causal)
            _close(got_q[r, :, j], dq, f"dQ {r},{j}", record=False)
            pairs["dQ"][0].append(got_q[r, :, j])
            pairs["dQ"][1].append(dq)
            if sel.size:
                _close(got_k[r, :, j], dk, f"dK {r},{j}", record=False)
                _close(got_v[r, :, j], dv, f"dV {r},{j}", record=False)
                pairs["dK"][0].append(got_k[r, :, j])
                pairs["dK"][1].append(dk)
                pairs["dV"][0].append(got_v[r, :, j])
                pairs["dV"][1].append(dv)
    for name, (g_l, r_l) in pairs.items():
        form = "two-pass" if deterministic else "one-pass"
        check_attention(f"backward dit19k causal={causal} {form} {name} (sampled rows)", np.stack(g_l),
                        np.stack(r_l), max_abs=None, mean_abs=None)


@pytest.mark.parametrize("P,N,H,cu,causal", [(2, 1024, 8, None, False), (4, 1001, 8, [0, 500, 1001], True)])
def test_backward_repeatability(gpu, P, N, H, cu, causal):
    """The two-pass form gives the same bits on every run.  The one-pass form
    gives the same dK and dV bits (each key block's loop runs in one CTA in a
    fixed order); its dQ is summed by L2 reductions in whatever order the CTAs
    reach them, so two runs agree to within rounding: here within one bf16
    step of the larger value, plus 1e-6 of the tensor's largest magnitude for
    sums that cancel to near zero."""
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    scale = 1.0 / math.sqrt(128)
    runs = {}
    for det in (False, True):
        plan = U.ulysses_plan(N, H, 128, P, 3, 0, 0, 0, cu, causal=causal, deterministic=det)
        Np, Hl = plan.padded_tokens, H // P
        S = inputs.qkv_seq(N, H, P, 3, 400, gpu)
        T = torch.empty((P, 3, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
        U.ulysses_repack_fwd(plan, S, T)
        OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
        lse = torch.empty(plan.lse_bytes // 4, dtype=torch.float32, device=gpu)
        U.ulysses_attn_fwd_lse(plan, T, OT, lse, scale)
        dO = _grad(gpu, (P, Np, Hl, 128), 401)
        dO[:, N:] = 0
        ws = torch.empty(plan.attn_bwd_workspace_bytes, dtype=torch.uint8, device=gpu)
        outs = []
        for _ in range(3):
            dT = torch.full((P, 3, Np, Hl, 128), float("nan"), dtype=torch.bfloat16, device=gpu)
            U.ulysses_attn_bwd(plan, T, OT, dO, lse, dT, ws, scale)
            outs.append(dT)
        torch.cuda.synchronize()
        assert U.ulysses_last_device_error(plan) == 0
        runs[det] = outs
    for dT in runs[True][1:]:
        assert torch.equal(dT.view(torch.int16), runs[True][0].view(torch.int16))
    a = runs[False][0]
    for b in runs[False][1:]:
        assert torch.equal(b[:, 1:].view(torch.int16), a[:, 1:].view(torch.int16))
        x, y = a[:, 0].double(), b[:, 0].double()
        tol = 2.0 ** -7 * torch.maximum(x.abs(), y.abs()) + 1e-6 * x.abs().max()
        assert ((x - y).abs() <= tol).all()


@pytest.mark.slow
def test_attention_backward_long104k(gpu):
    """The largest layer (P=8, N=104,448, H=56) through the default one-pass
    backward, whose fp32 dQ accumulator is 2.99 GB here.  Every head: the
    invariants sum_k dK[k] = 0 and sum_k dV[k] = sum_q dO[q]; pad rows zero;
    dQ at 34 sampled query rows of one head per rank against fp64."""
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    P, N, H = 8, 104_448, 56
    plan = U.ulysses_plan(N, H, 128, P, 3)
    Np, Hl = plan.padded_tokens, H // P
    scale = 1.0 / math.sqrt(128)
    S = inputs.qkv_seq(N, H, P, 3, 3, gpu)
    T = torch.empty((P, 3, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_repack_fwd(plan, S, T)
    del S
    OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    lse = torch.empty(plan.lse_bytes // 4, dtype=torch.float32, device=gpu)
    U.ulysses_attn_fwd_lse(plan, T, OT, lse, scale)
    dO = _grad(gpu, (P, Np, Hl, 128), 230)
    dO[:, N:] = 0
    dT = torch.empty((P, 3, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    ws = torch.empty(plan.attn_bwd_workspace_bytes, dtype=torch.uint8, device=gpu)
    U.ulysses_attn_bwd(plan, T, OT, dO, lse, dT, ws, scale)
    torch.cuda.synchronize()
    assert U.ulysses_last_device_error(plan) == 0
    del ws, OT
    assert not dT[:, :, N:].any()
    for r in range(P):
        dK = dT[r, 1, :N].double()
        dV = dT[r, 2, :N].double()
        g = dO[r, :N].double()
        assert (dK.sum(0).abs() <= 1e-3 * dK.abs().sum(0) + 1e-6).all(), r
        assert ((dV.sum(0) - g.sum(0)).abs() <= 1e-3 * g.abs().sum(0) + 1e-6).all(), r
        del dK, dV, g
    rng = np.random.default_rng(31)
    qr = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 32, replace=False)]))
    iq = torch.from_numpy(qr).to(gpu)
    got_l, ref_l = [], []
    for r in range(P):
        j = r % Hl
        q, k, v = (orc.bf16_bits_to_f64(inputs.host_bits(T[r, c, :N, j])) for c in range(3))
        g_h = orc.bf16_bits_to_f64(inputs.host_bits(dO[r, :N, j]))
        dq, _, _ = orc.attention_bwd_sampled(q, k, v, g_h, scale, qr, qr[:0])
        got = dT[r, 0, :, j].index_select(0, iq).double().cpu().numpy()
        _close(got, dq, f"dQ long104k {r},{j}", record=False)
        got_l.append(got)
        ref_l.append(dq)
    check_attention("backward long104k one-pass dQ (sampled rows)", np.stack(got_l), np.stack(ref_l),
                    max_abs=None, mean_abs=None)
