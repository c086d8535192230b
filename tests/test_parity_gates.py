"""The attention parity gates themselves, on the CPU.

At the Video-DiT length (19,394 keys) with N(0,1) inputs the output is small
(|O| ~ 0.01), so the layer's absolute gates (max-abs 2e-2, mean-abs 2e-3)
cannot see an output that is 10% off.  These tests plant such mistakes in the
oracle's result and check that the rel-L2 gate of tests/_parity.py fails them,
while an fp64 emulation of the kernel's two bf16 roundings (P before the P V
product, O at the store) passes with the margin the gate's derivation states.
"""
import math

import numpy as np
import pytest
from _parity import MAX_ABS, MEAN_ABS, REL_L2, REL_L2_FP8, check_attention, rel_l2

from oracle import ulysses_oracle as orc

N_KEYS = 19_394
ROWS = 96


def _bf16(x):
    return orc.bf16_bits_to_f64(orc.f64_to_bf16_bits(x))


def _e4m3(x):
    return orc.e4m3_bits_to_f64(orc.f64_to_e4m3_bits(x))


@pytest.fixture(scope="module")
def head():
    rng = np.random.default_rng(1234)
    q = _bf16(rng.standard_normal((ROWS, 128)))
    k = _bf16(rng.standard_normal((N_KEYS, 128)))
    v = _bf16(rng.standard_normal((N_KEYS, 128)))
    return q, k, v


def _rounded(q, k, v, scale, rnd):
    """The same softmax with P rounded by ``rnd`` before P V and O rounded to bf16."""
    z = scale * (q @ k.T)
    p = np.exp(z - z.max(axis=1, keepdims=True))
    return _bf16((rnd(p) @ v) / p.sum(axis=1, keepdims=True))


def test_rounding_model_passes_with_margin(head):
    q, k, v = head
    scale = 1.0 / math.sqrt(128)
    ref = orc.attention_rows(q, k, v, scale)
    r = rel_l2(_rounded(q, k, v, scale, _bf16), ref)
    # the derivation: two roundings of RMS 1.66e-3 in quadrature, ~2.35e-3
    assert 1.5e-3 < r < 3.5e-3, r
    assert r * 3 < REL_L2
    r8 = rel_l2(_rounded(q, k, v, scale, _e4m3), ref)
    assert 1.8e-2 < r8 < 3.6e-2, r8
    assert r8 * 2.5 < REL_L2_FP8


@pytest.mark.parametrize("mistake", ["output x 1.1", "scale x 1.1", "one key tile dropped"])
def test_planted_mistakes_pass_absolute_gates_but_fail_rel_l2(head, mistake):
    q, k, v = head
    scale = 1.0 / math.sqrt(128)
    ref = orc.attention_rows(q, k, v, scale)
    if mistake == "output x 1.1":
        bad = ref * 1.1
    elif mistake == "scale x 1.1":
        bad = orc.attention_rows(q, k, v, scale * 1.1)
    else:                                     # the last 128 keys never visited
        bad = orc.attention_rows(q, k[:-128], v[:-128], scale)
    err = np.abs(bad - ref)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS     # invisible to the absolute gates
    with pytest.raises(AssertionError, match="rel-L2"):
        check_attention(f"planted: {mistake}", bad, ref)


def test_rel_l2_of_zero_reference():
    assert rel_l2(np.zeros(4), np.zeros(4)) == 0.0
    assert rel_l2(np.ones(4), np.zeros(4)) == float("inf")
