"""Pins of the oracle's bfloat16 rounding and gate functions (CPU only).

* bf16_round against exact rational arithmetic: the result is a bfloat16 value,
  no bfloat16 value is nearer, and exact ties go to the even significand.
* bf16_round against torch's float32 -> bfloat16 conversion (single rounding,
  round-to-nearest-even) on float32-exact inputs.
* softplus / sigmoid against torch's float64 library routines and their
  special values (softplus(0) = ln 2, sigmoid(0) = 1/2, asymptotes).
* The gated oracle against the plain oracle fed with gate values computed by
  torch's routines ("com.microsoft.LinearAttentionGate", Description).
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle.gdr_oracle import (bf16_round, linear_attention_gate, recurrent_gated_delta_rule,
                               recurrent_gated_delta_rule_gated, sigmoid, softplus)


def _bf16_bits_to_float(bits):
    return float(np.array([bits << 16], dtype=np.uint32).view(np.float32)[0])


def _float_to_bf16_bits(x):
    """Bit pattern of a float64 that must be exactly a bfloat16 value."""
    f32 = np.array([x], dtype=np.float32)
    assert float(f32[0]) == x, "not representable in float32"
    u = int(f32.view(np.uint32)[0])
    assert u & 0xFFFF == 0, "not representable in bfloat16"
    return u >> 16


def _neighbours(bits):
    """Adjacent bfloat16 values (same sign direction), skipping inf/NaN patterns."""
    out = []
    for nb in (bits - 1, bits + 1):
        if 0 <= nb <= 0xFFFF:
            v = _bf16_bits_to_float(nb)
            if math.isfinite(v):
                out.append(v)
    return out


def _sample_values(rng, n):
    # magnitudes across the whole bfloat16 range, subnormals included
    exps = rng.uniform(-140, 126.9, n)  # finite results; overflow is pinned separately
    signs = rng.choice([-1.0, 1.0], n)
    return signs * np.exp2(exps) * rng.uniform(1.0, 2.0, n)


def test_bf16_round_is_nearest_exact():
    rng = np.random.default_rng(0)
    xs = _sample_values(rng, 3000)
    rs = bf16_round(xs)
    for x, r in zip(xs, rs):
        bits = _float_to_bf16_bits(float(r))
        err = abs(Fraction(float(x)) - Fraction(float(r)))
        for nb in _neighbours(bits):
            e2 = abs(Fraction(float(x)) - Fraction(nb))
            assert err <= e2, (x, r, nb)
            if err == e2:
                assert bits % 2 == 0, "tie must go to even"


def test_bf16_round_ties_to_even_and_no_double_rounding():
    one = 1.0
    ulp = 2.0**-7
    # exact midpoints between 1 and 1+ulp, and between 1+ulp and 1+2ulp
    assert bf16_round(np.array([one + ulp / 2]))[0] == one
    assert bf16_round(np.array([one + 1.5 * ulp]))[0] == one + 2 * ulp
    # just above a midpoint rounds up even though float32 would first drop the excess
    assert bf16_round(np.array([one + ulp / 2 + 2.0**-30]))[0] == one + ulp
    # subnormal quantum is 2**-133
    assert bf16_round(np.array([2.0**-133 * 0.5]))[0] == 0.0
    assert bf16_round(np.array([2.0**-133 * 0.51]))[0] == 2.0**-133
    assert bf16_round(np.array([2.0**-133 * 1.5]))[0] == 2.0**-132
    # overflow: the midpoint between the largest finite and 2**128 goes to inf
    big = (2.0 - 2.0**-7) * 2.0**127
    assert bf16_round(np.array([big]))[0] == big
    assert bf16_round(np.array([(2.0 - 2.0**-8) * 2.0**127]))[0] == math.inf
    assert bf16_round(np.array([-(2.0 - 2.0**-8) * 2.0**127]))[0] == -math.inf
    r = bf16_round(np.array([np.nan, np.inf, -np.inf, -0.0, 0.0]))
    assert math.isnan(r[0]) and r[1] == math.inf and r[2] == -math.inf
    assert r[3] == 0.0 and math.copysign(1.0, r[3]) == -1.0
    assert math.copysign(1.0, bf16_round(np.array([-1e-60]))[0]) == -1.0


def test_bf16_round_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(1)
    xs = _sample_values(rng, 20000).astype(np.float32)
    xs = xs[np.isfinite(xs)]
    want = torch.from_numpy(xs).to(torch.bfloat16).to(torch.float64).numpy()
    got = bf16_round(xs.astype(np.float64))
    np.testing.assert_array_equal(got, want)


def test_softplus_sigmoid_against_torch_and_special_values():
    x = np.concatenate([np.linspace(-50, 50, 2001), [-745.0, 745.0, 0.0]])
    tx = torch.from_numpy(x)
    # torch's softplus switches to the identity above a threshold; compare where
    # both use the same formula and check the large-x branch by its asymptote.
    mask = x < 20
    np.testing.assert_allclose(softplus(x)[mask],
                               torch.nn.functional.softplus(tx).numpy()[mask],
                               rtol=1e-15, atol=1e-300)
    big = x[x >= 20]
    np.testing.assert_allclose(softplus(big), big + np.exp(-big), rtol=1e-15)
    np.testing.assert_allclose(sigmoid(x), torch.sigmoid(tx).numpy(), rtol=1e-15,
                               atol=1e-300)
    assert softplus(np.array([0.0]))[0] == pytest.approx(math.log(2.0), rel=1e-16)
    assert sigmoid(np.array([0.0]))[0] == 0.5
    assert softplus(np.array([-745.0]))[0] >= 0.0
    assert sigmoid(np.array([745.0]))[0] == 1.0 and sigmoid(np.array([-745.0]))[0] >= 0.0


def test_gate_formula_and_shapes():
    rng = np.random.default_rng(2)
    a = rng.standard_normal((3, 2, 5))
    bb = rng.standard_normal((3, 2, 5))
    dtb = rng.uniform(0, 1, 5)
    A_log = rng.uniform(-1, 1, 5)
    ds = -np.exp(A_log)
    decay, beta = linear_attention_gate(a, dtb, ds, bb)
    ta = torch.from_numpy(a)
    want = torch.from_numpy(ds) * torch.nn.functional.softplus(ta + torch.from_numpy(dtb))
    np.testing.assert_allclose(decay, want.numpy(), rtol=1e-15)
    np.testing.assert_allclose(beta, torch.sigmoid(torch.from_numpy(bb)).numpy(), rtol=1e-15)
    assert np.all(decay < 0)  # decay_scale = -exp(A_log) < 0 and softplus > 0
    d2, b2 = linear_attention_gate(a, dtb, ds)
    assert b2 is None
    np.testing.assert_array_equal(d2, decay)
    with pytest.raises(ValueError):
        linear_attention_gate(a, dtb[:4], ds)


def test_gated_decode_equals_plain_decode_with_library_gate():
    rng = np.random.default_rng(3)
    B, H_qk, H_v, T, D_k, D_v, P = 2, 2, 4, 2, 4, 3, 3
    q = rng.standard_normal((B, H_qk, T, D_k))
    k = rng.standard_normal((B, H_qk, T, D_k))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, H_v, T, D_v))
    a = rng.standard_normal((B, T, H_v))
    bb = rng.standard_normal((B, T, H_v))
    dtb = rng.uniform(0, 1, H_v)
    ds = -np.exp(rng.uniform(-1, 1, H_v))
    gk = -0.1 * np.log1p(np.exp(rng.standard_normal((B, H_v, T, D_k))))
    state = bf16_round(0.1 * rng.standard_normal((P, H_v, D_k, D_v)))
    asl = np.array([2, 1])
    idx = np.array([2, 0])
    out_g, st_g = recurrent_gated_delta_rule_gated(q, k, v, a, bb, dtb, ds, state, asl, idx, gk,
                                                   asl, 0.5, round_out=False,
                                                   round_state=False)
    ta = torch.from_numpy(a)
    g = (torch.from_numpy(ds) * torch.nn.functional.softplus(ta + torch.from_numpy(dtb)))
    g = g.permute(0, 2, 1).numpy()  # [B, T, H_v] -> [B, H_v, T]
    beta = torch.sigmoid(torch.from_numpy(bb)).permute(0, 2, 1).numpy()
    out_p, st_p = recurrent_gated_delta_rule(q, k, v, beta, state, asl, idx, g, gk, asl, 0.5,
                                             round_out=False, round_state=False)
    np.testing.assert_allclose(out_g, out_p, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(st_g, st_p, rtol=1e-13, atol=1e-15)
