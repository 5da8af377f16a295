"""The 16-bit gate's log1p on [0, 1] (gdr_gate.cuh, log1p_narrow) against
numpy's log1p, in fp32 arithmetic as the kernel evaluates it (CPU).

softplus(x) = max(x, 0) + log1p(exp(-|x|)) needs log1p only on [0, 1]. The
kernel's polynomial must stay far below one unit in the last place of the
16-bit outputs (2^-11 relative for fp16, 2^-8 for bf16) over the whole
interval, small arguments included, where a relative error is what counts.
"""
import os
import re

import numpy as np

HEADER = os.path.join(os.path.dirname(__file__), os.pardir, "gated_delta_rule_recurrent_b200",
                      "csrc", "gdr_gate.cuh")


def coefficients():
    """The Horner coefficients of log1p_narrow, highest degree first."""
    src = open(HEADER).read()
    body = src[src.index("float log1p_narrow"):]
    body = body[:body.index("}")]
    first = re.search(r"float q = (-?[0-9.e+-]+)f;", body).group(1)
    rest = re.findall(r"q = fmaf\(q, z, (-?[0-9.e+-]+)f\);", body)
    return [np.float32(float(c)) for c in [first] + rest]


def log1p_narrow_fp32(z):
    z = z.astype(np.float32)
    c = coefficients()
    q = np.full_like(z, c[0])
    for cc in c[1:]:
        # q z is exact in float64; the sum is rounded to float32 as fmaf
        # rounds (up to a rare double rounding, one unit in the last place)
        q = (q.astype(np.float64) * z.astype(np.float64) + np.float64(cc)).astype(np.float32)
    return (z * q).astype(np.float32)


def test_relative_error_on_the_whole_interval():
    z = np.concatenate([np.geomspace(1e-30, 1e-3, 20000), np.linspace(1e-3, 1.0, 200001)])
    got = log1p_narrow_fp32(z).astype(np.float64)
    want = np.log1p(z.astype(np.float32).astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 1.2e-5, rel.max()
    assert rel.max() < 2.0 ** -11 / 16  # far below an fp16 unit in the last place


def test_degree_and_end_points():
    assert len(coefficients()) == 6
    assert log1p_narrow_fp32(np.array([0.0]))[0] == 0.0
    assert abs(float(log1p_narrow_fp32(np.array([1.0]))[0]) - np.log(2.0)) < 1e-5
