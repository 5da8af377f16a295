"""CPU oracle for the recurrent gated-delta-rule decode step and its gate prologue.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module: only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import or call it. It shares no code with the CUDA library and imports
nothing from the package; it works on plain NumPy float64 arrays.

Sources (page title, section):

* "lite_boost.ops.recurrent_gated_delta_rule" (MindSpore Lite API page):
  the signature, the four-step algorithm (section "算法流程", steps 1-4), the
  argument shapes/dtypes (section "参数") and the returned tensors
  (section "返回").
* "com.microsoft.LinearAttentionGate" (ONNX Runtime contrib op, WebGPU kernel
  README): section "Description" (decay = decay_scale * softplus(a + dt_bias),
  beta = sigmoid(b), float32 arithmetic narrowed on store) and sections
  "Inputs" / "Outputs" (heads on the last axis, per-head float32 vectors).

The oracle computes the plain definition in float64, vectorised over
(value head, D_k, D_v), looping over batch items and tokens in the pages'
order. It rounds to bfloat16 only where the pages' dtypes force a stored
bfloat16 tensor: the output ``out`` per token and the state once per call.

Readings of points the pages leave open (each one is listed with its reason
in the design notes of the repository):

* A  state layout is the public [slot, H_v, D_k, D_v] (D_v contiguous); the
     leading axis is a pool addressed through ``ssm_state_indices``.
* B  the four steps run in the listed order: the memory read uses the decayed
     state, the output uses the updated state.
* C  exp(g) is a scalar per (b, h, t); exp(gk) scales row i (the D_k axis).
* D  the state stays in high precision across the tokens of one call and is
     rounded to bfloat16 once, at the end; ``out`` is rounded per token.
* E  ``num_accepted_tokens`` (the page gives only its purpose, speculative
     decoding) selects which state is kept: n = clamp(nat[b], 0, L) leading
     tokens are committed. Outputs of all L tokens come from the full
     recurrence; the slot receives the state after token n - 1, and keeps its
     bits when n = 0. ``None`` means n = L, as does nat = L, the value every
     workload uses (so the outputs and pool then equal the plain recurrence).
* E2 lengths are clamped to [0, T]; an item whose slot index is outside
     [0, pool) is skipped (zero output, no slot touched).
* G  value head h reads query/key head h // (H_v / H_qk).
* J  for t >= length the inputs are not read, out is +0.0, the state is
     unchanged.
* M  in the fused gate path g and beta stay float64 here (float32 on the
     device); they are never stored, so nothing narrows them.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_round",
    "softplus",
    "sigmoid",
    "linear_attention_gate",
    "recurrent_gated_delta_rule",
    "recurrent_gated_delta_rule_gated",
]

# bfloat16: 8 significant bits (1 implicit + 7 stored), same exponent range as
# float32 (normal exponents -126..127, subnormal quantum 2**-133).
_BF16_SIG_BITS = 8
_BF16_MIN_NORMAL_EXP = -126
_BF16_OVERFLOW = 2.0**128


def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16, ties to even, in one step.

    Rounding goes straight from float64 to bfloat16 (no float32 intermediate,
    so no double rounding). The result is returned as float64 holding
    bfloat16-representable values. NaN stays NaN, +-inf stays +-inf, values
    whose rounded magnitude reaches 2**128 overflow to +-inf, and subnormal
    results use the fixed quantum 2**-133.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, dtype=np.float64, copy=True)
    finite = np.isfinite(x) & (x != 0.0)
    xf = x[finite]
    # x = m * 2**e with 0.5 <= |m| < 1, so |x| lies in [2**(e-1), 2**e).
    _, e = np.frexp(xf)
    # Spacing of bfloat16 numbers in that binade; below the normal range the
    # spacing is fixed at 2**(-126 - 7).
    e_eff = np.maximum(e - 1, _BF16_MIN_NORMAL_EXP)
    quantum_exp = e_eff - (_BF16_SIG_BITS - 1)
    # x / 2**q is exact in float64 (power-of-two scaling, no underflow for the
    # bfloat16 range); np.rint rounds half to even.
    scaled = np.ldexp(xf, -quantum_exp)
    r = np.ldexp(np.rint(scaled), quantum_exp)
    r = np.where(np.abs(r) >= _BF16_OVERFLOW, np.copysign(np.inf, xf), r)
    out[finite] = r
    return out


def softplus(x) -> np.ndarray:
    """softplus(x) = ln(1 + e^x), in the overflow-free form max(x,0) + ln(1 + e^-|x|)."""
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def sigmoid(x) -> np.ndarray:
    """sigmoid(x) = 1 / (1 + e^-x), evaluated without overflow for either sign."""
    x = np.asarray(x, dtype=np.float64)
    z = np.exp(-np.abs(x))
    return np.where(x >= 0.0, 1.0 / (1.0 + z), z / (1.0 + z))


def linear_attention_gate(a, dt_bias, decay_scale, b=None):
    """The LinearAttentionGate op ("com.microsoft.LinearAttentionGate", Description).

    decay = decay_scale * softplus(a + dt_bias), and beta = sigmoid(b) when b is
    given. The head axis is the last axis of ``a`` (section "Inputs"); dt_bias
    and decay_scale are per-head vectors broadcast over the leading axes.
    Returns (decay, beta-or-None) in float64, unrounded.
    """
    a = np.asarray(a, dtype=np.float64)
    dt_bias = np.asarray(dt_bias, dtype=np.float64)
    decay_scale = np.asarray(decay_scale, dtype=np.float64)
    if dt_bias.shape != (a.shape[-1],) or decay_scale.shape != (a.shape[-1],):
        raise ValueError("dt_bias and decay_scale must be [H] with H = a.shape[-1]")
    decay = decay_scale * softplus(a + dt_bias)
    beta = None
    if b is not None:
        b = np.asarray(b, dtype=np.float64)
        if b.shape != a.shape:
            raise ValueError("b must have the shape of a")
        beta = sigmoid(b)
    return decay, beta


def _check_decode_shapes(query, key, value, state, asl, idx, gk):
    B, H_qk, T, D_k = query.shape
    if key.shape != query.shape:
        raise ValueError("key must have the shape of query")
    if value.ndim != 4 or value.shape[0] != B or value.shape[2] != T:
        raise ValueError("value must be [B, H_v, T, D_v]")
    H_v, D_v = value.shape[1], value.shape[3]
    if H_v % H_qk != 0:
        raise ValueError("H_v must be a multiple of H_qk")
    if state.ndim != 4 or state.shape[1:] != (H_v, D_k, D_v):
        raise ValueError("state must be [pool, H_v, D_k, D_v]")
    if gk.shape != (B, H_v, T, D_k):
        raise ValueError("gk must be [B, H_v, T, D_k]")
    if asl.shape != (B,) or idx.shape != (B,):
        raise ValueError("actual_seq_lengths and ssm_state_indices must be [B]")
    return B, H_qk, H_v, T, D_k, D_v


def _decode(query, key, value, state, asl, idx, gk, scale_value, gate_of,
            round_state, round_out, nat=None):
    """Shared token loop of both entry points; ``gate_of(b, t)`` gives (g[H_v], beta[H_v]).
    ``nat`` holds the committed token counts (reading E), or None."""
    query = np.asarray(query, dtype=np.float64)
    key = np.asarray(key, dtype=np.float64)
    value = np.asarray(value, dtype=np.float64)
    gk = np.asarray(gk, dtype=np.float64)
    asl = np.asarray(asl, dtype=np.int64)
    idx = np.asarray(idx, dtype=np.int64)
    state_out = np.array(state, dtype=np.float64, copy=True)
    B, H_qk, H_v, T, D_k, D_v = _check_decode_shapes(query, key, value, state_out,
                                                      asl, idx, gk)
    P = state_out.shape[0]
    group = H_v // H_qk
    hq = np.arange(H_v) // group  # reading G: value head h uses q/k head h // group
    out = np.zeros((B, H_v, T, D_v), dtype=np.float64)
    rnd_out = bf16_round if round_out else (lambda z: z)
    for b in range(B):
        L = int(min(max(asl[b], 0), T))  # reading E2
        s = int(idx[b])
        if not 0 <= s < P:
            continue  # reading E2: zero output, no slot touched
        if L == 0:
            continue  # reading J: no token, state unchanged
        n = L if nat is None else int(min(max(int(nat[b]), 0), L))  # reading E
        S = state_out[s].copy()  # [H_v, D_k, D_v], float64 across the whole call
        S_commit = None if n == 0 else S
        for t in range(L):
            g_t, beta_t = gate_of(b, t)  # [H_v], [H_v]
            q_t = query[b, hq, t, :] * scale_value  # [H_v, D_k]; q is scaled first
            k_t = key[b, hq, t, :]  # [H_v, D_k]
            v_t = value[b, :, t, :]  # [H_v, D_v]
            # step 1, state decay: S = S * exp(g) * exp(gk), gk indexed by the D_k row
            S = S * np.exp(g_t)[:, None, None] * np.exp(gk[b, :, t, :])[:, :, None]
            # step 2, memory read: kv_mem = S^T k
            kv_mem = np.einsum("hij,hi->hj", S, k_t)
            # step 3, delta update: S = S + k^T ((v - kv_mem) * beta)
            delta = (v_t - kv_mem) * beta_t[:, None]
            S = S + k_t[:, :, None] * delta[:, None, :]
            # step 4, output: o = S^T q
            out[b, :, t, :] = rnd_out(np.einsum("hij,hi->hj", S, q_t))
            if t == n - 1:
                S_commit = S  # reading E: the state after the last committed token
        if S_commit is not None:
            state_out[s] = bf16_round(S_commit) if round_state else S_commit  # reading D
    return out, state_out


def recurrent_gated_delta_rule(query, key, value, beta, state, actual_seq_lengths,
                               ssm_state_indices, g, gk, num_accepted_tokens,
                               scale_value=1.0, *, round_state=True, round_out=True):
    """The decode op of "lite_boost.ops.recurrent_gated_delta_rule" (算法流程, steps 1-4).

    Arguments follow the page's signature and shapes (section "参数"):
    query, key [B, H_qk, T, D_k]; value [B, H_v, T, D_v]; beta [B, H_v, T];
    state [pool, H_v, D_k, D_v] (reading A); actual_seq_lengths,
    ssm_state_indices, num_accepted_tokens [B] integers; g [B, H_v, T];
    gk [B, H_v, T, D_k]; scale_value multiplies the query (default 1.0).
    Inputs are arrays of the exact values (bfloat16 tensors widened to float64).

    Returns (out [B, H_v, T, D_v], state_out [pool, H_v, D_k, D_v]) as float64
    arrays of bfloat16-representable values (section "返回"); state_out is a
    new array and ``state`` is not modified. ``round_state``/``round_out``
    switch the bfloat16 narrowing off, for tests of the exact recurrence.
    """
    beta = np.asarray(beta, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    B, _, T, _ = np.shape(query)
    H_v = np.shape(value)[1]
    if beta.shape != (B, H_v, T) or g.shape != (B, H_v, T):
        raise ValueError("beta and g must be [B, H_v, T]")
    return _decode(query, key, value, state, actual_seq_lengths, ssm_state_indices, gk,
                   scale_value, lambda b, t: (g[b, :, t], beta[b, :, t]),
                   round_state, round_out, num_accepted_tokens)


def recurrent_gated_delta_rule_gated(query, key, value, a, b, dt_bias, decay_scale, state,
                                     actual_seq_lengths, ssm_state_indices, gk,
                                     num_accepted_tokens, scale_value=1.0, *,
                                     round_state=True, round_out=True):
    """The decode op with the LinearAttentionGate prologue in front of it.

    g = decay_scale * softplus(a + dt_bias) and beta = sigmoid(b)
    ("com.microsoft.LinearAttentionGate", Description), with a and b shaped
    [B, T, H_v] (heads last, section "Inputs") and dt_bias, decay_scale
    shaped [H_v]. The gate values feed the four decode steps unrounded
    (reading M). Everything else is as in ``recurrent_gated_delta_rule``.
    """
    a = np.asarray(a, dtype=np.float64)
    braw = np.asarray(b, dtype=np.float64)
    B, _, T, _ = np.shape(query)
    H_v = np.shape(value)[1]
    if a.shape != (B, T, H_v) or braw.shape != (B, T, H_v):
        raise ValueError("a and b must be [B, T, H_v]")
    def gate_of(bi, t):
        decay, beta = linear_attention_gate(a[bi, t], dt_bias, decay_scale, braw[bi, t])
        return decay, beta

    return _decode(query, key, value, state, actual_seq_lengths, ssm_state_indices, gk,
                   scale_value, gate_of, round_state, round_out, num_accepted_tokens)
