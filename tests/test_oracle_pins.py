"""Pins of the CPU oracle to things other than itself (CPU only).

Each test fixes a property that the pages or the mathematics determine, chosen
so that a plausible slip in the oracle (a dropped term, a wrong sign, a
transposed operand, a wrong index, a wrong step order) fails at least one:

* hand-worked cases from the four algorithm steps (tests/golden);
* closed forms: zero state, pure decay, identity update;
* invariants: the delta rule writes v at key k; composition over tokens;
  pool slots not referenced are untouched; permutation equivariance;
* an independent matrix form of one step, S' = (I - beta k k^T) D S + beta k v^T;
* a scalar-loop brute force on tiny inputs.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle.gdr_oracle import (bf16_round, recurrent_gated_delta_rule,
                               recurrent_gated_delta_rule_gated)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "handworked_decode.json")


def _rng(seed):
    return np.random.default_rng(seed)


def _rand_case(seed, B=2, H_qk=2, H_v=4, T=3, D_k=4, D_v=6, P=3, unit=True):
    r = _rng(seed)
    q = r.standard_normal((B, H_qk, T, D_k))
    k = r.standard_normal((B, H_qk, T, D_k))
    if unit:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    return dict(
        query=q, key=k,
        value=r.standard_normal((B, H_v, T, D_v)),
        beta=1.0 / (1.0 + np.exp(-r.standard_normal((B, H_v, T)))),
        state=0.3 * r.standard_normal((P, H_v, D_k, D_v)),
        actual_seq_lengths=np.full(B, T, dtype=np.int64),
        ssm_state_indices=r.permutation(P)[:B].astype(np.int64),
        g=-np.log1p(np.exp(r.standard_normal((B, H_v, T)))),
        gk=-0.1 * np.log1p(np.exp(r.standard_normal((B, H_v, T, D_k)))),
        num_accepted_tokens=np.full(B, T, dtype=np.int64),
        scale_value=0.7,
    )


def _run(case, **kw):
    return recurrent_gated_delta_rule(
        case["query"], case["key"], case["value"], case["beta"], case["state"],
        case["actual_seq_lengths"], case["ssm_state_indices"], case["g"], case["gk"],
        case["num_accepted_tokens"], case["scale_value"], **kw)


# ---------------------------------------------------------------- golden cases

def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_handworked_golden(case):
    inp = {k: (np.asarray(v, dtype=np.float64) if isinstance(v, list) else v)
           for k, v in case["inputs"].items()}
    for name in ("actual_seq_lengths", "ssm_state_indices", "num_accepted_tokens"):
        inp[name] = inp[name].astype(np.int64)
    if "a" in inp:
        out, st = recurrent_gated_delta_rule_gated(
            inp["query"], inp["key"], inp["value"], inp["a"], inp["b"], inp["dt_bias"],
            inp["decay_scale"], inp["state"], inp["actual_seq_lengths"],
            inp["ssm_state_indices"], inp["gk"], inp["num_accepted_tokens"],
            inp["scale_value"])
    else:
        out, st = recurrent_gated_delta_rule(
            inp["query"], inp["key"], inp["value"], inp["beta"], inp["state"],
            inp["actual_seq_lengths"], inp["ssm_state_indices"], inp["g"], inp["gk"],
            inp["num_accepted_tokens"], inp["scale_value"])
    exp_out = np.asarray(case["expected"]["out"], dtype=np.float64)
    exp_st = np.asarray(case["expected"]["state_out"], dtype=np.float64)
    # The expected values are bfloat16-exact and the fp64 arithmetic is within
    # a few ulps of them, so after rounding they must agree exactly.
    np.testing.assert_array_equal(out, exp_out)
    np.testing.assert_array_equal(st, exp_st)


# ---------------------------------------------------------------- closed forms

def test_zero_state_single_token_closed_form():
    """S0 = 0, T = 1: o = beta * (k . q*scale) * v, whatever the decay."""
    c = _rand_case(1, T=1)
    c["state"][:] = 0.0
    out, st = _run(c, round_out=False, round_state=False)
    B, H_v = c["value"].shape[:2]
    group = H_v // c["query"].shape[1]
    for b in range(B):
        for h in range(H_v):
            hq = h // group
            kq = float(np.dot(c["key"][b, hq, 0], c["query"][b, hq, 0])) * c["scale_value"]
            want = c["beta"][b, h, 0] * kq * c["value"][b, h, 0]
            np.testing.assert_allclose(out[b, h, 0], want, rtol=1e-13, atol=1e-15)
            s = c["ssm_state_indices"][b]
            want_S = c["beta"][b, h, 0] * np.outer(c["key"][b, hq, 0], c["value"][b, h, 0])
            np.testing.assert_allclose(st[s, h], want_S, rtol=1e-13, atol=1e-15)


def test_delta_rule_writes_value_at_unit_key():
    """beta = 1, |k| = 1, any decay: after the update S'^T k = v exactly (in fp64)."""
    c = _rand_case(2, T=1, unit=True)
    c["beta"][:] = 1.0
    _, st = _run(c, round_state=False)
    B, H_v = c["value"].shape[:2]
    group = H_v // c["query"].shape[1]
    for b in range(B):
        s = c["ssm_state_indices"][b]
        for h in range(H_v):
            k = c["key"][b, h // group, 0]
            np.testing.assert_allclose(st[s, h].T @ k, c["value"][b, h, 0], rtol=1e-12,
                                       atol=1e-12)


def test_pure_decay_closed_form():
    """beta = 0: S_T = S_0 scaled row-wise by exp(sum_t (g_t + gk_t,i)); o_t = S_t^T q_t*scale."""
    c = _rand_case(3, T=3, D_k=3, D_v=5)
    c["beta"][:] = 0.0
    out, st = _run(c, round_out=False, round_state=False)
    B, H_v = c["value"].shape[:2]
    group = H_v // c["query"].shape[1]
    for b in range(B):
        s = c["ssm_state_indices"][b]
        for h in range(H_v):
            S = c["state"][s, h]
            for t in range(3):
                logd = c["g"][b, h, : t + 1].sum() + c["gk"][b, h, : t + 1, :].sum(axis=0)
                St = np.exp(logd)[:, None] * S
                qs = c["query"][b, h // group, t] * c["scale_value"]
                np.testing.assert_allclose(out[b, h, t], St.T @ qs, rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(st[s, h], St, rtol=1e-12, atol=1e-14)


def test_identity_update_is_plain_matvec():
    """beta = 0 and g = gk = 0: S unchanged and o = S^T (q*scale) (numpy matmul)."""
    c = _rand_case(4, T=2)
    c["beta"][:] = 0.0
    c["g"][:] = 0.0
    c["gk"][:] = 0.0
    c["state"] = bf16_round(c["state"])
    out, st = _run(c, round_out=False)
    np.testing.assert_array_equal(st, c["state"])
    B, H_v = c["value"].shape[:2]
    group = H_v // c["query"].shape[1]
    for b in range(B):
        s = c["ssm_state_indices"][b]
        for h in range(H_v):
            for t in range(2):
                qs = c["query"][b, h // group, t] * c["scale_value"]
                np.testing.assert_allclose(out[b, h, t], np.matmul(c["state"][s, h].T, qs),
                                           rtol=1e-13, atol=1e-15)


def test_grouped_heads_use_floor_division():
    """H_v = 2 H_qk: value head h uses q/k head h // 2 (not h % 2)."""
    c = _rand_case(5, B=1, H_qk=2, H_v=4, T=1)
    c["state"][:] = 0.0
    out, _ = _run(c, round_out=False, round_state=False)
    for h in range(4):
        hq = h // 2
        kq = np.dot(c["key"][0, hq, 0], c["query"][0, hq, 0]) * c["scale_value"]
        np.testing.assert_allclose(out[0, h, 0], c["beta"][0, h, 0] * kq * c["value"][0, h, 0],
                                   rtol=1e-13)
    # the other mapping would differ on this draw
    h = 1
    kq_wrong = np.dot(c["key"][0, h % 2, 0], c["query"][0, h % 2, 0]) * c["scale_value"]
    assert not np.allclose(out[0, h, 0], c["beta"][0, h, 0] * kq_wrong * c["value"][0, h, 0])


# ---------------------------------------------------------------- invariants

def test_tokens_compose():
    """Without rounding, one call over T = 3 tokens equals three T = 1 calls."""
    c = _rand_case(6, T=3)
    out_all, st_all = _run(c, round_out=False, round_state=False)
    st = c["state"].copy()
    for t in range(3):
        ct = dict(c)
        for name in ("query", "key", "value"):
            ct[name] = c[name][:, :, t : t + 1]
        ct["beta"] = c["beta"][:, :, t : t + 1]
        ct["g"] = c["g"][:, :, t : t + 1]
        ct["gk"] = c["gk"][:, :, t : t + 1]
        ct["actual_seq_lengths"] = np.ones_like(c["actual_seq_lengths"])
        ct["state"] = st
        out_t, st = _run(ct, round_out=False, round_state=False)
        np.testing.assert_allclose(out_t[:, :, 0], out_all[:, :, t], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(st, st_all, rtol=1e-12, atol=1e-14)


def test_long_prompt_equals_chunks_of_eight():
    """A prefill-length call: without rounding, one call over T = 128 tokens
    equals sixteen consecutive T = 8 calls (the state of each passed to the
    next), bit for bit, with ragged lengths that end inside a chunk."""
    c = _rand_case(16, B=3, H_qk=1, H_v=2, T=128, D_k=5, D_v=3, P=4)
    c["actual_seq_lengths"] = np.array([128, 77, 8])
    out_all, st_all = _run(c, round_out=False, round_state=False)
    st = c["state"].copy()
    for k in range(16):
        ck = dict(c)
        sl = slice(8 * k, 8 * k + 8)
        for name in ("query", "key", "value"):
            ck[name] = c[name][:, :, sl]
        for name in ("beta", "g", "gk"):
            ck[name] = c[name][:, :, sl]
        ck["actual_seq_lengths"] = np.clip(c["actual_seq_lengths"] - 8 * k, 0, 8)
        ck["num_accepted_tokens"] = ck["actual_seq_lengths"]
        ck["state"] = st
        out_k, st = _run(ck, round_out=False, round_state=False)
        valid = (8 * k + np.arange(8))[None, :] < c["actual_seq_lengths"][:, None]  # [B, 8]
        assert np.array_equal(out_k[valid[:, None, :].repeat(2, 1)],
                              out_all[:, :, sl][valid[:, None, :].repeat(2, 1)])
    assert np.array_equal(st, st_all)


def test_untouched_slots_and_permutation():
    """Slots no item references keep their exact bits; permuting items permutes outputs."""
    c = _rand_case(7, B=3, P=6)
    c["state"] = bf16_round(c["state"])
    out, st = _run(c)
    untouched = sorted(set(range(6)) - set(c["ssm_state_indices"].tolist()))
    assert untouched
    np.testing.assert_array_equal(st[untouched], c["state"][untouched])
    perm = np.array([2, 0, 1])
    cp = dict(c)
    for name in ("query", "key", "value", "beta", "g", "gk", "actual_seq_lengths",
                 "ssm_state_indices", "num_accepted_tokens"):
        cp[name] = c[name][perm]
    out_p, st_p = _run(cp)
    np.testing.assert_array_equal(out_p, out[perm])
    np.testing.assert_array_equal(st_p, st)


def test_padding_lengths_and_bad_slots():
    """t >= length is not read (NaN inputs change nothing) and gives +0.0; length 0 and a
    slot outside the pool leave every slot as it was and give zero output."""
    c = _rand_case(8, B=4, P=5, T=3)
    c["state"] = bf16_round(c["state"])
    c["actual_seq_lengths"] = np.array([3, 1, 0, 2])
    c["ssm_state_indices"] = np.array([4, 0, 2, 7])  # item 3 points outside the pool
    out, st = _run(c)
    poisoned = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in c.items()}
    for b, L in enumerate(c["actual_seq_lengths"]):
        for name in ("query", "key", "value", "gk"):
            poisoned[name][b, :, L:] = np.nan
        for name in ("beta", "g"):
            poisoned[name][b, :, L:] = np.nan
    out_p, st_p = _run(poisoned)
    np.testing.assert_array_equal(out_p, out)
    np.testing.assert_array_equal(st_p, st)
    assert np.all(out[0, :, 3:] == 0)
    assert np.all(out[1, :, 1:] == 0) and not np.all(out[1, :, :1] == 0)
    assert np.all(out[2] == 0) and np.all(out[3] == 0)
    assert not np.signbit(out[2]).any()
    for s in (1, 2, 3):  # unreferenced, length-0 item's slot, nothing maps to 3
        np.testing.assert_array_equal(st[s], c["state"][s])
    # lengths beyond T are clamped to T
    c2 = dict(c)
    c2["actual_seq_lengths"] = np.array([9, 1, 0, 2])
    out2, st2 = _run(c2)
    np.testing.assert_array_equal(out2, out)
    np.testing.assert_array_equal(st2, st)


def test_matrix_form_of_one_step():
    """Independent formulation: S' = (I - beta k k^T) D S + beta k v^T, o = S'^T q*scale."""
    c = _rand_case(9, B=1, H_qk=1, H_v=1, T=1, D_k=5, D_v=3, P=1, unit=False)
    out, st = _run(c, round_out=False, round_state=False)
    k = c["key"][0, 0, 0]
    q = c["query"][0, 0, 0] * c["scale_value"]
    v = c["value"][0, 0, 0]
    beta = c["beta"][0, 0, 0]
    D = np.diag(np.exp(c["g"][0, 0, 0] + c["gk"][0, 0, 0]))
    S = c["state"][c["ssm_state_indices"][0], 0]
    S1 = (np.eye(5) - beta * np.outer(k, k)) @ D @ S + beta * np.outer(k, v)
    np.testing.assert_allclose(st[c["ssm_state_indices"][0], 0], S1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(out[0, 0, 0], S1.T @ q, rtol=1e-12, atol=1e-14)


def test_scalar_brute_force_tiny():
    """Scalar loops, element by element, on a tiny case with several heads and tokens."""
    c = _rand_case(10, B=2, H_qk=1, H_v=2, T=3, D_k=3, D_v=4, P=2)
    c["actual_seq_lengths"] = np.array([3, 2])
    out, st = _run(c, round_out=False, round_state=False)
    B, H_qk, T, D_k = c["query"].shape
    H_v, D_v = c["value"].shape[1], c["value"].shape[3]
    for b in range(B):
        s = int(c["ssm_state_indices"][b])
        for h in range(H_v):
            hq = h // (H_v // H_qk)
            S = [[float(c["state"][s, h, i, j]) for j in range(D_v)] for i in range(D_k)]
            for t in range(int(c["actual_seq_lengths"][b])):
                for i in range(D_k):
                    f = math.exp(c["g"][b, h, t]) * math.exp(c["gk"][b, h, t, i])
                    for j in range(D_v):
                        S[i][j] *= f
                mem = [sum(S[i][j] * c["key"][b, hq, t, i] for i in range(D_k))
                       for j in range(D_v)]
                for i in range(D_k):
                    for j in range(D_v):
                        S[i][j] += c["key"][b, hq, t, i] * (c["value"][b, h, t, j] - mem[j]) \
                            * c["beta"][b, h, t]
                for j in range(D_v):
                    o = sum(S[i][j] * c["query"][b, hq, t, i] * c["scale_value"]
                            for i in range(D_k))
                    assert abs(o - out[b, h, t, j]) <= 1e-12
            for i in range(D_k):
                for j in range(D_v):
                    assert abs(S[i][j] - st[s, h, i, j]) <= 1e-12


def test_state_rounded_once_per_call():
    """The state is narrowed to bfloat16 once, after the last token (reading D): a T = 2
    call equals the unrounded recurrence followed by one rounding."""
    c = _rand_case(11, T=2)
    c["state"] = bf16_round(c["state"])
    _, st_once = _run(c, round_out=False)
    _, st_exact = _run(c, round_out=False, round_state=False)
    np.testing.assert_array_equal(st_once, bf16_round(st_exact))


# ------------------------------------------------------- committed tokens (reading E)

def test_committed_state_equals_a_shorter_call():
    """num_accepted_tokens = n < L: the slot receives the state a call over the
    first n tokens alone leaves (the shorter call is a separate run of the
    plain recurrence), while every output matches the full-length call."""
    c = _rand_case(21, B=3, T=5, P=4)
    full_out, _ = _run(c, round_out=False, round_state=False)
    n = np.array([2, 5, 1])
    cn = dict(c, num_accepted_tokens=n)
    out_n, st_n = _run(cn, round_out=False, round_state=False)
    np.testing.assert_array_equal(out_n, full_out)
    short = dict(c, actual_seq_lengths=n, num_accepted_tokens=n)
    _, st_short = _run(short, round_out=False, round_state=False)
    np.testing.assert_allclose(st_n, st_short, rtol=1e-13, atol=1e-15)
    # the committed state differs from the full call's where n < L
    _, st_full = _run(c, round_out=False, round_state=False)
    s0 = c["ssm_state_indices"][0]
    assert np.abs(st_n[s0] - st_full[s0]).max() > 1e-3


def test_nothing_committed_keeps_the_slot_bits():
    c = _rand_case(22, B=2, T=3, P=3)
    c["state"] = bf16_round(c["state"])
    n = np.array([0, 0])
    out0, st0 = _run(dict(c, num_accepted_tokens=n))
    out_full, _ = _run(c)
    np.testing.assert_array_equal(out0, out_full)
    np.testing.assert_array_equal(st0.view(np.int64), c["state"].view(np.int64))


def test_committed_count_is_clamped_and_none_means_all():
    c = _rand_case(23, B=2, T=4, P=2)
    ref = _run(c)
    for n in (np.array([9, 4]), np.array([4, 100])):
        got = _run(dict(c, num_accepted_tokens=n))
        np.testing.assert_array_equal(got[0], ref[0])
        np.testing.assert_array_equal(got[1], ref[1])
    got = _run(dict(c, num_accepted_tokens=None))
    np.testing.assert_array_equal(got[1], ref[1])
    neg = _run(dict(c, num_accepted_tokens=np.array([-2, 0])))
    np.testing.assert_array_equal(neg[1], _run(dict(c, num_accepted_tokens=np.array([0, 0])))[1])
