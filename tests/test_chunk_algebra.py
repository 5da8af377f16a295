"""The chunked form of the recurrence that the tensor-core and prefill kernels
compute, stated in float64 and checked against the oracle's token loop (CPU).

The token loop ("lite_boost.ops.recurrent_gated_delta_rule", section 算法流程,
steps 1-4) runs, per token t with decays d_t = exp(g_t + gk_t) on the rows,
    S = d_t o S;  kv_t = S^T k_t;  delta_t = beta_t (v_t - kv_t);
    S = S + k_t delta_t^T;  o_t = S^T (q_t scale).
Over a chunk of L tokens from S_0, with running products of the decays
P_t = d_0 ... d_t and P_{s->t} = d_{s+1} ... d_t (P_{t->t} = 1), it regroups to
    u_t = P_t o k_t,  w_t = P_t o q^_t,
    A_ts = sum_i k_s[i] P_{s->t}[i] k_t[i]   (s < t),
    B_ts = sum_i k_s[i] P_{s->t}[i] q^_t[i]  (s <= t),
    kv_t = S_0^T u_t + sum_{s<t} A_ts delta_s,  delta_t = beta_t (v_t - kv_t),
    o_t = S_0^T w_t + sum_{s<=t} B_ts delta_s,
    S after n tokens = P_{n-1} o S_0 + sum_{s<n} (P_{s->n-1} o k_s) delta_s^T.
The kernels evaluate exactly these terms (the first two products on the
tensor cores, the sums and the unit lower-triangular solve on the CUDA cores),
so this pins the algebra they rest on, independently of the GPU: a wrong index
in a running product, a missing diagonal term or a transposed sum fails here.
"""
import numpy as np
import pytest

from oracle import gdr_oracle as O


def _inputs(rng, L, D_k=6, D_v=5, g_scale=1.0):
    return dict(
        S0=rng.standard_normal((D_k, D_v)),
        q=rng.standard_normal((L, D_k)),
        k=rng.standard_normal((L, D_k)) / np.sqrt(D_k),
        v=rng.standard_normal((L, D_v)),
        g=-g_scale * np.log1p(np.exp(rng.standard_normal(L))),
        gk=-0.1 * g_scale * np.log1p(np.exp(rng.standard_normal((L, D_k)))),
        beta=1.0 / (1.0 + np.exp(-rng.standard_normal(L))),
        scale=0.7,
    )


def chunked(x, n, wrong_A=False):
    """(outputs of the L tokens, state after n tokens) by the chunked form."""
    S0, q, k, v, g, gk, beta, scale = (x[n_] for n_ in ("S0", "q", "k", "v", "g", "gk", "beta",
                                                         "scale"))
    L = q.shape[0]
    d = np.exp(g[:, None] + gk)  # [L, D_k]
    qh = q * scale
    P = np.cumprod(d, axis=0)  # P_t

    def Pst(s, t):  # P_{s->t}: the decays of tokens s + 1 .. t
        return np.prod(d[s + 1:t + 1], axis=0) if t > s else np.ones(d.shape[1])

    u, w = P * k, P * qh
    A = np.zeros((L, L))
    Bm = np.zeros((L, L))
    for t in range(L):
        for s in range(t + 1):
            ps = Pst(s - 1, t) if (wrong_A and s > 0) else Pst(s, t)
            if s < t:
                A[t, s] = np.sum(k[s] * ps * k[t])
            Bm[t, s] = np.sum(k[s] * Pst(s, t) * qh[t])
    delta = np.zeros((L, S0.shape[1]))
    out = np.zeros((L, S0.shape[1]))
    for t in range(L):
        kv = S0.T @ u[t] + A[t, :t] @ delta[:t]
        delta[t] = beta[t] * (v[t] - kv)
        out[t] = S0.T @ w[t] + Bm[t, :t + 1] @ delta[:t + 1]
    if n == 0:
        return out, S0.copy()
    S_n = P[n - 1][:, None] * S0
    for s in range(n):
        S_n += (Pst(s, n - 1) * k[s])[:, None] * delta[s][None, :]
    return out, S_n


def token_loop(x, n):
    """The oracle's token loop on one head, unrounded."""
    S0, q, k, v, g, gk, beta, scale = (x[n_] for n_ in ("S0", "q", "k", "v", "g", "gk", "beta",
                                                         "scale"))
    L, D_k = q.shape
    gate = lambda b, t: (np.array([g[t]]), np.array([beta[t]]))  # noqa: E731
    out, state = O._decode(q[None, None], k[None, None], v[None, None], S0[None, None],
                           np.array([L]), np.array([0]), gk[None, None], scale, gate,
                           round_state=False, round_out=False, nat=np.array([n]))
    return out[0, 0], state[0, 0]


def close(a, b):
    return np.allclose(a, b, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("L", range(1, 9))
def test_chunk_equals_token_loop_for_every_length_and_committed_count(L):
    rng = np.random.default_rng(100 + L)
    x = _inputs(rng, L)
    for n in range(L + 1):
        out_c, S_c = chunked(x, n)
        out_t, S_t = token_loop(x, n)
        assert close(out_c, out_t), (L, n)
        assert close(S_c, S_t), (L, n)


def test_vanishing_decays_stay_finite():
    """Decays that underflow within the chunk: the running products reach 0,
    nothing divides, and the chunked form still equals the token loop."""
    rng = np.random.default_rng(7)
    x = _inputs(rng, 8)
    x["g"][:] = -30.0
    x["gk"][:] = -5.0
    out_c, S_c = chunked(x, 8)
    out_t, S_t = token_loop(x, 8)
    assert np.isfinite(out_c).all() and np.isfinite(S_c).all()
    assert close(out_c, out_t) and close(S_c, S_t)


def test_chained_chunks_equal_a_long_prompt():
    """A 37-token prompt as chunks that end at multiples of 8 and at the
    committed count n = 21 (the prefill kernel's boundaries): outputs of all
    tokens and the state after n tokens."""
    rng = np.random.default_rng(11)
    T, n = 37, 21
    x = _inputs(rng, T)
    bounds = sorted({0, T, n} | set(range(8, T, 8)))
    S = x["S0"].copy()
    S_commit = None
    outs = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        part = {key: (val[a:b] if key not in ("S0", "scale") else val) for key, val in x.items()}
        part["S0"] = S
        o, S = chunked(part, b - a)
        outs.append(o)
        if b == n:
            S_commit = S
    out_t, S_t = token_loop(x, n)
    assert close(np.concatenate(outs), out_t)
    assert close(S_commit, S_t)


def test_a_wrong_running_product_is_caught():
    """The same check with A_ts taking one decay too many (P_{s-1->t}) fails:
    the comparison has the resolution to see an index slip."""
    rng = np.random.default_rng(13)
    x = _inputs(rng, 6)
    out_c, _ = chunked(x, 6, wrong_A=True)
    out_t, _ = token_loop(x, 6)
    assert not close(out_c, out_t)
