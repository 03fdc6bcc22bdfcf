"""Pins of the oracle's vector-valued gate (one log-decay per key coordinate; row j of
the dk x dv state decays by alpha_t[j] = exp(g_t[j])), the per-coordinate form of the
scalar gate of page "混合注意力学习(1)", section "Gated DeltaNet":
    S_t = (I - beta_t k_t k_t^T) diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,  o_t = S_t^T q_t.
Each pin uses a formula other than the oracle's token step: the scalar gate when every
coordinate decays alike, the full product of transition matrices, and the explicit
per-coordinate decay-masked sum for linear attention."""
import numpy as np
import pytest

import oracle


def _rand(shape, rng, unit=False):
    x = rng.standard_normal(shape)
    if unit:
        x /= np.linalg.norm(x, axis=-1, keepdims=True)
    return x


@pytest.mark.parametrize("delta", [True, False])
def test_equal_coordinates_reduce_to_the_scalar_gate(delta):
    rng = np.random.default_rng(21)
    B, H, L, dk, dv = 2, 2, 45, 7, 5
    q, k = _rand((B, H, L, dk), rng), _rand((B, H, L, dk), rng, unit=True)
    v = _rand((B, H, L, dv), rng)
    beta = rng.uniform(0.1, 0.9, (B, H, L)) if delta else None
    g = rng.uniform(-0.2, 0.0, (B, H, L))
    s0 = 0.1 * _rand((B, H, dk, dv), rng)
    o1, S1 = oracle.recurrent_fwd(q, k, v, beta, g, s0)
    o2, S2 = oracle.recurrent_fwd(q, k, v, beta, np.repeat(g[..., None], dk, -1), s0)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-13 * np.abs(o1).max())
    np.testing.assert_allclose(S2, S1, rtol=0, atol=1e-13 * np.abs(S1).max())


@pytest.mark.parametrize("delta", [True, False])
@pytest.mark.parametrize("dk,dv", [(6, 4), (4, 7)])
def test_bruteforce_transition_products(delta, dk, dv):
    # closed form: S_L = P(L..1) S_0 + sum_t P(L..t+1) b_t k_t v_t^T with M_t =
    # (I - b_t k_t k_t^T) diag(alpha_t) (b_t = beta_t; M_t = diag(alpha_t), b_t = 1 without
    # the delta term) and P(b..a) = M_b ... M_a; every output from the state after its write
    rng = np.random.default_rng(22)
    L = 11
    q, k, v = _rand((L, dk), rng), _rand((L, dk), rng, unit=True), _rand((L, dv), rng)
    beta = rng.uniform(0.2, 1.0, L) if delta else None
    g = rng.uniform(-0.7, 0.0, (L, dk))
    S0 = _rand((dk, dv), rng)
    o, S = oracle.recurrent_fwd(q, k, v, beta, g, S0)
    I = np.eye(dk)
    M = []
    for t in range(L):
        D = np.diag(np.exp(g[t]))
        M.append((I - beta[t] * np.outer(k[t], k[t])) @ D if delta else D)

    def prod(b, a):           # M_b ... M_a (identity when b < a)
        P = I.copy()
        for t in range(a, b + 1):
            P = M[t] @ P
        return P

    for T_ in range(1, L + 1):
        St = prod(T_ - 1, 0) @ S0
        for t in range(T_):
            bt = beta[t] if delta else 1.0
            St = St + prod(T_ - 1, t + 1) @ (bt * np.outer(k[t], v[t]))
        np.testing.assert_allclose(o[T_ - 1], St.T @ q[T_ - 1], rtol=1e-12, atol=1e-12)
        if T_ == L:
            np.testing.assert_allclose(S, St, rtol=1e-12, atol=1e-12)


def test_plain_vector_gated_equals_decay_masked_sum():
    # linear attention: o_r = sum_{s<=r} sum_j q_r[j] k_s[j] prod_{t=s+1..r} alpha_t[j] v_s
    #                       + sum_j q_r[j] prod_{t<=r} alpha_t[j] S0[j, :]
    rng = np.random.default_rng(23)
    L, dk, dv = 17, 5, 3
    q, k, v = _rand((L, dk), rng), _rand((L, dk), rng), _rand((L, dv), rng)
    g = rng.uniform(-0.5, 0.0, (L, dk))
    S0 = _rand((dk, dv), rng)
    o, _ = oracle.recurrent_fwd(q, k, v, None, g, S0, scale=0.5)
    a = np.exp(g)
    for r in range(L):
        ref = (0.5 * q[r] * np.prod(a[: r + 1], axis=0)) @ S0
        for s in range(r + 1):
            dec = np.prod(a[s + 1: r + 1], axis=0)
            ref = ref + np.sum(0.5 * q[r] * k[s] * dec) * v[s]
        np.testing.assert_allclose(o[r], ref, rtol=1e-12, atol=1e-12)


def test_decay_acts_on_key_rows_not_value_columns():
    # a gate that zeroes key coordinate 0 at step 2 erases row 0 of the state (all value
    # columns), and nothing else
    L, dk, dv = 2, 3, 4
    k = np.zeros((L, dk)); k[0] = [1.0, 2.0, 0.5]
    v = np.zeros((L, dv)); v[0] = [1.0, -1.0, 3.0, 2.0]
    g = np.zeros((L, dk)); g[1, 0] = -np.inf
    _, S = oracle.recurrent_fwd(np.zeros((L, dk)), k, v, None, g)
    want = np.outer(k[0], v[0]); want[0] = 0.0
    np.testing.assert_array_equal(S, want)


def test_gate_shape_is_checked():
    rng = np.random.default_rng(24)
    q = _rand((2, 5, 3), rng)
    with pytest.raises(ValueError):
        oracle.recurrent_fwd(q, q, q, None, np.zeros((2, 5, 4)))


@pytest.mark.parametrize("delta", [True, False])
def test_decode_steps_with_vector_gate_and_skip_match_prefill(delta):
    # the decode entry of the oracle (its own head indexing of g, (N, H, dk), and its own
    # numpy skip term) against the pinned token recurrence over the same tokens: L decode
    # steps from S0 give the prefill's o_t at every step and its final state
    rng = np.random.default_rng(31)
    N, H, L, dk, dv = 2, 3, 12, 6, 5
    q, k = _rand((N, H, L, dk), rng), _rand((N, H, L, dk), rng, unit=True)
    v = _rand((N, H, L, dv), rng)
    beta = rng.uniform(0.1, 0.9, (N, H, L)) if delta else None
    gv = rng.uniform(-0.6, 0.0, (N, H, L, dk))
    s0 = 0.3 * _rand((N, H, dk, dv), rng)
    D = rng.standard_normal((H, dv))
    o, S = oracle.recurrent_fwd(q, k, v, beta, gv, s0, d_skip=D)
    st = np.ascontiguousarray(s0.copy())
    for t in range(L):
        ot = oracle.decode_step(q[:, :, t], k[:, :, t], v[:, :, t], None if beta is None else beta[:, :, t],
                                gv[:, :, t], st, d_skip=D)
        np.testing.assert_allclose(ot, o[:, :, t], rtol=0, atol=1e-13 * np.abs(o).max())
    np.testing.assert_allclose(st, S, rtol=0, atol=1e-13 * np.abs(S).max())
