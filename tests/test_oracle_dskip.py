"""Pins of the oracle's skip term (page "【CS336】lecture4", section "继续改进：Mamba": the
output gains a term in v, like a residual connection, so the input reaches the output
without passing through the state): o_t = S_t^T q_t + D_h v_t elementwise."""
import numpy as np
import pytest

import oracle


def _gdn_inputs(rng, B, H, L, dk, dv):
    q = rng.standard_normal((B, H, L, dk))
    k = rng.standard_normal((B, H, L, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, H, L, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, H, L))))
    g = rng.uniform(-0.05, 0.0, (B, H, L))
    s0 = 0.1 * rng.standard_normal((B, H, dk, dv))
    return q, k, v, beta, g, s0


def test_zero_queries_leave_only_the_skip_term():
    # q = 0 reads nothing from the state, whatever it holds: o is the skip term alone,
    # v itself (not the delta rule's u = beta (v - S^T k)) scaled per head and channel
    rng = np.random.default_rng(11)
    B, H, L, dk, dv = 2, 3, 37, 6, 5
    q, k, v, beta, g, s0 = _gdn_inputs(rng, B, H, L, dk, dv)
    D = rng.standard_normal((H, dv))
    o, S = oracle.recurrent_fwd(np.zeros_like(q), k, v, beta, g, s0, d_skip=D)
    for b in range(B):
        for h in range(H):
            for t in range(L):
                np.testing.assert_array_equal(o[b, h, t], D[h] * v[b, h, t])
    # the skip term leaves the state untouched
    _, S_ref = oracle.recurrent_fwd(np.zeros_like(q), k, v, beta, g, s0)
    np.testing.assert_array_equal(S, S_ref)


@pytest.mark.parametrize("with_decay", [False, True])
def test_skip_term_adds_to_exact_recall(with_decay):
    # alpha = beta = 1 (DeltaNet), distinct basis keys, each token queries its own key:
    # the state returns v_t exactly (Householder identity), so o_t = v_t + D_h v_t, and
    # D = -1 cancels the recalled value to exactly zero
    rng = np.random.default_rng(12)
    H, L, d, dv = 2, 9, 12, 4
    perm = rng.permutation(d)
    keys = np.eye(d)[perm[:L]]
    k = np.broadcast_to(keys, (H, L, d)).copy()
    v = rng.integers(-6, 7, size=(H, L, dv)).astype(np.float64)
    beta = np.ones((H, L))
    g = np.zeros((H, L)) if with_decay else None
    D = np.array([[-1.0] * dv, [0.5, -2.0, 3.0, 0.25]])
    o, _ = oracle.recurrent_fwd(k, k, v, beta, g, d_skip=D)
    np.testing.assert_array_equal(o[0], np.zeros((L, dv)))
    np.testing.assert_array_equal(o[1], v[1] + D[1] * v[1])


def test_varlen_skip_term_is_per_head():
    rng = np.random.default_rng(13)
    H, dk, dv = 3, 5, 4
    lens = [7, 0, 12, 3]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T = int(cu[-1]) + 2
    q = rng.standard_normal((H, T, dk))
    k = rng.standard_normal((H, T, dk))
    v = rng.standard_normal((H, T, dv))
    beta = rng.uniform(0.1, 0.9, (H, T))
    D = rng.standard_normal((H, dv))
    o, _ = oracle.recurrent_fwd_varlen(q, k, v, cu, beta=beta, d_skip=D)
    o0, _ = oracle.recurrent_fwd_varlen(q, k, v, cu, beta=beta)
    inside = np.zeros(T, bool)
    inside[: int(cu[-1])] = True
    np.testing.assert_allclose(o[:, inside] - o0[:, inside], D[:, None, :] * v[:, inside], rtol=0, atol=1e-14)
    np.testing.assert_array_equal(o[:, ~inside], 0.0)


def test_skip_weights_must_match_heads():
    rng = np.random.default_rng(14)
    q, k, v, beta, g, s0 = _gdn_inputs(rng, 1, 2, 5, 3, 4)
    with pytest.raises(ValueError):
        oracle.recurrent_fwd(q, k, v, beta, d_skip=np.ones((4, 2)))
