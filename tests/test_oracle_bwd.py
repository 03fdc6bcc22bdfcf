"""Pins of the oracle's gradients (page "混合注意力学习(1)", section "Transformers 就是 RNNs":
on the full training sequence all gradients follow from the chain rule through the
recurrence; the page's formulas are stripped, the reading is the exact gradient of the
definition). recurrent_bwd differentiates its own fp64 token loop by autograd; these
tests tie it to facts fixed elsewhere: its forward equals the C oracle's, central finite
differences of the C oracle's forward, and the closed-form gradients of the masked parallel
form O = (Q K^T o M) V of plain linear attention (page "LinearAttention 概述", section
"快速预览")."""
import numpy as np
import pytest

import oracle

MODES = {"plain": (False, False), "gated": (False, True), "delta": (True, False), "gdn": (True, True)}


def _inputs(rng, lead, L, dk, dv, mode):
    delta, gated = MODES[mode]
    q = rng.standard_normal(lead + (L, dk))
    k = rng.standard_normal(lead + (L, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal(lead + (L, dv))
    beta = rng.uniform(0.1, 0.9, lead + (L,)) if delta else None
    g = rng.uniform(-0.3, 0.0, lead + (L,)) if gated else None
    s0 = 0.3 * rng.standard_normal(lead + (dk, dv))
    return q, k, v, beta, g, s0


@pytest.mark.parametrize("mode", list(MODES))
def test_forward_of_the_gradient_oracle_is_the_oracle(mode):
    rng = np.random.default_rng(51)
    q, k, v, beta, g, s0 = _inputs(rng, (2, 3), 11, 5, 4, mode)
    o, S, _ = oracle.recurrent_bwd(q, k, v, beta, g, s0, do=np.ones((2, 3, 11, 4)), scale=0.7)
    o_ref, S_ref = oracle.recurrent_fwd(q, k, v, beta, g, s0, scale=0.7)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-13)
    np.testing.assert_allclose(S, S_ref, rtol=0, atol=1e-13)


@pytest.mark.parametrize("mode", list(MODES))
def test_gradients_match_finite_differences_of_the_c_oracle(mode):
    rng = np.random.default_rng(52)
    L, dk, dv = 7, 4, 3
    q, k, v, beta, g, s0 = _inputs(rng, (), L, dk, dv, mode)
    do = rng.standard_normal((L, dv))
    dsf = rng.standard_normal((dk, dv))
    _, _, gr = oracle.recurrent_bwd(q, k, v, beta, g, s0, do=do, ds_final=dsf, scale=1.3)
    args = {"q": q, "k": k, "v": v, "beta": beta, "g": g, "s0": s0}

    def loss(a):
        o, S = oracle.recurrent_fwd(a["q"], a["k"], a["v"], a["beta"], a["g"], a["s0"], scale=1.3)
        return float((o * do).sum() + (S * dsf).sum())

    h = 1e-6
    for name, gname in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("beta", "dbeta"), ("g", "dg"), ("s0", "ds0")):
        if args[name] is None:
            assert gr[gname] is None
            continue
        x = args[name]
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            num[idx] = (loss({**args, name: xp}) - loss({**args, name: xm})) / (2 * h)
        np.testing.assert_allclose(gr[gname], num, rtol=0, atol=1e-6 * max(1.0, np.abs(num).max()),
                                   err_msg=f"{mode} {gname}")


def test_plain_gradients_match_the_masked_parallel_form():
    # O = (Q K^T o M) V with M lower-triangular including the diagonal:
    # dQ = (dO V^T o M) K, dK = (dO V^T o M)^T Q, dV = (Q K^T o M)^T dO
    rng = np.random.default_rng(53)
    L, dk, dv = 13, 6, 5
    q, k, v = rng.standard_normal((L, dk)), rng.standard_normal((L, dk)), rng.standard_normal((L, dv))
    do = rng.standard_normal((L, dv))
    _, _, gr = oracle.recurrent_bwd(q, k, v, do=do)
    M = np.tril(np.ones((L, L)))
    dP = (do @ v.T) * M
    np.testing.assert_allclose(gr["dq"], dP @ k, rtol=0, atol=1e-12)
    np.testing.assert_allclose(gr["dk"], dP.T @ q, rtol=0, atol=1e-12)
    np.testing.assert_allclose(gr["dv"], ((q @ k.T) * M).T @ do, rtol=0, atol=1e-12)
