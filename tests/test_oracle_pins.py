"""Pins of the fp64 oracle to facts the pages and the mathematics fix.

Each test ties the oracle to something other than itself: an independent formula
(the masked parallel form, brute-force d x d transition products), a library
route (autograd for the delta rule's gradient step), a worked example with
hand-computed values (tests/golden), or an exact invariant (recall, reflection,
chunk-size invariance). A plausible slip in the oracle -- output read before the
write, a dropped decay on the read, a wrong sign, a transposed state -- fails
at least one of them (see test_planted_mistakes_are_caught).
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, rng, unit=False):
    x = rng.standard_normal(shape)
    if unit:
        x /= np.linalg.norm(x, axis=-1, keepdims=True)
    return x


# --- "LinearAttention 概述", section 快速预览 / causal mask: O = (Q K^T o M) V ---------
@pytest.mark.parametrize("L,dk,dv", [(1, 3, 2), (17, 5, 3), (64, 8, 6)])
def test_plain_la_equals_masked_parallel_form(L, dk, dv):
    rng = np.random.default_rng(1)
    q, k, v = _rand((L, dk), rng), _rand((L, dk), rng), _rand((L, dv), rng)
    o, S = oracle.recurrent_fwd(q, k, v)
    M = np.tril(np.ones((L, L)))               # lower-triangular, diagonal included
    ref = ((q @ k.T) * M) @ v
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12 * max(1.0, np.abs(ref).max()))
    np.testing.assert_allclose(S, k.T @ v, atol=1e-12)


def test_gated_la_equals_decay_masked_parallel_form():
    # unrolling S_t = a_t S_{t-1} + k_t v_t^T: o_t = sum_{s<=t} (prod_{s<i<=t} a_i) (q_t.k_s) v_s
    rng = np.random.default_rng(2)
    L, dk, dv = 23, 4, 5
    q, k, v = _rand((L, dk), rng), _rand((L, dk), rng), _rand((L, dv), rng)
    g = -rng.uniform(0, 0.5, L)
    o, _ = oracle.recurrent_fwd(q, k, v, g=g)
    D = np.zeros((L, L))
    for t in range(L):
        for s in range(t + 1):
            D[t, s] = np.prod(np.exp(g[s + 1:t + 1]))
    ref = ((q @ k.T) * D) @ v
    np.testing.assert_allclose(o, ref, atol=1e-12)


# --- "LinearAttention 概述", section Lightning Attention: positions 1..4 -----------------
def _read_cumsum_golden():
    rows, S = [], None
    with open(os.path.join(GOLDEN, "lightning_cumsum_positions_1_4.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            tok = line.split()
            if tok[0] == "S":
                S = np.array([float(x) for x in tok[1:]]).reshape(2, 2)
            else:
                rows.append([float(x) for x in tok[1:]])
    a = np.array(rows)
    return a[:, 0:2], a[:, 2:4], a[:, 4:6], a[:, 6:8], S


def test_positions_1_to_4_worked_example():
    q, k, v, expect, S_expect = _read_cumsum_golden()
    o, S = oracle.recurrent_fwd(q, k, v)
    np.testing.assert_array_equal(o, expect)     # integers: exact
    np.testing.assert_array_equal(S, S_expect)
    # chunked form at every chunk size reproduces it too
    for C in (1, 2, 3, 4):
        oc, Sc = oracle.chunked_fwd(q, k, v, chunk=C)
        np.testing.assert_allclose(oc, expect, atol=1e-13)
        np.testing.assert_allclose(Sc, S_expect, atol=1e-13)


# --- "混合注意力学习(1)", FWP & DeltaNet: the delta rule is one SGD step -------------------
@pytest.mark.parametrize("gated", [False, True])
def test_delta_rule_is_one_gradient_step(gated):
    rng = np.random.default_rng(3)
    dk, dv = 6, 4
    S0 = _rand((dk, dv), rng)
    k = _rand((1, dk), rng, unit=True)
    v = _rand((1, dv), rng)
    q = _rand((1, dk), rng)
    beta = np.array([0.37])
    g = np.array([-0.3]) if gated else None
    _, S1 = oracle.recurrent_fwd(q, k, v, beta=beta, g=g, s0=S0)
    # gated DeltaNet = weight decay then one SGD step on 1/2 ||S^T k - v||^2 with lr beta
    alpha = float(np.exp(g[0])) if gated else 1.0
    St = (torch.tensor(S0) * alpha).requires_grad_(True)
    kt, vt = torch.tensor(k[0]), torch.tensor(v[0])
    loss = 0.5 * ((St.T @ kt - vt) ** 2).sum()
    loss.backward()
    ref = (St - beta[0] * St.grad).detach().numpy()
    np.testing.assert_allclose(S1, ref, atol=1e-13)


# --- exact recall with orthogonal keys (Householder identity) -----------------------------
def _read_recall_golden():
    writes, queries = [], []
    with open(os.path.join(GOLDEN, "delta_rule_recall.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            tok = line.split()
            if tok[0] == "write":
                writes.append((int(tok[2]), [float(tok[3]), float(tok[4])]))
            else:
                queries.append((int(tok[1]), [float(tok[3]), float(tok[4])],
                                [float(tok[6]), float(tok[7])]))
    return writes, queries


@pytest.mark.parametrize("mode", ["delta", "plain"])
def test_exact_recall_worked_example(mode):
    writes, queries = _read_recall_golden()
    d = 3
    k = np.array([np.eye(d)[i] for i, _ in writes])
    v = np.array([val for _, val in writes])
    q = np.zeros_like(k)
    beta = np.ones(len(writes)) if mode == "delta" else None
    _, S = oracle.recurrent_fwd(q, k, v, beta=beta)
    for i, want_delta, want_plain in queries:
        got = S.T @ np.eye(d)[i]
        np.testing.assert_array_equal(got, want_delta if mode == "delta" else want_plain)


def test_exact_recall_many_keys_and_queries_through_outputs():
    # alpha = beta = 1, distinct basis keys: after writing m pairs, querying key j
    # (as the query of a later token whose own write uses a fresh key) returns v_j exactly
    rng = np.random.default_rng(4)
    d, m = 16, 10
    perm = rng.permutation(d)
    keys = np.eye(d)[perm[:m]]
    vals = rng.integers(-8, 8, size=(m, 5)).astype(np.float64)
    # token m+i queries key i while writing a zero value under an unused key
    spare = np.eye(d)[perm[m]]
    q = np.vstack([np.zeros((m, d)), keys])
    k = np.vstack([keys, np.tile(spare, (m, 1))])
    v = np.vstack([vals, np.zeros((m, 5))])
    o, _ = oracle.recurrent_fwd(q, k, v, beta=np.ones(2 * m))
    np.testing.assert_array_equal(o[m:], vals)


# --- Householder reflection: beta = 2, v = 0, unit k keeps ||S||_F --------------------------
def test_reflection_preserves_frobenius_norm():
    rng = np.random.default_rng(5)
    dk, dv, L = 7, 5, 9
    S0 = _rand((dk, dv), rng)
    k = _rand((L, dk), rng, unit=True)
    norms = []
    S = S0
    for t in range(L):
        _, S = oracle.recurrent_fwd(np.zeros((1, dk)), k[t:t + 1], np.zeros((1, dv)),
                                    beta=np.array([2.0]), s0=S)
        norms.append(np.linalg.norm(S))
    np.testing.assert_allclose(norms, np.linalg.norm(S0), rtol=1e-13)
    # and it is a reflection, not the identity
    assert np.abs(S - S0).max() > 1e-3


# --- brute-force products of the full d x d transition matrices ----------------------------
@pytest.mark.parametrize("dk,dv", [(4, 3), (8, 8), (16, 5)])
def test_bruteforce_transition_products(dk, dv):
    rng = np.random.default_rng(6 + dk)
    L = 12
    q = _rand((L, dk), rng)
    k = _rand((L, dk), rng, unit=True)
    v = _rand((L, dv), rng)
    beta = rng.uniform(0.05, 0.95, L)
    g = -rng.uniform(0, 0.3, L)
    S0n = _rand((dv, dk), rng)                    # value-by-key orientation of the pages
    o, S = oracle.recurrent_fwd(q, k, v, beta=beta, g=g, s0=S0n.T)
    I = np.eye(dk)
    M = [np.exp(g[t]) * (I - beta[t] * np.outer(k[t], k[t])) for t in range(L)]
    for t in range(L):
        P = np.eye(dk)
        for i in range(t + 1):
            P = P @ M[i]
        St = S0n @ P
        for s in range(t + 1):
            Ps = np.eye(dk)
            for i in range(s + 1, t + 1):
                Ps = Ps @ M[i]
            St = St + beta[s] * np.outer(v[s], k[s]) @ Ps
        np.testing.assert_allclose(o[t], St @ q[t], atol=1e-12)
    np.testing.assert_allclose(S, St.T, atol=1e-12)


# --- WY representation of the product of rank-1 corrections --------------------------------
@pytest.mark.parametrize("gated", [False, True])
def test_wy_form_of_transition_product(gated):
    rng = np.random.default_rng(7)
    n, dk = 13, 9
    K = _rand((n, dk), rng, unit=True)
    beta = rng.uniform(0.05, 0.95, n)
    g = -rng.uniform(0, 0.3, n) if gated else np.zeros(n)
    T = oracle.ut_transform(K, beta, g if gated else None)
    G = np.cumsum(g)
    gamma = np.exp(G)
    W = T @ np.diag(beta * gamma) @ K
    Kt = np.exp(G[-1] - G)[:, None] * K
    P = np.eye(dk)
    for t in range(n):
        P = P @ (np.exp(g[t]) * (np.eye(dk) - beta[t] * np.outer(K[t], K[t])))
    np.testing.assert_allclose(P, gamma[-1] * np.eye(dk) - W.T @ Kt, atol=1e-13)
    # T is unit lower-triangular
    np.testing.assert_array_equal(np.diag(T), np.ones(n))
    assert np.all(np.triu(T, 1) == 0)


# --- chunk-size invariance: C = 1 is the recurrence, C = L the parallel form ---------------
MODES = {"plain": (False, False), "gated": (False, True), "delta": (True, False), "gdn": (True, True)}


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("L", [1, 37, 70])
def test_chunk_size_invariance(mode, L):
    delta, gated = MODES[mode]
    rng = np.random.default_rng(8 + L)
    B, dk, dv = 2, 8, 6
    q = _rand((B, L, dk), rng, unit=True)
    k = _rand((B, L, dk), rng, unit=True)
    v = _rand((B, L, dv), rng)
    beta = rng.uniform(0.05, 0.95, (B, L)) if delta else None
    g = -rng.uniform(0, 0.1, (B, L)) if gated else None
    s0 = _rand((B, dk, dv), rng) * 0.1
    o_ref, S_ref = oracle.recurrent_fwd(q, k, v, beta, g, s0, scale=0.7)
    for C in sorted({1, 2, 3, 8, 64, L}):
        o, S = oracle.chunked_fwd(q, k, v, beta, g, s0, chunk=C, scale=0.7)
        np.testing.assert_allclose(o, o_ref, atol=1e-12)
        np.testing.assert_allclose(S, S_ref, atol=1e-12)


def test_chunk_equal_L_is_parallel_form_plain():
    rng = np.random.default_rng(9)
    L, dk, dv = 20, 4, 3
    q, k, v = _rand((L, dk), rng), _rand((L, dk), rng), _rand((L, dv), rng)
    o, _ = oracle.chunked_fwd(q, k, v, chunk=L)
    ref = ((q @ k.T) * np.tril(np.ones((L, L)))) @ v
    np.testing.assert_allclose(o, ref, atol=1e-12)


# --- state passing and decode -------------------------------------------------------------
def test_state_passing_and_decode_match_prefill():
    rng = np.random.default_rng(10)
    B, L1, L2, dk, dv = 3, 11, 9, 8, 5
    L = L1 + L2
    q = _rand((B, L, dk), rng, unit=True)
    k = _rand((B, L, dk), rng, unit=True)
    v = _rand((B, L, dv), rng)
    beta = rng.uniform(0.05, 0.95, (B, L))
    g = -rng.uniform(0, 0.1, (B, L))
    s0 = _rand((B, dk, dv), rng)
    o, S = oracle.recurrent_fwd(q, k, v, beta, g, s0)
    o1, S1 = oracle.recurrent_fwd(q[:, :L1], k[:, :L1], v[:, :L1], beta[:, :L1], g[:, :L1], s0)
    o2, S2 = oracle.recurrent_fwd(q[:, L1:], k[:, L1:], v[:, L1:], beta[:, L1:], g[:, L1:], S1)
    np.testing.assert_allclose(np.concatenate([o1, o2], 1), o, atol=1e-13)
    np.testing.assert_allclose(S2, S, atol=1e-13)
    st = np.ascontiguousarray(s0.copy())
    for t in range(L):
        ot = oracle.decode_step(q[:, t], k[:, t], v[:, t], beta[:, t], g[:, t], st)
        np.testing.assert_allclose(ot, o[:, t], atol=1e-13)
    np.testing.assert_allclose(st, S, atol=1e-13)


def test_output_is_linear_in_v():
    rng = np.random.default_rng(11)
    L, dk, dv = 19, 6, 4
    q = _rand((L, dk), rng, unit=True)
    k = _rand((L, dk), rng, unit=True)
    v1, v2 = _rand((L, dv), rng), _rand((L, dv), rng)
    beta = rng.uniform(0.05, 0.95, L)
    g = -rng.uniform(0, 0.1, L)
    c = -1.7
    oa, _ = oracle.recurrent_fwd(q, k, v1 + c * v2, beta, g)
    ob, _ = oracle.recurrent_fwd(q, k, v1, beta, g)
    oc, _ = oracle.recurrent_fwd(q, k, v2, beta, g)
    np.testing.assert_allclose(oa, ob + c * oc, atol=1e-12)


def test_scale_multiplies_q_only():
    rng = np.random.default_rng(12)
    L, dk, dv = 9, 5, 4
    q, k, v = _rand((L, dk), rng), _rand((L, dk), rng, unit=True), _rand((L, dv), rng)
    beta = rng.uniform(0.05, 0.95, L)
    oa, Sa = oracle.recurrent_fwd(q, k, v, beta, scale=0.25)
    ob, Sb = oracle.recurrent_fwd(0.25 * q, k, v, beta)
    np.testing.assert_allclose(oa, ob, atol=1e-14)
    np.testing.assert_array_equal(Sa, Sb)
