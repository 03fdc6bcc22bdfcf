"""Pins of the packed variable-length oracle (test infrastructure).

A packed batch holds N sequences of different lengths in one head-major token grid;
every sequence is its own recurrence from its own initial state. The pins: for plain
linear attention each packed sequence equals the masked parallel form (QK^T o M) V
plus the carried initial state Q S0 (page "LinearAttention 概述", section 快速预览),
an independent formula; sequences do not see each other's data; rows outside every
sequence stay zero; an empty sequence returns its initial state.
"""
import numpy as np
import pytest

import oracle


def _packed(lens, H, dk, dv, pad, rng):
    T = sum(lens) + pad
    q = rng.standard_normal((H, T, dk))
    k = rng.standard_normal((H, T, dk))
    v = rng.standard_normal((H, T, dv))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return q, k, v, cu


@pytest.mark.parametrize("lens,pad", [([5, 0, 9, 1], 3), ([17], 0), ([0, 0], 2)])
def test_plain_packed_equals_parallel_form_per_sequence(lens, pad):
    rng = np.random.default_rng(3)
    H, dk, dv = 2, 4, 3
    q, k, v, cu = _packed(lens, H, dk, dv, pad, rng)
    s0 = rng.standard_normal((len(lens), H, dk, dv))
    o, sf = oracle.recurrent_fwd_varlen(q, k, v, cu, s0=s0, scale=0.5)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        for h in range(H):
            Q, K, V = 0.5 * q[h, a:b], k[h, a:b], v[h, a:b]
            M = np.tril(np.ones((b - a, b - a)))
            ref = ((Q @ K.T) * M) @ V + Q @ s0[n, h]
            np.testing.assert_allclose(o[h, a:b], ref, rtol=0, atol=1e-12 * max(1.0, np.abs(ref).max(initial=0)))
            np.testing.assert_allclose(sf[n, h], s0[n, h] + K.T @ V, rtol=0, atol=1e-12 * max(1.0, np.abs(sf).max()))
    # rows outside every sequence (the padding) stay zero
    assert not np.any(o[:, cu[-1]:])


def test_sequences_do_not_see_each_other():
    rng = np.random.default_rng(4)
    lens, H, dk, dv = [6, 11, 4], 2, 5, 3
    q, k, v, cu = _packed(lens, H, dk, dv, 0, rng)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((H, sum(lens)))))
    g = -0.1 * rng.random((H, sum(lens)))
    o, sf = oracle.recurrent_fwd_varlen(q, k, v, cu, beta=beta, g=g)
    # replace the middle sequence's data: the other sequences' outputs and states are unchanged
    a, b = cu[1], cu[2]
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[:, a:b] = rng.standard_normal(q2[:, a:b].shape)
    k2[:, a:b] = rng.standard_normal(k2[:, a:b].shape)
    v2[:, a:b] = rng.standard_normal(v2[:, a:b].shape)
    o2, sf2 = oracle.recurrent_fwd_varlen(q2, k2, v2, cu, beta=beta, g=g)
    np.testing.assert_array_equal(o2[:, :a], o[:, :a])
    np.testing.assert_array_equal(o2[:, b:], o[:, b:])
    np.testing.assert_array_equal(sf2[[0, 2]], sf[[0, 2]])
    assert not np.allclose(o2[:, a:b], o[:, a:b])


def test_empty_sequence_returns_initial_state_and_bad_offsets_raise():
    rng = np.random.default_rng(5)
    q, k, v, cu = _packed([3, 0, 2], 1, 2, 2, 0, rng)
    s0 = rng.standard_normal((3, 1, 2, 2))
    _, sf = oracle.recurrent_fwd_varlen(q, k, v, cu, beta=np.full((1, 5), 0.5), s0=s0)
    np.testing.assert_array_equal(sf[1], s0[1])
    with pytest.raises(ValueError):
        oracle.recurrent_fwd_varlen(q, k, v, [0, 4, 3, 5])
