"""Plant plausible mistakes in a copy of the oracle and check that the pins catch each.

Every mutant is a textual edit of a temporary copy of oracle/gdn_oracle.c (a
dropped decay, a flipped sign, a transposed index, the output read before the
write, a dropped diagonal ...), compiled with gcc on the CPU. The pins below are
the same facts tests/test_oracle_pins.py checks; a mutant passes this test only
if at least one of them rejects it, and the unmodified copy must pass them all.
"""
import os

import numpy as np
import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")

MUTANTS = {
    "read_without_decay": ("v[c] - alpha * sk[c]", "v[c] - sk[c]"),
    "blend_sign": ("(*beta) * (v[c] - alpha * sk[c])", "(*beta) * (v[c] + alpha * sk[c])"),
    "state_without_decay": ("S[j * dv + c] = alpha * S[j * dv + c] + k[j] * sk[c]",
                            "S[j * dv + c] = S[j * dv + c] + k[j] * sk[c]"),
    "output_before_write": (
        "    for (long j = 0; j < dk; ++j)\n"
        "        for (long c = 0; c < dv; ++c) S[j * dv + c] = alpha * S[j * dv + c] + k[j] * sk[c];\n"
        "    /* output from the state after this token's write */\n"
        "    read_out(S, q, scale, dk, dv, o);",
        "    read_out(S, q, scale, dk, dv, o);\n"
        "    for (long j = 0; j < dk; ++j)\n"
        "        for (long c = 0; c < dv; ++c) S[j * dv + c] = alpha * S[j * dv + c] + k[j] * sk[c];"),
    "transposed_read": ("sk[c] += S[j * dv + c] * k[j]", "sk[c] += S[c * dk + j] * k[j]"),
    "log_alpha_sign": ("exp(*g) : 1.0", "exp(-*g) : 1.0"),
    "scale_dropped": ("const double qj = scale * q[j];", "const double qj = q[j];"),
    "chunk_W_without_gamma": ("T[r * n + s] * bt[s] * exp(G[s]) * K[s * dk + j]",
                              "T[r * n + s] * bt[s] * K[s * dk + j]"),
    "chunk_Gamma_sign": ("intra += qk * exp(G[r] - G[s])", "intra += qk * exp(G[s] - G[r])"),
    "chunk_mask_without_diagonal": ("for (long s = 0; s <= r; ++s) {", "for (long s = 0; s < r; ++s) {"),
    "chunk_state_key_without_decay": ("x += exp(G[n - 1] - G[s]) * K[s * dk + j]", "x += K[s * dk + j]"),
    "chunk_solve_sign": ("x -= A[r * C + s] * T[s * n + jc]", "x += A[r * C + s] * T[s * n + jc]"),
    "ut_solve_sign": ("x -= beta[r] * exp(G[r] - G[s]) * kk * T[s * n + jc]",
                      "x += beta[r] * exp(G[r] - G[s]) * kk * T[s * n + jc]"),
}


def _pins(lib):
    """Run the oracle pins against ``lib``; return the names of those that fail."""
    failed = []
    rng = np.random.default_rng(0)

    def close(a, b, tol=1e-10):
        return np.allclose(a, b, rtol=0, atol=tol)

    # masked parallel form, plain LA (dk != dv)
    L, dk, dv = 17, 5, 3
    q, k, v = rng.standard_normal((L, dk)), rng.standard_normal((L, dk)), rng.standard_normal((L, dv))
    o, _ = oracle.recurrent_fwd(q, k, v, scale=1.0, lib=lib)
    if not close(o, ((q @ k.T) * np.tril(np.ones((L, L)))) @ v):
        failed.append("parallel_form")
    # scale multiplies q
    o2, _ = oracle.recurrent_fwd(q, k, v, scale=0.5, lib=lib)
    if not close(o2, 0.5 * o):
        failed.append("scale")
    # delta rule = decay then one SGD step (closed form of the gradient of 1/2||S^T k - v||^2)
    S0 = rng.standard_normal((6, 4))
    kk = rng.standard_normal(6)
    kk /= np.linalg.norm(kk)
    vv = rng.standard_normal(4)
    a = np.exp(-0.3)
    _, S1 = oracle.recurrent_fwd(np.zeros((1, 6)), kk[None], vv[None], beta=np.array([0.4]),
                                 g=np.array([-0.3]), s0=S0, lib=lib)
    Sb = a * S0
    if not close(S1, Sb - 0.4 * np.outer(kk, Sb.T @ kk - vv)):
        failed.append("sgd_step")
    # brute-force transition products with gates, dk != dv, outputs at every step
    L, dk, dv = 8, 6, 4
    q = rng.standard_normal((L, dk))
    k = rng.standard_normal((L, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((L, dv))
    beta = rng.uniform(0.1, 0.9, L)
    g = -rng.uniform(0, 0.3, L)
    S0n = rng.standard_normal((dv, dk))
    o, S = oracle.recurrent_fwd(q, k, v, beta, g, S0n.T, lib=lib)
    St = S0n
    ok = True
    for t in range(L):
        St = np.exp(g[t]) * St @ (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) + beta[t] * np.outer(v[t], k[t])
        ok &= close(o[t], St @ q[t])
    if not (ok and close(S, St.T)):
        failed.append("bruteforce")
    # WY product form of the UT factor
    n = 9
    K = rng.standard_normal((n, dk))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    b = rng.uniform(0.1, 0.9, n)
    gg = -rng.uniform(0, 0.3, n)
    T = oracle.ut_transform(K, b, gg, lib=lib)
    G = np.cumsum(gg)
    W = T @ np.diag(b * np.exp(G)) @ K
    P = np.eye(dk)
    for t in range(n):
        P = P @ (np.exp(gg[t]) * (np.eye(dk) - b[t] * np.outer(K[t], K[t])))
    if not close(P, np.exp(G[-1]) * np.eye(dk) - W.T @ (np.exp(G[-1] - G)[:, None] * K)):
        failed.append("wy_form")
    # chunk-size invariance, all four modes
    L = 23
    q = rng.standard_normal((2, L, dk))
    k = rng.standard_normal((2, L, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((2, L, dv))
    beta = rng.uniform(0.1, 0.9, (2, L))
    g = -rng.uniform(0, 0.2, (2, L))
    s0 = rng.standard_normal((2, dk, dv))
    for bb, gg2 in ((None, None), (None, g), (beta, None), (beta, g)):
        o_ref, S_ref = oracle.recurrent_fwd(q, k, v, bb, gg2, s0, lib=lib)
        for C in (1, 4, 8):
            oc, Sc = oracle.chunked_fwd(q, k, v, bb, gg2, s0, chunk=C, lib=lib)
            if not (close(oc, o_ref) and close(Sc, S_ref)):
                failed.append("chunk_invariance")
                break
    return failed


@pytest.fixture(scope="module")
def src_text():
    with open(SRC) as f:
        return f.read()


def _compile(text, tmp_path, name):
    c = tmp_path / f"{name}.c"
    c.write_text(text)
    return oracle.load_variant(oracle.compile_c(str(c), str(tmp_path / f"lib{name}.so")))


def test_unmodified_copy_passes_all_pins(src_text, tmp_path):
    assert _pins(_compile(src_text, tmp_path, "clean")) == []


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_is_caught(name, src_text, tmp_path):
    old, new = MUTANTS[name]
    assert src_text.count(old) == 1, f"mutation site for {name} not unique"
    failed = _pins(_compile(src_text.replace(old, new), tmp_path, name))
    assert failed, f"planted mistake {name} passed every pin"


# ------------------------------------------------------------- vector-valued gates
VG_MUTANTS = {
    "vg_log_alpha_sign": ("a[j] = gv ? exp(gv[j]) : 1.0", "a[j] = gv ? exp(-gv[j]) : 1.0"),
    "vg_decay_on_value_columns": ("for (long c = 0; c < dv; ++c) S[j * dv + c] *= a[j];",
                                  "for (long c = 0; c < dv; ++c) S[j * dv + c] *= a[c % dk];"),
    "vg_read_before_decay": (
        "    /* decay first: row j of the state by alpha[j] */\n"
        "    for (long j = 0; j < dk; ++j)\n"
        "        for (long c = 0; c < dv; ++c) S[j * dv + c] *= a[j];\n"
        "    if (beta) {",
        "    if (beta) {"),
    "vg_blend_sign": ("sk[col] = (*beta) * (v[col] - rd);", "sk[col] = (*beta) * (v[col] + rd);"),
    "vg_decode_head_index": ("c->g ? c->g + h * c->dk : NULL", "c->g ? c->g + h : NULL"),
}


def _vg_pins(lib):
    """The vector-gate pins of tests/test_oracle_vector_gate.py against ``lib``; names that fail."""
    failed = []
    rng = np.random.default_rng(3)
    # equal coordinates reduce to the scalar gate (GDN, dk != dv)
    L, dk, dv = 13, 6, 4
    q, k, v = rng.standard_normal((L, dk)), rng.standard_normal((L, dk)), rng.standard_normal((L, dv))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    beta = rng.uniform(0.2, 0.9, L)
    g = rng.uniform(-0.4, 0.0, L)
    o1, S1 = oracle.recurrent_fwd(q, k, v, beta, g, lib=lib)
    o2, S2 = oracle.recurrent_fwd(q, k, v, beta, np.repeat(g[:, None], dk, 1), lib=lib)
    if not (np.allclose(o1, o2, atol=1e-12) and np.allclose(S1, S2, atol=1e-12)):
        failed.append("vg_equal_coordinates")
    # brute-force transition products with per-coordinate decays
    gv = rng.uniform(-0.6, 0.0, (L, dk))
    S0 = rng.standard_normal((dk, dv))
    o, S = oracle.recurrent_fwd(q, k, v, beta, gv, S0, lib=lib)
    St = S0.copy()
    ok = True
    for t in range(L):
        M = (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(gv[t]))
        St = M @ St + beta[t] * np.outer(k[t], v[t])
        ok = ok and np.allclose(o[t], St.T @ q[t], atol=1e-10)
    if not (ok and np.allclose(S, St, atol=1e-10)):
        failed.append("vg_transition_products")
    # a zeroed coordinate erases its key row only
    kk = np.zeros((2, 3)); kk[0] = [1.0, 2.0, 0.5]
    vv = np.zeros((2, 4)); vv[0] = [1.0, -1.0, 3.0, 2.0]
    gz = np.zeros((2, 3)); gz[1, 0] = -np.inf
    _, Sz = oracle.recurrent_fwd(np.zeros((2, 3)), kk, vv, None, gz, lib=lib)
    want = np.outer(kk[0], vv[0]); want[0] = 0.0
    if not np.array_equal(Sz, want):
        failed.append("vg_key_rows")
    # decode steps with vector-valued gates equal the recurrence over the same tokens
    if not _decode_matches_prefill(lib, rng, vector_gate=True):
        failed.append("vg_decode_steps")
    return failed


def _decode_matches_prefill(lib, rng, vector_gate, d_skip=False, mod=oracle):
    """L decode steps of ``mod.decode_step`` (oracle library ``lib``) from S0 against the
    token recurrence of the unmodified oracle over the same tokens (several heads)."""
    N, H, L, dk, dv = 2, 3, 7, 5, 4
    q = rng.standard_normal((N, H, L, dk))
    k = rng.standard_normal((N, H, L, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((N, H, L, dv))
    beta = rng.uniform(0.1, 0.9, (N, H, L))
    g = rng.uniform(-0.6, 0.0, (N, H, L, dk) if vector_gate else (N, H, L))
    s0 = rng.standard_normal((N, H, dk, dv))
    D = rng.standard_normal((H, dv)) if d_skip else None
    o, S = oracle.recurrent_fwd(q, k, v, beta, g, s0, d_skip=D)
    st = np.ascontiguousarray(s0.copy())
    for t in range(L):
        ot = mod.decode_step(q[:, :, t], k[:, :, t], v[:, :, t], beta[:, :, t], g[:, :, t], st, lib=lib, d_skip=D)
        if not np.allclose(ot, o[:, :, t], rtol=0, atol=1e-10):
            return False
    return bool(np.allclose(st, S, rtol=0, atol=1e-10))


def test_unmodified_copy_passes_vector_gate_pins(src_text, tmp_path):
    assert _vg_pins(_compile(src_text, tmp_path, "clean_vg")) == []


@pytest.mark.parametrize("name", list(VG_MUTANTS))
def test_planted_vector_gate_mistake_is_caught(name, src_text, tmp_path):
    old, new = VG_MUTANTS[name]
    assert src_text.count(old) == 1, f"mutation site for {name} not unique"
    failed = _vg_pins(_compile(src_text.replace(old, new), tmp_path, name))
    assert failed, f"planted mistake {name} passed every vector-gate pin"


# ------------------------------------------------------------- decode skip term (numpy side)
def test_planted_decode_skip_mistake_is_caught(tmp_path):
    # the decode skip term is numpy code in oracle/__init__.py: drop it in a copy of that
    # module and check that the decode-vs-recurrence pin rejects the copy (and accepts the
    # unmodified module)
    import importlib.util
    src = open(oracle.__file__).read()
    old = "        o += D * v\n    return o"
    assert src.count(old) == 1, "mutation site of the decode skip term not unique"
    mod_path = tmp_path / "oracle_mut.py"
    mod_path.write_text(src.replace(old, "    return o"))
    spec = importlib.util.spec_from_file_location("oracle_mut", mod_path)
    mut = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mut)
    lib = oracle._load()
    assert _decode_matches_prefill(lib, np.random.default_rng(5), vector_gate=False, d_skip=True)
    assert not _decode_matches_prefill(lib, np.random.default_rng(5), vector_gate=False, d_skip=True, mod=mut)
