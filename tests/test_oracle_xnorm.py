"""Pins of the oracle's output normalisation (page "LinearAttention 概述", section "The Devil
in Linear Transformer": the normaliser's denominator is dropped and the output is normalised
instead, O = XNorm(Q (K^T V)); reading: each output row of each head normalised over its dv
values, RMS or layer normalisation, then an elementwise weight (H, dv))."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "xnorm_rows.txt")


def _golden():
    rows = []
    for line in open(GOLDEN):
        if line.strip() and not line.startswith("#"):
            kind, w0, w1, y0, y1 = line.split()
            rows.append((kind, float(w0), float(w1), float(y0), float(y1)))
    return rows


@pytest.mark.parametrize("row", _golden())
def test_hand_worked_rows(row):
    kind, w0, w1, y0, y1 = row
    q = np.array([[[1.0, 0.0]]])               # (H=1, L=1, dk=2)
    v = np.array([[[3.0, 4.0]]])
    o, _ = oracle.recurrent_fwd(q, q, v)
    assert np.array_equal(o, v)
    out = oracle.xnorm(o, kind, weight=np.array([[w0, w1]]), eps=0.0)
    np.testing.assert_allclose(out[0, 0], [y0, y1], rtol=0, atol=1e-14)


@pytest.mark.parametrize("kind", ["rms", "layer"])
def test_rows_are_normalised_per_token_and_head(kind):
    # rows of very different magnitudes (scaled per token and per head) come out with the
    # same statistics: each (head, token) row is normalised on its own, over dv
    rng = np.random.default_rng(41)
    H, L, dv = 3, 9, 8
    base = rng.standard_normal((H, L, dv))
    mag = np.exp(rng.uniform(-6, 6, (H, L, 1)))
    a = oracle.xnorm(base, kind, eps=0.0)
    b = oracle.xnorm(base * mag, kind, eps=0.0)
    np.testing.assert_allclose(b, a, rtol=0, atol=1e-12)
    ms = (a * a).mean(-1)
    np.testing.assert_allclose(ms, np.ones((H, L)), rtol=0, atol=1e-12)
    if kind == "layer":
        np.testing.assert_allclose(a.mean(-1), np.zeros((H, L)), rtol=0, atol=1e-12)


def test_normalised_gdn_output_is_invariant_to_scaling_v():
    # with S0 = 0 the GDN output is linear in v, so the normalised output does not change
    # when v is scaled (eps negligible against the row statistics)
    rng = np.random.default_rng(42)
    B, H, L, dk, dv = 2, 2, 13, 5, 6
    q = rng.standard_normal((B, H, L, dk))
    k = rng.standard_normal((B, H, L, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, H, L, dv))
    beta = rng.uniform(0.1, 0.9, (B, H, L))
    g = rng.uniform(-0.1, 0.0, (B, H, L))
    w = rng.standard_normal((H, dv))
    o1, _ = oracle.recurrent_fwd(q, k, v, beta, g)
    o2, _ = oracle.recurrent_fwd(q, k, 37.0 * v, beta, g)
    for kind in ("rms", "layer"):
        np.testing.assert_allclose(oracle.xnorm(o2, kind, w, 1e-30), oracle.xnorm(o1, kind, w, 1e-30),
                                   rtol=0, atol=1e-12)


def test_weight_is_per_head_and_channel():
    rng = np.random.default_rng(43)
    H, L, dv = 2, 4, 3
    o = rng.standard_normal((H, L, dv))
    w = np.array([[1.0, 2.0, 3.0], [-1.0, 0.5, 0.0]])
    base = oracle.xnorm(o, "rms", eps=1e-6)
    np.testing.assert_allclose(oracle.xnorm(o, "rms", w, 1e-6), base * w[:, None, :], rtol=0, atol=1e-15)
    with pytest.raises(ValueError):
        oracle.xnorm(o, "rms", np.ones((3, 3)))


def test_eps_bounds_an_all_zero_row():
    o = np.zeros((1, 2, 4))
    assert np.array_equal(oracle.xnorm(o, "rms", eps=1e-6), o)
    assert np.array_equal(oracle.xnorm(o, "layer", eps=1e-6), o)


XNORM_MUTANTS = {
    "wrong_axis": ("(x * x).mean(axis=-1, keepdims=True) + eps", "(x * x).mean(axis=-2, keepdims=True) + eps"),
    "layer_not_centred": ("x = o - o.mean(axis=-1, keepdims=True)", "x = o"),
    "weight_over_tokens": ("out = out * w[:, None, :]", "out = out * w[:, :, None].mean(axis=1, keepdims=True)"),
    "eps_outside_root": ("np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps)",
                         "(np.sqrt((x * x).mean(axis=-1, keepdims=True)) + eps)"),
}


def _xnorm_pins(mod):
    """The pins above against module ``mod``'s xnorm; names of those that fail."""
    failed = []
    for kind, w0, w1, y0, y1 in _golden():
        out = mod.xnorm(np.array([[[3.0, 4.0]]]), kind, weight=np.array([[w0, w1]]), eps=0.0)
        if not np.allclose(out[0, 0], [y0, y1], rtol=0, atol=1e-12):
            failed.append("golden")
            break
    rng = np.random.default_rng(44)
    base = rng.standard_normal((3, 9, 8))
    mag = np.exp(rng.uniform(-6, 6, (3, 9, 1)))
    for kind in ("rms", "layer"):
        a = mod.xnorm(base, kind, eps=0.0)
        b = mod.xnorm(base * mag, kind, eps=0.0)
        if not (np.allclose(a, b, rtol=0, atol=1e-12) and np.allclose((a * a).mean(-1), 1.0, rtol=0, atol=1e-12)):
            failed.append("per_row")
            break
    # eps enters under the root: a row of mean square m scales by 1 / sqrt(m + eps)
    row = np.array([[[1.0, -1.0, 1.0, -1.0]]])
    if not np.allclose(mod.xnorm(row, "rms", eps=3.0), row / 2.0, rtol=0, atol=1e-15):
        failed.append("eps")
    return failed


@pytest.mark.parametrize("name", list(XNORM_MUTANTS))
def test_planted_xnorm_mistake_is_caught(name, tmp_path):
    import importlib.util
    src = open(oracle.__file__).read()
    old, new = XNORM_MUTANTS[name]
    assert src.count(old) == 1, f"mutation site of {name} not unique"
    path = tmp_path / f"oracle_{name}.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"oracle_{name}", path)
    mut = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mut)
    assert _xnorm_pins(oracle) == []
    assert _xnorm_pins(mut), f"planted mistake {name} passed every xnorm pin"
