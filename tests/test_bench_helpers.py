"""Host-side arithmetic of bench.py: the algorithmic FLOP and byte counts it divides by, and
the seeded generators of the option inputs (no GPU)."""
import importlib.util
import os

import pytest
import torch

from gated_deltanet_sequence_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_flop_counts_per_head_token(bench):
    # GDN 2C(3dk + 2dv) + 6 dk dv and plain LA 2C(dk + dv) + 4 dk dv at d = 128, C = 64
    assert bench.flops_per_head_token("gdn", 128, 128, 64) == 180224
    assert bench.flops_per_head_token("la", 128, 128, 64) == 98304


def test_prefill_bytes_of_the_workloads(bench):
    # workload 2: q, k, v bf16 + beta, g fp32 in; o fp32 + S_final out = 683.7 MB
    assert bench.prefill_bytes(8, 16, 4096, 128, 128, 2, True, True, False, True) == 683671552
    # workload 1 (plain LA): 201.3 MB in, 134.2 MB out
    assert bench.prefill_bytes(4, 16, 4096, 128, 128, 2, False, False, False, False) == 335544320
    # the bf16 output option halves the output bytes
    full = bench.prefill_bytes(4, 16, 4096, 128, 128, 2, False, False, False, False)
    half = bench.prefill_bytes(4, 16, 4096, 128, 128, 2, False, False, False, False, out_bytes=2)
    assert full - half == 4 * 16 * 4096 * 128 * 2


def test_decode_bytes_per_step(bench):
    # 256 x 32 heads: state read + write 1073.7 MB, q, k, v, o, beta, g about 10.6 MB
    assert bench.decode_bytes(256, 32, 128, 128, 2) == 1084293120


def test_fp32_alu_peak_constant(bench):
    assert 148 * 128 * 2 * bench.FP32_CLOCK_GHZ / 1e3 == pytest.approx(74.45, abs=0.01)


def test_option_input_generators():
    g = W.make_gate_per_key((2, 3), 50, 16, seed=5, g_low=-0.3)
    assert g.shape == (2, 3, 50, 16) and g.dtype == torch.float32
    assert float(g.min()) >= -0.3 and float(g.max()) <= 0.0
    assert torch.equal(g, W.make_gate_per_key((2, 3), 50, 16, seed=5, g_low=-0.3))   # seeded
    D = W.make_dskip(4, 64, seed=6)
    assert D.shape == (4, 64) and D.dtype == torch.float32
    assert not torch.equal(D, W.make_dskip(4, 64, seed=7))
