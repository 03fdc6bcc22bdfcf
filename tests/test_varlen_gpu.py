"""GPU parity of the packed variable-length entry points.

Against the fp64 oracle (every sequence its own recurrence) in every mode, on the
bf16 tensor-core path (dk = dv = 128, C = 64) and the fp32 path, with empty
sequences, one-token sequences, chunk-aligned and ragged lengths and padding rows
that belong to no sequence (they must stay untouched). Against the dense entry
points run on each sequence alone: the packed kernels must give the same bits.
Malformed offsets must come back from gdn_sync_status() as GDN_ERR_INVALID_ARG.
Error metric and bounds as in test_parity_gpu.py.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_sequence_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-3, torch.float32: 1e-5}
MODES = {"plain": (False, False), "gated": (False, True), "delta": (True, False), "gdn": (True, True)}
CASES = {"mixed": ([1, 63, 64, 65, 0, 130, 300, 7], 5), "single": ([200], 0), "empties": ([0, 0, 64, 0], 3)}


@pytest.fixture(scope="module")
def lib():
    from gated_deltanet_sequence_b200 import _lib
    return _lib


def _inputs(lens, pad, H, d, mode, dtype, seed):
    delta, gated = MODES[mode]
    inp = W.make_varlen_inputs(lens, H, d, d, mode="gdn", in_dtype=dtype, s0=True, seed=seed, pad=pad)
    if not delta:
        inp["beta"] = None
    if not gated:
        inp["g"] = None
    return inp


def _run(lib, inp, delta):
    dev = "cuda"
    q, k, v, cu = (inp[n].to(dev) for n in ("q", "k", "v", "cu_seqlens"))
    beta = None if inp["beta"] is None else inp["beta"].to(dev)
    g = None if inp["g"] is None else inp["g"].to(dev)
    s0 = inp["s0"].to(dev)
    H, T, _ = q.shape
    N = cu.numel() - 1
    o = torch.full((H, T, v.shape[-1]), float("nan"), device=dev)
    sf = torch.full((N, H, q.shape[-1], v.shape[-1]), float("nan"), device=dev)
    if delta:
        lib.gdn_chunk_fwd_varlen(q, k, v, beta, cu, g, o=o, s0=s0, s_final=sf)
    else:
        lib.lin_attn_chunk_fwd_varlen(q, k, v, cu, g, o=o, s0=s0, s_final=sf)
    assert lib.gdn_sync_status() == 0
    return o.cpu(), sf.cpu()


def _covered(cu, T):
    m = np.zeros(T, bool)
    for a, b in zip(cu[:-1], cu[1:]):
        m[a:b] = True
    return m


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_varlen_matches_oracle(lib, case, mode, dtype, d):
    lens, pad = CASES[case]
    inp = _inputs(lens, pad, 3, d, mode, dtype, seed=700 + len(lens))
    o, sf = _run(lib, inp, MODES[mode][0])
    cu = inp["cu_seqlens"].tolist()
    ref_o, ref_sf = oracle.recurrent_fwd_varlen(inp["q"], inp["k"], inp["v"], cu, beta=inp["beta"],
                                                g=inp["g"], s0=inp["s0"])
    inside = _covered(cu, o.shape[1])
    tol = TOL[dtype]
    if inside.any():
        err = oracle.max_norm_err(o[:, inside].numpy(), ref_o[:, inside])
        assert err <= tol, f"o: {err:.3e}"
    assert torch.isnan(o[:, ~inside]).all(), "rows outside every sequence were written"
    err = oracle.max_norm_err(sf.numpy(), ref_sf)
    assert err <= tol, f"S_final: {err:.3e}"


@pytest.mark.parametrize("mode", ["gdn", "plain", "gated"])
def test_varlen_equals_dense_per_sequence(lib, mode):
    lens, pad = CASES["mixed"]
    delta, _ = MODES[mode]
    inp = _inputs(lens, pad, 2, 128, mode, torch.bfloat16, seed=900)
    o, sf = _run(lib, inp, delta)
    cu = inp["cu_seqlens"].tolist()
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        if a == b:
            assert torch.equal(sf[n], inp["s0"][n]), "empty sequence: S_final must equal s0"
            continue
        sl = lambda x: None if x is None else x[:, a:b].unsqueeze(0).contiguous().cuda()
        s0 = inp["s0"][n:n + 1].cuda()
        sfd = torch.empty_like(s0)
        if delta:
            od, _ = lib.gdn_chunk_fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["beta"]), sl(inp["g"]),
                                      s0=s0, s_final=sfd)
        else:
            od, _ = lib.lin_attn_chunk_fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]), s0=s0,
                                           s_final=sfd)
        assert lib.gdn_sync_status() == 0
        assert torch.equal(od[0].cpu(), o[:, a:b]), f"sequence {n}: packed and dense outputs differ"
        assert torch.equal(sfd[0].cpu(), sf[n]), f"sequence {n}: packed and dense states differ"


@pytest.mark.parametrize("cu", [[0, 10, 5, 20], [0, 4, 30], [-1, 3, 6]])
@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_malformed_offsets_are_reported(lib, cu, dtype, d):
    H, T = 2, 24
    # unit-norm keys keep the valid sequences' states bounded (no other condition pending)
    q = torch.nn.functional.normalize(torch.randn(H, T, d, device="cuda"), dim=-1).to(dtype)
    cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
    beta = torch.full((H, T), 0.5, device="cuda")
    lib.gdn_chunk_fwd_varlen(q, q, q, beta, cu_t)
    assert lib.gdn_sync_status() == 1          # GDN_ERR_INVALID_ARG
    assert lib.gdn_sync_status() == 0          # the report clears


def test_full_size_packed_batch_sampled_sequences(lib):
    # the benchmark's packed workload: 24 sequences (log-uniform length mix), 16 heads, 32768 tokens
    w = W.VARLEN_WORKLOAD
    lens = W.draw_seqlens(w["N"], w["T"], seed=w["seed"], min_len=w["min_len"])
    inp = W.make_varlen_inputs(lens, w["H"], 128, 128, mode="gdn", in_dtype=torch.bfloat16, s0=False,
                               seed=w["seed"])
    inp["s0"] = torch.zeros(len(lens), w["H"], 128, 128)
    o, sf = _run(lib, inp, True)
    cu = inp["cu_seqlens"].tolist()
    for n, h in [(0, 0), (len(lens) // 2, 7), (int(np.argmax(lens)), 15)]:
        a, b = cu[n], cu[n + 1]
        ref_o, ref_sf = oracle.recurrent_fwd(inp["q"][h, a:b], inp["k"][h, a:b], inp["v"][h, a:b],
                                             inp["beta"][h, a:b], inp["g"][h, a:b])
        assert oracle.max_norm_err(o[h, a:b].numpy(), ref_o) <= 2e-3
        assert oracle.max_norm_err(sf[n, h].numpy(), ref_sf) <= 2e-3
