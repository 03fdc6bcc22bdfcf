"""Sequence-split (context-parallel) prefill on CPU.

The split rests on one fact of the recurrence (page "混合注意力学习(1)", section "Gated
DeltaNet": each token maps the key-row state by S -> alpha (I - beta k k^T) S + beta k v^T):
over a segment the state leaves as M S_in + N, with M the ordered product of the token maps
and N the state from a zero start, and a run from S0 = I ends in M + N. These tests pin that
on the oracle (against brute-force products of the token maps and against one run of the
whole sequence), then run the multi-rank host path of ``context_parallel_prefill`` as gloo
processes (world sizes 2 and 3, so a middle rank builds its pair), with the oracle standing
in for the CUDA kernels, and compare every rank's outputs with one oracle run of the whole
sequence.
"""
import datetime
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from gated_deltanet_sequence_b200 import workloads as W  # noqa: E402
from gated_deltanet_sequence_b200.context_parallel import segment_bounds  # noqa: E402

MODES = ["gdn", "delta", "gated", "plain"]


def _inputs(mode, H=2, L=40, d=8, seed=7):
    base = "gdn" if mode in ("gdn", "delta") else "la"
    gated = mode in ("gdn", "gated")
    inp = W.make_prefill_inputs(1, H, L, d, d, mode=base, in_dtype=torch.float32, s0=True, seed=seed,
                                gated=gated, g_low=-0.3)
    if mode == "delta":
        inp["g"] = None
    return inp


def _token_map(k, beta, g):
    """alpha (I - beta k k^T) (beta None: alpha I), fp64, written out for one token."""
    d = k.shape[0]
    alpha = 1.0 if g is None else np.exp(g)
    m = np.eye(d)
    if beta is not None:
        m = m - beta * np.outer(k, k)
    return alpha * m


@pytest.mark.parametrize("mode", MODES)
def test_run_from_identity_ends_in_transition_plus_zero_start(mode):
    inp = _inputs(mode)
    q, k, v, beta, g = (inp[n] for n in ("q", "k", "v", "beta", "g"))
    H, L, d = q.shape[1], q.shape[2], q.shape[3]
    eye = np.broadcast_to(np.eye(d), (1, H, d, d)).copy()
    _, mn = oracle.recurrent_fwd(q, k, v, beta, g, eye)
    _, n = oracle.recurrent_fwd(q, k, v, beta, g, None)
    kk = k.double().numpy()
    for h in range(H):
        M = np.eye(d)
        for t in range(L):
            M = _token_map(kk[0, h, t], None if beta is None else float(beta[0, h, t]),
                           None if g is None else float(g[0, h, t])) @ M
        np.testing.assert_allclose(mn[0, h] - n[0, h], M, rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode", MODES)
def test_composed_segments_equal_one_run(mode):
    inp = _inputs(mode, L=70)
    q, k, v, beta, g, s0 = (inp[n] for n in ("q", "k", "v", "beta", "g", "s0"))
    H, L, d = q.shape[1], q.shape[2], q.shape[3]
    o_ref, s_ref = oracle.recurrent_fwd(q, k, v, beta, g, s0)
    b = [0, 17, 40, 41, 70]                         # uneven, one segment of a single token
    s_in = s0.double().numpy()[0]
    eye = np.broadcast_to(np.eye(d), (1, H, d, d)).copy()
    for a, e in zip(b[:-1], b[1:]):
        sl = slice(a, e)
        part = [None if t is None else t[:, :, sl] for t in (q, k, v, beta, g)]
        o_seg, _ = oracle.recurrent_fwd(*part, s_in[None])
        np.testing.assert_allclose(o_seg, o_ref[:, :, sl], rtol=0, atol=1e-12)
        _, mn = oracle.recurrent_fwd(*part, eye)
        _, n = oracle.recurrent_fwd(*part, None)
        s_in = np.einsum("hij,hjk->hik", mn[0] - n[0], s_in) + n[0]
    np.testing.assert_allclose(s_in, s_ref[0], rtol=0, atol=1e-12)


def test_segment_bounds_follow_chunks():
    assert segment_bounds(4096, 4) == [0, 1024, 2048, 3072, 4096]
    assert segment_bounds(300, 4) == [0, 64, 128, 192, 300]        # 5 chunks over 4 segments
    assert segment_bounds(100, 8) == [0, 64, 100]                  # no more segments than chunks
    assert segment_bounds(0, 3) == [0, 0]
    b = segment_bounds(65536, 3)
    assert b[0] == 0 and b[-1] == 65536 and all(x % 64 == 0 for x in b[:-1])


class OracleOps:
    """CPU stand-ins for the library calls (fp64 oracle, results stored in the fp32 buffers)."""

    @staticmethod
    def prefill(q, k, v, beta, g, s0, o, s_final, chunk, scale, stream=None):
        oo, sf = oracle.recurrent_fwd(q, k, v, beta, g, s0, scale=scale)
        o.copy_(torch.from_numpy(oo))
        s_final.copy_(torch.from_numpy(sf))

    @staticmethod
    def identity(count, d, device, value=1.0, stream=None):
        return value * torch.eye(d, dtype=torch.float32).repeat(count, 1, 1)

    @staticmethod
    def compose(mn, n, s_in, out, lam=1.0, stream=None):
        out.copy_(torch.matmul((mn - n).double() / lam, s_in.double()) + n.double())
        return out


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, mode, bounds, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from gated_deltanet_sequence_b200.context_parallel import context_parallel_prefill
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        inp = _inputs(mode, L=bounds[-1])
        sl = slice(bounds[rank], bounds[rank + 1])
        part = {n: (None if inp[n] is None else inp[n][:, :, sl].contiguous())
                for n in ("q", "k", "v", "beta", "g")}
        o, s_end = context_parallel_prefill(part["q"], part["k"], part["v"], part["beta"], part["g"],
                                            inp["s0"] if rank == 0 else None, ops=OracleOps)
        q.put((rank, (o.numpy(), s_end.numpy())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode,bounds", [("gdn", [0, 23, 50]), ("gdn", [0, 20, 37, 64]),
                                         ("plain", [0, 30, 31, 64]), ("delta", [0, 16, 48, 64])])
def test_ranks_exchange_pairs_and_match_one_run(mode, bounds):
    world = len(bounds) - 1
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, mode, bounds, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    try:
        for _ in range(world):
            r, val = q.get(timeout=180)
            out[r] = val
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()                          # only the processes this test started
                p.join()
    inp = _inputs(mode, L=bounds[-1])
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["s0"])
    for r in range(world):
        o, s_end = out[r]
        ref_o = o_ref[:, :, bounds[r]:bounds[r + 1]]
        assert oracle.max_norm_err(o, ref_o) < 1e-5, r
        # every rank ends with the state at the end of its segment (the last: the final state)
        upto = {n: (None if inp[n] is None else inp[n][:, :, :bounds[r + 1]]) for n in ("q", "k", "v", "beta", "g")}
        _, s_upto = oracle.recurrent_fwd(upto["q"], upto["k"], upto["v"], upto["beta"], upto["g"], inp["s0"])
        assert oracle.max_norm_err(s_end, s_upto) < 1e-5, r
    assert oracle.max_norm_err(out[world - 1][1], s_ref) < 1e-5
