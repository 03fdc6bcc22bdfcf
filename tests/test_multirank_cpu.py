"""The multi-rank host path of bench.py on CPU: gloo, world size 2.

bench.py --gpus N runs one process per GPU, each on its own batch of the headline
workload (weak scaling, no data-path collective), times its steps between barriers
and reports the slowest rank's time; rank 0 alone prints, and the reference arm runs
on rank 0 only. These tests run that plumbing (the same helpers bench.py calls) in two
CPU processes over gloo, and check that a rank which dies before a collective makes the
other rank's next collective fail within the process group's timeout instead of hanging.
"""
import argparse
import datetime
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    # a short timeout where a rank is meant to die; elsewhere room for a loaded machine (rank 0
    # times the oracle while rank 1 waits in the barrier)
    pg_timeout = 10 if case == "dead_rank" else 120
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=pg_timeout))
    ok_exit = True
    try:
        import bench
        barrier, max_over_ranks = bench.rank_collectives(world)
        if case == "collectives":
            barrier()
            m = max_over_ranks(10.0 * rank + 1.5)
            agg = bench.aggregate_tokens_per_s(32768, world, m)
            q.put((rank, {"max": m, "agg": agg}))
        elif case == "shards":
            seed = bench.rank_seed(rank)
            inp = bench.W.make_prefill_inputs(1, 2, 70, 8, 8, mode="gdn", seed=seed)
            digest = torch.tensor([float(inp["q"].float().sum()), float(inp["v"].float().sum())])
            got = [torch.zeros(2) for _ in range(world)]
            dist.all_gather(got, digest)
            q.put((rank, {"seed": seed, "digests": [g.tolist() for g in got]}))
        elif case == "reference":
            args = argparse.Namespace(steps=1, warmup=0, cpu_seconds=1.0)
            line = bench.run_reference(args, rank, world)
            barrier()
            q.put((rank, line))
        elif case == "dead_rank":
            if rank == 1:
                ok_exit = False
                q.put((rank, "exiting"))
                q.close()
                q.join_thread()                  # the message is out before the process goes
                os._exit(0)                      # leaves without joining the collective
            import time
            t0 = time.time()
            try:
                max_over_ranks(1.0)
                q.put((rank, "no error"))
            except Exception as e:               # the collective must fail, not hang
                q.put((rank, f"raised: {type(e).__name__} after {time.time() - t0:.1f} s"))
            ok_exit = False
    finally:
        if ok_exit:
            dist.destroy_process_group()


def _run(case, world=2, timeout=120):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    try:
        for _ in range(world):
            r, v = q.get(timeout=timeout)
            out[r] = v
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()                          # only the processes this test started
                p.join()
    return out


def test_max_over_ranks_and_aggregate():
    out = _run("collectives")
    for r in (0, 1):
        assert out[r]["max"] == 11.5                # the slowest rank's time, on every rank
        assert out[r]["agg"] == pytest.approx(2 * 32768 / 11.5e-3)


def test_each_rank_draws_its_own_batch():
    out = _run("shards")
    assert out[0]["seed"] != out[1]["seed"]
    assert out[0]["digests"] == out[1]["digests"]   # both ranks see the same gathered pair
    d0, d1 = out[0]["digests"]
    assert d0 != d1                                  # and the two batches differ


def test_reference_arm_runs_on_rank_zero_only():
    out = _run("reference", timeout=300)
    assert out[1] is None
    line = out[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_a_dead_rank_fails_the_next_collective():
    out = _run("dead_rank", timeout=120)
    assert out[1] == "exiting"
    assert out[0].startswith("raised"), out[0]
