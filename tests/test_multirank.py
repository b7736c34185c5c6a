"""The N > 1 path of bench.py on CPU: two ranks over gloo (127.0.0.1).

The hot path shards with no exchange step (each rank runs its own replica of
the workload on its own seed: weak scaling), so the only cross-rank steps are
the barrier around the timed region, the maximum of the ranks' times, and
the reference arm's rule that rank 0 alone prints.  Those run here as two
spawned processes."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import argparse

        import bench
        import synth
        t = bench._max_over_ranks(1.5 * (rank + 1), world)
        bench._barrier(world)
        name = "decode_llama3_8b_b16_l32_t65536_d128_bf16"
        seed = synth.WORKLOAD_SEED[name] + 7919 * rank  # per-rank replica inputs
        ref = bench.run_reference(argparse.Namespace(workload=name, steps=1, warmup=0), world, rank)
        q.put((rank, t, seed, ref is None))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_rank0_reference():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(2):
        rank, t, seed, ref_none = q.get(timeout=120)
        got[rank] = (t, seed, ref_none)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # both ranks see the slower rank's time
    assert got[0][0] == got[1][0] == 3.0
    # replicas run on different inputs
    assert got[0][1] != got[1][1]
    # the reference arm: rank 1 returns without work
    assert got[1][2] is True
