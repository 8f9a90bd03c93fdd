"""The multi-process bench plumbing, run as two gloo ranks on the CPU.

`bench.py --gpus N` runs one process per GPU: every rank indexes its own
independent layer (weak scaling, no data-path collective), the timed region is
bracketed by barriers, and the job's time is the maximum over ranks.  These
tests run exactly that plumbing (`bench.RankGroup`, `weak_value`, `rank_seed`)
with world size 2 over gloo on 127.0.0.1.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench
import synthetic


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    try:
        ranks = bench.RankGroup("gloo", torch.device("cpu"))
        ranks.barrier()
        # each rank "times" a different step; the job's time is the slowest
        my_ms = 10.0 + 5.0 * rank
        ms_max = ranks.max(my_ms)
        # each rank draws its own layer: a different seed, hence different data
        c = dict(synthetic.CONFIGS["C0"])
        q_np, _ = synthetic.gen_iid(64, 2, 16, bench.rank_seed(c["seed"], rank))
        digest = int(q_np.astype("int64").sum())
        ranks.barrier()
        ranks.close()
        q.put((rank, ms_max, digest, bench.weak_value(world, 1024, 8, ms_max)))
    except Exception as e:  # report to the parent instead of hanging it
        q.put((rank, "error", repr(e), None))


@pytest.mark.timeout(120)
def test_two_gloo_ranks_reduce_the_max_and_scale_weakly():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, ms_max, digest, value = q.get(timeout=100)
        assert ms_max != "error", digest
        res[r] = (ms_max, digest, value)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    # the max over ranks is the slowest rank's time, seen identically by all
    assert res[0][0] == res[1][0] == 15.0
    # independent layers per rank
    assert res[0][1] != res[1][1]
    # whole-job throughput: both ranks' work over the slowest rank's time
    assert res[0][2] == pytest.approx(2 * 1024 * 8 / 0.015)


def test_single_process_needs_no_process_group():
    os.environ.pop("WORLD_SIZE", None)
    ranks = bench.RankGroup("gloo", torch.device("cpu"))
    assert ranks.world == 1
    assert ranks.max(3.5) == 3.5
    ranks.barrier()
    ranks.close()
    assert bench.weak_value(1, 100, 2, 1000.0) == pytest.approx(200.0)
