"""The head-split multi-GPU path, run as two gloo ranks on the CPU.

`bench.py --gpus N` runs one process per GPU and splits the heads of one layer:
rank r indexes heads `head_range(H, r, N)` as a contiguous layer of its own.
Heads are independent ("PIVOT explained", "Show Me The Code": the loop over
heads), so no rank needs another's data.  These tests check the partition, and
that indexing each rank's heads separately and putting the pieces back in rank
order gives the whole layer's result: each rank runs the oracle on its slice,
the pieces travel over a gloo all-gather (verification only, as on GPUs), and
every rank compares the assembly with the oracle on the whole layer.  They
also run the bench's own plumbing: `bench.RankGroup`'s barrier and max over
ranks, and the job throughput.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import bench
import oracle
import synthetic
from query_group_top_b200 import head_range


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("H", [1, 2, 3, 7, 8, 16, 32, 33])
def test_head_range_partitions_the_heads(H):
    for world in range(1, min(H, 9) + 1):
        ranges = [head_range(H, r, world) for r in range(world)]
        assert ranges[0][0] == 0 and ranges[-1][1] == H
        for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
            assert a1 == b0                      # contiguous, in rank order
        sizes = [b - a for a, b in ranges]
        assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
        covered = np.concatenate([np.arange(a, b) for a, b in ranges])
        assert np.array_equal(covered, np.arange(H))   # every head exactly once


def test_head_range_rejects_bad_ranks():
    with pytest.raises(ValueError):
        head_range(4, 4, 4)
    with pytest.raises(ValueError):
        head_range(0, 0, 1)


def test_sequence_split_covers_the_batch():
    for n in (1, 5, 64):
        for world in range(1, 9):
            parts = [bench.split(n, r, world) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            assert all(a1 == b0 for (_, a1), (b0, _) in zip(parts, parts[1:]))


# a small prefill layer: 4 heads over 2 ranks, several groups and a ragged tail
L, H, D, G_SZ, TOP_K, KC = 200, 4, 64, 8, 16, 40


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    try:
        import torch.distributed as dist
        ranks = bench.RankGroup("gloo", torch.device("cpu"))
        # every rank draws the same layer and keeps its own heads
        q_all, k_all = synthetic.gen_prefill(L, H, D, seed=5)
        h0, h1 = head_range(H, rank, world)
        qs = np.ascontiguousarray(q_all[:, h0:h1])
        ks = np.ascontiguousarray(k_all[:, h0:h1])
        mine = {m: oracle.prefill(qs, ks, G_SZ, TOP_K, KC, m)["out"] for m in (oracle.REFINE, oracle.REUSE)}
        ranks.barrier()
        ok = {}
        for m, piece in mine.items():
            # verification only: gather the pieces, assemble in rank order
            got = [torch.empty((L, head_range(H, r, world)[1] - head_range(H, r, world)[0], TOP_K),
                               dtype=torch.int32) for r in range(world)]
            dist.all_gather(got, torch.from_numpy(piece))
            assembled = torch.cat(got, dim=1).numpy()
            whole = oracle.prefill(q_all, k_all, G_SZ, TOP_K, KC, m)["out"]
            ok[m] = bool(np.array_equal(assembled, whole))
        # each rank "times" a different step; the job's time is the slowest
        ms_max = ranks.max(10.0 + 5.0 * rank)
        ranks.close()
        q.put((rank, ok, ms_max, bench.job_value(L, H, ms_max), (h0, h1)))
    except Exception as e:  # report to the parent instead of hanging it
        q.put((rank, "error", repr(e), None, None))


@pytest.mark.timeout(180)
def test_two_gloo_ranks_split_heads_and_reassemble_the_layer():
    oracle.build()   # once, before the ranks load it
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, ok, ms_max, value, hr = q.get(timeout=150)
        assert ok != "error", ms_max
        res[r] = (ok, ms_max, value, hr)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert res[0][3] == (0, 2) and res[1][3] == (2, 4)
    for r in range(world):
        assert res[r][0] == {oracle.REFINE: True, oracle.REUSE: True}
    # the max over ranks is the slowest rank's time, seen identically by all
    assert res[0][1] == res[1][1] == 15.0
    # whole-job throughput: the layer's query-heads over the slowest rank's time
    assert res[0][2] == pytest.approx(L * H / 0.015)


def test_single_process_needs_no_process_group():
    os.environ.pop("WORLD_SIZE", None)
    ranks = bench.RankGroup("gloo", torch.device("cpu"))
    assert ranks.world == 1
    assert ranks.max(3.5) == 3.5
    ranks.barrier()
    ranks.close()
    assert bench.job_value(100, 2, 1000.0) == pytest.approx(200.0)
