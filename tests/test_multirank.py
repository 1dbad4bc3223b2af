"""Two-rank (gloo, CPU) checks of the multi-process plumbing around the decode path.

Units are independent, so ranks exchange nothing on the data path: each rank builds its own
inputs (keyed by its rank), and the only collectives are the timing barrier and the max over
ranks. These tests run that plumbing with world size 2 on the CPU.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth_inputs as si


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, loc = bench.dist_env()
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(w)
        t = bench.max_over_ranks(1.0 + 2.5 * r, w)
        # per-rank inputs differ (seed offset by rank), as in the benchmark
        k, _ = si.keys_values(1 + r, si.unit_id(0, 0, 0, 1, 8), 64, 4)
        digest = int(np.bitwise_xor.reduce(k.reshape(-1).astype(np.uint64)))
        d = torch.tensor([digest], dtype=torch.int64)
        all_d = [torch.zeros_like(d) for _ in range(world)]
        dist.all_gather(all_d, d)
        q.put((r, w, loc, t, [int(x) for x in all_d]))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction_and_rank_keyed_inputs():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for r, (rank, w, loc, t, digests) in enumerate(res):
        assert (rank, w, loc) == (r, world, r)
        assert t == 3.5  # max over ranks of 1.0 and 3.5
        assert digests[0] != digests[1]  # ranks hold different inputs


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(2.0, 1) == 2.0
    bench.barrier(1)
