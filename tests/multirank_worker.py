"""Rank body for the two-process gloo test of bench.py's multi-rank host logic (imported by
spawned children; not a test module)."""
import datetime
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def rank_main(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch.distributed as dist

    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank 0 times [1, 5] ms, rank 1 [2, 4] ms: every rank must see [2, 5]
        got = bench.max_over_ranks([1.0 + rank, 5.0 - rank])
        ws = bench.world_size()
        rate = bench.job_rate(3.0e9, got[0], ws)
        # each rank builds its own seeded batch (rank 0 the workload's own inputs)
        w = synth.WORKLOADS[1]
        q = synth.prefill_inputs(w)[0] if rank == 0 else bench.PrefillRun._shifted(w, rank)[0]
        digests = [None] * world
        dist.all_gather_object(digests, float(np.abs(q).sum()))
        out_q.put((rank, got, ws, rate, digests))
    finally:
        dist.destroy_process_group()
