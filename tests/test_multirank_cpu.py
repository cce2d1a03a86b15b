"""bench.py's multi-rank host path on CPU: two gloo ranks (one spawned process each) take the
max of their timings, report the whole-job rate over all ranks and build distinct seeded
batches; the reference arm runs on rank 0 only and the other ranks exit without work."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_max_timing_and_job_rate():
    import multiprocessing as mp
    import multirank_worker
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=multirank_worker.rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, ws, rate, digests in res:
        assert got == [2.0, 5.0]                       # element-wise max over the two ranks
        assert ws == 2
        assert abs(rate - 2 * 3.0e9 / 2.0e-3) < 1e-3 * rate   # all ranks' units / the slowest time
        assert digests[0] != digests[1]                # independent batches per rank
    assert res[0][4] == res[1][4]


def _reference_arm(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                           "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_runs_on_rank_zero_only():
    r1 = _reference_arm(1)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _reference_arm(0)
    assert r0.returncode == 0, r0.stderr[-2000:]
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
