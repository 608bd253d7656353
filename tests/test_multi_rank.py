"""The N > 1 benchmark path on CPU: two gloo ranks (127.0.0.1).  On one GPU
the path has no exchange step, so --gpus N runs N independent replicas; what
is shared is host logic: per-rank seeding, the barrier, and the max over
ranks of the timed duration."""
import os
import socket
import subprocess
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import synth

    w_, r_, _ = bench.dist_init()
    assert (w_, r_) == (world, rank)
    bench.barrier(world)
    t = bench.max_over_ranks(10.0 + rank, world)
    w = synth.workload("tiny")
    idx, _ = synth.make_routing(w, replica=rank)
    q.put((rank, t, idx.sum()))
    bench.dist_done(world)


def test_two_gloo_ranks_replicas_and_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][1] == res[1][1] == 11.0          # both ranks see the max
    assert res[0][2] != res[1][2]                   # replicas draw different routings


def test_reference_arm_prints_once_under_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "2", "--warmup", "1", "--workload", "tiny"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    import json
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_synth_replicas_are_deterministic():
    sys.path.insert(0, ROOT)
    import synth
    w = synth.workload("decode", T=8)
    a = synth.make_routing(w, replica=1)[0]
    b = synth.make_routing(w, replica=1)[0]
    assert np.array_equal(a, b)
