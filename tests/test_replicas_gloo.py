"""The multi-GPU (replica) path's host logic with two gloo ranks on CPU:
rendezvous, the max-over-ranks timing, whole-job throughput, per-rank seeds,
and the benchmark's reference arm printing only on rank 0."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from invariant_numerics_b200 import replicas
    assert replicas.init("gloo", timeout_s=60)
    replicas.barrier()
    my_ms = 2.0 + rank                       # rank 1 is the slow one
    m = replicas.max_over_ranks(my_ms)
    q.put((rank, m, replicas.job_throughput(128, world, m), replicas.replica_seed(5, rank)))
    replicas.finalize()


def test_two_gloo_ranks_agree_on_the_slowest_timing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [3.0, 3.0]
    assert out[0][2] == out[1][2] == 128 * 2 / 3e-3
    assert out[0][3] != out[1][3]


def test_reference_arm_prints_once_under_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--oracle-rows", "1",
           "--kv", "128", "--batch", "2", "--hidden", "256", "--heads", "8", "--kv-heads", "2", "--ffn", "512"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=900, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["e2e"]["h2d_bytes_per_step"] == 0
