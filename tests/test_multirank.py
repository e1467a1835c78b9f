"""Host logic of the multi-GPU bench on CPU: two gloo ranks, each running
its own batch (weak scaling, no data-path collective), reduce their step
times with a MAX all-reduce, and only rank 0 reports.  The rank/seed and
reduction code is the same that bench.py uses."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import sa3_inputs
    # each rank draws its own batch (seed = rank)
    qq, _, _ = sa3_inputs.make_qkv("tiny_b1h2n256d64", seed=rank)
    t = torch.tensor([float(rank + 1)], dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    digest = float(qq.float().sum())
    q.put((rank, float(t.item()), digest))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_max_reduce_and_independent_batches():
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
    assert [r[1] for r in res] == [2.0, 2.0]      # max over ranks
    assert res[0][2] != res[1][2]                 # different batches per rank


def test_bench_cli_rejects_world_mismatch(monkeypatch):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")
    with pytest.raises(SystemExit):
        bench.dist_init(2)


def test_bench_reference_arm_under_torchrun_two_ranks():
    """bench.py itself, launched as the multi-GPU runs are (torchrun, one
    process per rank), on the reference arm (CPU oracle; gloo on a host
    without CUDA): rank 0 prints the one JSON line for the whole job, the
    other rank exits 0 without work."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(root, "bench.py"),
           "--gpus", "2", "--impl", "reference", "--workload", "tiny_b1h2n256d64", "--steps", "2", "--warmup", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
