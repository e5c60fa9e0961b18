"""The benchmark's multi-process plumbing on CPU (gloo, world size 2).

The layer shards by (batch, head) with no collective on the data path: each
rank runs its own batch shard, and the only cross-rank steps are the timing
barrier and a max of the elapsed time.  These tests cover that host-side
logic without a GPU.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from mixed_head_causal_b200 import inputs as I

    class Args:
        gpus = world
    w, r, _ = bench.dist_setup(Args())
    try:
        # the time reported is the max over ranks
        t = bench.max_over_ranks(float(10 * (rank + 1)), w)
        bench.barrier(w)
        # each rank draws its own batch shard (seed = rank): shards differ
        wl = I.custom(1, 2, 8, [1])
        x = I.make_tensor(wl, rank, "q")
        gathered = [torch.zeros_like(x.float()) for _ in range(w)]
        dist.all_gather(gathered, x.float())
        q.put((rank, w, t, not torch.equal(gathered[0], gathered[1])))
    finally:
        dist.destroy_process_group()


def test_timing_max_and_distinct_shards_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, world, t, distinct in res:
        assert world == 2
        assert t == 20.0
        assert distinct


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    env = dict(os.environ, PYTHONPATH=ROOT)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "tiny_b1_h4_t256"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU refusal")
def test_our_arm_refuses_without_a_gpu():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0
    assert "no CUDA device" in (out.stderr + out.stdout)
