"""Multi-process host logic of the benchmark, on CPU with gloo (world size 2).

With N GPUs the benchmark runs N independent replicas (weak scaling, no
collective on the data path); ranks only agree on the timing, max over ranks.
The reference arm runs on rank 0 alone; the other ranks exit at once."""
import datetime
import json
import os
import socket
import subprocess
import sys
import time

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_ffn_16_b200.inputs import CONFIGS
    t = bench.max_over_ranks(1.5 + rank, world)
    seed = bench.replica_seed(CONFIGS["prefill_softmax"], rank)
    bench.barrier(world)
    q.put((rank, t, seed))
    dist.destroy_process_group()


def test_max_over_ranks_and_replica_seeds_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.5, 2.5]           # both ranks see the max
    assert res[0][2] != res[1][2]                       # replicas draw different batches


def _worker_one_leaves(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    sys.path.insert(0, ROOT)
    import bench
    bench.barrier(world)                        # one step completed together
    if rank == 1:
        q.put((rank, "left"))
        q.close()
        q.join_thread()                         # the message is out before the process goes
        os._exit(3)                             # leaves between steps, no collective in flight
    t0 = time.monotonic()
    try:
        bench.max_over_ranks(1.0, world)
        q.put((rank, "no error"))
    except Exception as e:  # noqa: BLE001
        q.put((rank, f"error after {time.monotonic() - t0:.1f} s: {type(e).__name__}"))


def test_rank_that_leaves_ends_the_others_collective_with_an_error():
    """Failure on the host: when one rank exits between steps, the timing
    reduction on the other rank fails within the process group's short
    timeout instead of waiting forever."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker_one_leaves, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = dict(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
    assert res[1] == "left" and ps[1].exitcode == 3
    assert res[0].startswith("error after"), res[0]
    assert float(res[0].split()[2]) < 30.0
    assert ps[0].exitcode == 0


def test_reference_arm_under_torchrun_prints_once_from_rank0():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--config", "tiny", "--steps", "2", "--warmup", "1", "--gpus", "2"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["workload"] == "tiny"
