"""The N>1 host logic of bench.py on CPU: two ranks over gloo.

bench.py runs one replica per GPU (weak scaling, no data-path collective);
the only cross-rank steps are a barrier and the max-over-ranks reduction of
the timed interval, plus per-rank seeding of the inputs.  Here two CPU
processes exercise exactly those steps, and a two-process launch of the
reference arm prints one JSON line from rank 0 while rank 1 does no work.
"""
import json
import os
import socket
import subprocess
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    from combine_moe_dispatch_05_b200 import workloads as W
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        bench.barrier(world)
        mx = bench.max_over_ranks(10.0 + rank * 3.5, world)
        s = W.config(2, bench.rank_seed_offset(rank))
        ids = W.topk_ids(s.with_(T=64))
        bench.barrier(world)
        out.put((rank, mx, s.seed, int(ids.sum())))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(2))
    assert [r[1] for r in res] == [13.5, 13.5]          # both ranks see the max
    assert res[0][2] != res[1][2]                       # each replica has its own seed
    assert res[0][3] != res[1][3]                       # and so its own routing


def test_reference_arm_under_two_ranks_prints_one_line():
    env = dict(os.environ, MASTER_ADDR="127.0.0.1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1", "--warmup", "1",
           "--gpus", "2"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "GB/s"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    # the same metric, workload and direction as the library's own line
    assert d["metric"] == bench_metric() and d["higher_is_better"] is True
    assert d["config"]["workload"].startswith("dsv3_decode: T=4096 H=7168 E=256 K=8 R=8")
    assert d["steps"] == 1 and d["warmup"] == 1
    assert d["e2e"]["value"] == d["value"] == d["cpu_baseline"]["value"]


def bench_metric():
    sys.path.insert(0, ROOT)
    import bench
    return bench.METRIC
