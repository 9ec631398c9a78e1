"""The N > 1 path of bench.py on CPU: two `gloo` ranks exchange the timing
(max over ranks), every rank draws its own replica inputs, and the reference arm
under torchrun prints exactly one JSON line from rank 0 while the other ranks
exit 0 without work."""
import datetime
import json
import os
import socket
import subprocess
import sys

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        m = bench.max_over_ranks(1.5 + rank, world, "cpu")
        ids, _ = workloads.routing(64, 16, 4, "uniform", bench.replica_seed(0, rank))
        out_q.put((rank, m, ids.tobytes()))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_replica_inputs_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [m for _, m, _ in res] == [2.5, 2.5]           # every rank sees the max
    assert res[0][2] != res[1][2]                          # replicas draw different token batches


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
    assert len({bench.replica_seed(0, r) for r in range(8)}) == 8


def test_reference_arm_under_torchrun_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--config", "moe_decode_t512",
           "--ref-seconds", "0.5"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    # the reference arm describes the workload with the GPU arm's config object (same keys and values)
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    want = bench.moe_config_dict("moe_decode_t512", workloads.CONFIGS["moe_decode_t512"],
                                 bench.moe_counts(workloads.CONFIGS["moe_decode_t512"],
                                                  workloads.config_routing("moe_decode_t512")[0]), 2)
    assert d["config"] == json.loads(json.dumps(want))
