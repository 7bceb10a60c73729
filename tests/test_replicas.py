"""The multi-GPU plumbing on CPU: two gloo ranks shard independent streams with no data-path
collective and agree on the max of their timings (the bench's max-over-ranks rule)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from mla_latent_kv_window_b200 import replicas


def test_shard_covers_every_unit_once():
    for n in (0, 1, 4, 7, 1560, 4680):
        for world in (1, 2, 3, 8):
            got = [list(replicas.shard(n, r, world)) for r in range(world)]
            flat = [u for g in got for u in g]
            assert flat == list(range(n))
            assert max(map(len, got)) - min(map(len, got)) <= 1
    with pytest.raises(ValueError):
        replicas.shard(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    assert replicas.init("gloo", timeout_s=60)
    mine = list(replicas.shard(4, rank, world))          # B = 4 streams over 2 ranks
    t = 1.5 + rank                                        # this rank's "device time"
    replicas.barrier()
    q.put((rank, mine, replicas.max_over_ranks(t), replicas.sum_over_ranks(len(mine))))
    replicas.shutdown()


def test_two_gloo_ranks():
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
    assert res[0][1] == [0, 1] and res[1][1] == [2, 3]
    assert res[0][2] == res[1][2] == 2.5
    assert res[0][3] == res[1][3] == 4


def test_reference_arm_under_torchrun_prints_once():
    # The reference arm (the oracle on host cores) launched like the driver launches N > 1: rank 0
    # alone works and prints one JSON line; the other rank exits 0 without work.  CPU only.
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(root, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["steps"] == 1 and d["warmup"] == 3
