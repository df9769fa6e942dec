"""The multi-GPU plumbing of bench.py on CPU: two gloo ranks rendezvous on
127.0.0.1, agree on the max-over-ranks time, pass the barriers, and draw
independent replicas (no data-path exchange exists to test)."""
from __future__ import annotations

import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.multiprocessing as mp  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    r, w, _ = bench.dist_setup(world)
    assert (r, w) == (rank, world)
    t = bench.dist_max(10.0 + 5.0 * rank, world)
    bench.dist_barrier(world)
    seeds = [bench.replica_seed(rank, li) for li in range(bench.N_LAYERS)]
    out.put((rank, t, seeds))
    bench.dist_barrier(world)
    bench.dist_done(world)


def test_two_gloo_ranks_agree_on_max_time_and_draw_distinct_replicas():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res.sort()
    assert [t for _, t, _ in res] == [15.0, 15.0]
    assert not set(res[0][2]) & set(res[1][2])


def _bench(args, env_extra=None, timeout=300):
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args], env=env,
                          capture_output=True, text=True, timeout=timeout)


def test_bench_gpus_2_starts_two_ranks_itself():
    """`bench.py --gpus 2` without torchrun launches two ranks (gloo on CPU)
    and reports n_gpus 2 -- never a single replica for a request of two."""
    import json
    r = _bench(["--gpus", "2", "--plumbing-only"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert lines == [{"plumbing_only": True, "n_gpus": 2, "max_rank": 1.0}]


def test_bench_refuses_a_world_that_is_not_the_request():
    r = _bench(["--gpus", "2", "--plumbing-only"], {"WORLD_SIZE": "1", "RANK": "0",
                                                     "LOCAL_RANK": "0"})
    assert r.returncode != 0
    assert "--gpus 2 but WORLD_SIZE is 1" in r.stderr
