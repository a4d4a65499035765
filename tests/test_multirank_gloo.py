"""The benchmark's multi-rank path on CPU: two gloo ranks in separate processes.

Each rank runs an independent replica of the layer; the bench brackets the timed region with a
barrier, takes the slowest rank's time and reports all ranks' tokens over that time.  Here the
ranks report different times and must agree on the whole-job rate; under the reference arm every
rank but 0 leaves without work.
"""
import os
import socket
import types

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    r = bench.Ranks("gloo", timeout_s=60)
    r.barrier()
    ms = 10.0 * (rank + 1)          # rank 1 is the slowest replica
    rate = r.rate(1000.0, ms)       # 1000 tokens per rank
    slowest = r.max(ms)
    r.close()
    q.put((rank, rate, slowest))


@pytest.mark.parametrize("world", [2])
def test_replica_rate_is_all_tokens_over_slowest_rank(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest_ms = 10.0 * world
    for rank, rate, slowest in res:
        assert slowest == slowest_ms
        assert rate == pytest.approx(world * 1000.0 / (slowest_ms / 1e3))


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    args = types.SimpleNamespace(workload="prefill", steps=1, warmup=0, gpus=2)
    assert bench.run_reference(args) is None  # returns before touching a GPU
