"""Expert parallelism on CPU ranks (gloo): partition, dispatch order, both all-to-alls and the combine.

"Welcome Beam" page, section "Multi-GPU and multi-node": each expert on one device, the device count
dividing the expert count.  N ranks in separate processes each own E/N experts and their own slice of
the tokens; the compute steps are the oracle's (tests/ep_oracle_ops.py), the orchestration is the
product's (group_limited_routing_router_b200/ep.py).  Every token's output must equal the one-process
oracle's bit for bit: each expert row is computed alone and the combine sums in the same order.
"""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import beam_synth as bs
import oracle
from group_limited_routing_router_b200 import ep


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(name):
    wl = bs.get(name)
    x = bs.make_x(wl)
    W = bs.make_router(wl).numpy()
    b = bs.load_bias(wl)
    wg, wu, wd = bs.make_experts(wl, device="cpu")
    fetch = lambda e: (oracle.bf16_bits(wg[e]), oracle.bf16_bits(wu[e]), oracle.bf16_bits(wd[e]))  # noqa: E731
    return wl, x, W, None if b is None else b.numpy(), fetch


def _token_slice(T, world, rank):
    return slice(rank * T // world, (rank + 1) * T // world)


def _rank_main(rank, world, port, name, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist

    from tests.ep_oracle_ops import OracleOps
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        wl, x, W, b, fetch = _inputs(name)
        part = ep.Partition(wl.n_experts, world)
        r = ep.Rank(part, rank, OracleOps(wl.layer, W, b, fetch, part.experts_of(rank).start))
        x_mine = x[_token_slice(wl.T, world, rank)].contiguous().view(torch.int16)
        y = ep.forward(r, x_mine)
        np.save(os.path.join(out_dir, f"y{rank}.npy"), y.numpy())
        np.save(os.path.join(out_dir, f"splits{rank}.npy"), np.array([r.send_splits(), r.recv_splits()]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,world", [("tiny", 2), ("mid_b", 2), ("mid_b", 4), ("mid_skew", 2)])
def test_ep_ranks_match_one_process_oracle(name, world):
    ctx = mp.get_context("spawn")
    port = _free_port()
    with tempfile.TemporaryDirectory() as d:
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, name, d)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
            assert p.exitcode == 0
        ys = [np.load(os.path.join(d, f"y{r}.npy")) for r in range(world)]
        splits = [np.load(os.path.join(d, f"splits{r}.npy")) for r in range(world)]
    wl, x, W, b, fetch = _inputs(name)
    ref = oracle.forward(oracle.bf16_bits(x), W, b, fetch, wl.layer)
    assert np.array_equal(np.concatenate(ys), ref["y"])
    # what rank s sent to rank d is what rank d received from s
    for s in range(world):
        for dd in range(world):
            assert splits[s][0][dd] == splits[dd][1][s]
    assert sum(int(sp[0].sum()) for sp in splits) == wl.T * wl.topk


def test_partition_arithmetic():
    p = ep.Partition(256, 8)
    assert p.per_rank == 32 and list(p.experts_of(3)) == list(range(96, 128)) and p.owner(255) == 7
    counts = list(range(256))
    sc = p.send_counts(counts)
    assert len(sc) == 8 and sc[1] == list(range(32, 64))
    assert ep.Partition.splits(sc)[0] == sum(range(32))
    assert ep.Partition.received_experts([[2, 0, 1], [0, 1, 0]]) == [0, 0, 2, 1]
    with pytest.raises(ValueError):
        ep.Partition(256, 3)


def test_emulated_ranks_match_one_process_oracle():
    """The one-process emulation of the exchange (used on a single GPU) gives the same outputs."""
    from tests.ep_oracle_ops import OracleOps
    wl, x, W, b, fetch = _inputs("mid_b")
    world = 4
    part = ep.Partition(wl.n_experts, world)
    ranks = [ep.Rank(part, r, OracleOps(wl.layer, W, b, fetch, part.experts_of(r).start)) for r in range(world)]
    xs = [x[_token_slice(wl.T, world, r)].contiguous().view(torch.int16) for r in range(world)]
    ys = ep.forward_emulated(ranks, xs)
    ref = oracle.forward(oracle.bf16_bits(x), W, b, fetch, wl.layer)
    assert np.array_equal(np.concatenate([y.numpy() for y in ys]), ref["y"])


def _failing_rank_main(rank, world, port, out_dir):
    """Rank 1 fails on the host before its first exchange (an exception, as a crashed step would);
    rank 0 runs its forward pass and must get an error from the exchange, not wait for ever."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import time

    import torch.distributed as dist

    from tests.ep_oracle_ops import OracleOps
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=10))
    wl, x, W, b, fetch = _inputs("tiny")
    part = ep.Partition(wl.n_experts, world)
    r = ep.Rank(part, rank, OracleOps(wl.layer, W, b, fetch, part.experts_of(rank).start))
    if rank == 1:
        os._exit(3)           # leaves without a word to its peer
    t0 = time.monotonic()
    try:
        ep.forward(r, x[_token_slice(wl.T, world, rank)].contiguous().view(torch.int16))
        outcome = "completed"
    except Exception as e:  # noqa: BLE001 - the kind of error depends on how gloo notices the loss
        outcome = f"error: {type(e).__name__}"
    with open(os.path.join(out_dir, "rank0.txt"), "w") as f:
        f.write(f"{outcome}\n{time.monotonic() - t0:.1f}\n")
    os._exit(0)


def test_lost_rank_surfaces_as_an_error_on_the_others():
    """Failure detection on the host: a rank that dies between steps makes the surviving rank's next
    exchange raise within the process group's timeout (10 s here) instead of hanging."""
    ctx = mp.get_context("spawn")
    port = _free_port()
    with tempfile.TemporaryDirectory() as d:
        procs = [ctx.Process(target=_failing_rank_main, args=(r, 2, port, d)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert [p.exitcode for p in procs] == [0, 3]
        with open(os.path.join(d, "rank0.txt")) as f:
            outcome, secs = f.read().splitlines()
    assert outcome.startswith("error"), outcome
    assert float(secs) < 60.0
