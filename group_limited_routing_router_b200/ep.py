"""Expert parallelism for the Beam MoE block: each rank holds E/N experts, tokens stay with their rank.

"Welcome Beam" page, section "Multi-GPU and multi-node": each expert lives on one device while the
non-expert parameters are replicated, and the device count must divide the 256 experts.  Rank r of
N owns experts [r E/N, (r+1) E/N).  One forward pass of the layer on a rank, for its own tokens x:

  1. route x over all E experts (replicated router weights) and build the dispatch order (rows
     sorted by expert, then token), then gather x into that order.  Because the experts of a rank
     are contiguous, the rows bound for rank d are one contiguous block of the dispatch order;
  2. exchange the per-expert row counts, then the row blocks (all-to-all): each rank receives, from
     every source rank in rank order, the rows for its own experts, sorted by expert then token;
  3. run the local experts on the received rows (FP32 outputs, in the received order);
  4. send the outputs back (the reverse all-to-all): they arrive in the source's dispatch order;
  5. combine: the weighted sum in slot order, x routed_scale, bf16.
Each output row sees the same expert, the same K order and the same tile shapes as on one device,
and the combine the same FP32 order, so the result is bit-identical to the one-device forward.

The data path runs in the library's CUDA kernels (GpuOps); the exchanges are collectives of the
caller's process group (NCCL over NVLink between GPUs).  The rank's steps are written as phases
(dispatch, experts, combine) so that the same code runs with real collectives between the phases
(`forward`) or with N ranks emulated one after another in one process (`forward_emulated`), which
needs no kernel of one rank to wait for another's.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import torch


@dataclasses.dataclass(frozen=True)
class Partition:
    """Host arithmetic of the expert partition: E experts over N ranks, E/N contiguous per rank."""
    n_experts: int
    world: int

    def __post_init__(self):
        if self.world < 1 or self.n_experts % self.world:
            raise ValueError(f"the rank count {self.world} must divide the expert count {self.n_experts}")

    @property
    def per_rank(self) -> int:
        return self.n_experts // self.world

    def experts_of(self, rank: int) -> range:
        return range(rank * self.per_rank, (rank + 1) * self.per_rank)

    def owner(self, expert: int) -> int:
        return expert // self.per_rank

    def send_counts(self, counts: Sequence[int]) -> List[List[int]]:
        """Per destination rank, the per-local-expert row counts of this rank's dispatch."""
        p = self.per_rank
        return [list(counts[d * p:(d + 1) * p]) for d in range(self.world)]

    @staticmethod
    def splits(counts_by_rank: Sequence[Sequence[int]]) -> List[int]:
        """Rows per rank (dim-0 split sizes of an all-to-all)."""
        return [int(sum(c)) for c in counts_by_rank]

    @staticmethod
    def received_experts(counts_from: Sequence[Sequence[int]]) -> List[int]:
        """Local expert id of every received row: sources in rank order, each source's rows sorted
        by local expert (its dispatch order)."""
        out: List[int] = []
        for counts in counts_from:
            for e, n in enumerate(counts):
                out.extend([e] * int(n))
        return out


def _bm():
    import sys
    return sys.modules[__package__]


class GpuOps:
    """The rank's compute steps on the CUDA library (bf16 token rows, FP32 expert outputs)."""

    def __init__(self, layer, w_router, bias, w_gate, w_up, w_down):
        self.c = _bm()._cfg(layer)
        self.w_router, self.bias = w_router, bias
        self.w_gate, self.w_up, self.w_down = w_gate, w_up, w_down  # this rank's experts only

    def route(self, x):
        return _bm().route(self.c, x, self.w_router, self.bias)

    def permute(self, ids):
        p = _bm().permute(self.c, ids)
        return p, p["counts"].cpu().tolist()

    def gather_rows(self, x, dest_row):
        return _bm().gather_rows(self.c, x, dest_row)

    def expert_rows(self, x_rows, row_expert: List[int]):
        re = torch.tensor(row_expert, dtype=torch.int32, device=x_rows.device)
        return _bm().expert_rows(x_rows, re, self.w_gate, self.w_up, self.w_down)

    def combine(self, o_rows, perm, w):
        return _bm().combine(self.c, o_rows, perm["dest_row"], w)


@dataclasses.dataclass
class _Dispatch:
    perm: dict
    w: torch.Tensor
    send_rows: torch.Tensor
    send_counts: List[List[int]]


class Rank:
    """One rank's phases.  `ops` provides route / permute / gather_rows / expert_rows / combine."""

    def __init__(self, part: Partition, rank: int, ops):
        self.part, self.rank, self.ops = part, rank, ops
        self._d: Optional[_Dispatch] = None
        self._recv_counts: Optional[List[List[int]]] = None

    # phase 1: route, dispatch order, rows in that order; returns what to send to every rank
    def dispatch(self, x):
        ids, w = self.ops.route(x)
        perm, counts = self.ops.permute(ids)
        rows = self.ops.gather_rows(x, perm["dest_row"])
        self._d = _Dispatch(perm, w, rows, self.part.send_counts(counts))
        return self._d.send_rows, self._d.send_counts

    # phase 2: the local experts on the rows received from every source (in rank order)
    def experts(self, recv_rows, recv_counts: List[List[int]]):
        self._recv_counts = recv_counts
        return self.ops.expert_rows(recv_rows, self.part.received_experts(recv_counts))

    # phase 3: outputs back in dispatch order -> weighted combine
    def combine(self, o_back):
        d = self._d
        return self.ops.combine(o_back, d.perm, d.w)

    def send_splits(self) -> List[int]:
        return self.part.splits(self._d.send_counts)

    def recv_splits(self) -> List[int]:
        return self.part.splits(self._recv_counts)


def forward(rank: Rank, x, group=None):
    """One expert-parallel forward pass with torch.distributed collectives between the phases
    (every rank of `group` calls this with its own tokens; backend NCCL on GPUs, gloo on CPUs)."""
    import torch.distributed as dist
    N = rank.part.world
    rows, send_counts = rank.dispatch(x)
    # per-expert counts: [N, E/N] to send, [N, E/N] received (source-major)
    sc = torch.tensor(send_counts, dtype=torch.int64, device=rows.device).reshape(N * rank.part.per_rank)
    rc = torch.empty_like(sc)
    dist.all_to_all_single(rc, sc, group=group)
    recv_counts = rc.reshape(N, rank.part.per_rank).cpu().tolist()
    send_splits = Partition.splits(send_counts)
    recv_splits = Partition.splits(recv_counts)
    recv = _exchange(rows, send_splits, recv_splits, group)
    o = rank.experts(recv, recv_counts)
    back = _exchange(o, recv_splits, send_splits, group)
    return rank.combine(back)


def _exchange(rows, send_splits: List[int], recv_splits: List[int], group):
    """All-to-all of row blocks, as raw bytes (any row dtype on any backend)."""
    import torch.distributed as dist
    src = rows.contiguous()
    width = src.shape[1] * src.element_size()
    out = torch.empty(sum(recv_splits), width, dtype=torch.uint8, device=src.device)
    dist.all_to_all_single(out, src.view(torch.uint8).reshape(src.shape[0], width), output_split_sizes=recv_splits,
                           input_split_sizes=send_splits, group=group)
    return out.view(src.dtype).reshape(sum(recv_splits), src.shape[1])


def forward_emulated(ranks: Sequence[Rank], xs: Sequence) -> list:
    """The same exchange for N ranks in one process, phase by phase (the all-to-alls become
    concatenations of row blocks).  Returns each rank's y."""
    N = len(ranks)
    sent = [r.dispatch(x) for r, x in zip(ranks, xs)]
    blocks = []  # blocks[s][d]: rows from source s to destination d
    for rows, counts in sent:
        sp = Partition.splits(counts)
        blocks.append(list(torch.split(rows, sp, dim=0)))
    outs = []
    for d, r in enumerate(ranks):
        recv = torch.cat([blocks[s][d] for s in range(N)], dim=0)
        recv_counts = [sent[s][1][d] for s in range(N)]
        outs.append(r.experts(recv, recv_counts))
    ys = []
    for s, r in enumerate(ranks):
        pieces = []
        for d in range(N):
            sp = Partition.splits([sent[q][1][d] for q in range(N)])
            pieces.append(torch.split(outs[d], sp, dim=0)[s])
        ys.append(r.combine(torch.cat(pieces, dim=0)))
    return ys


def gpu_ranks(layer, w_router, bias, w_gate, w_up, w_down, world: int) -> List[Rank]:
    """N emulated ranks over one device's copy of the layer: rank r gets views of its E/N experts."""
    part = Partition(int(w_gate.shape[0]), world)
    out = []
    for r in range(world):
        sl = slice(r * part.per_rank, (r + 1) * part.per_rank)
        out.append(Rank(part, r, GpuOps(layer, w_router, bias, w_gate[sl], w_up[sl], w_down[sl])))
    return out

