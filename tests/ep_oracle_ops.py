"""The expert-parallel rank's compute steps done by the CPU oracle (test infrastructure).

The expert-parallel orchestration (group_limited_routing_router_b200/ep.py) takes its compute steps
from an `ops` object; on GPUs that is the CUDA library.  Here the same steps are the oracle's, on
host tensors, so that ranks on CPUs (gloo) exercise the partition, the dispatch order, both
exchanges and the combine against the one-process oracle: token rows travel as bf16 bit patterns
(int16 tensors), expert outputs as FP64.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle


def _np_bits(t: torch.Tensor) -> np.ndarray:
    return np.ascontiguousarray(t.numpy().view(np.uint16))


class OracleOps:
    def __init__(self, layer: dict, w_router: np.ndarray, bias, fetch, first_expert: int):
        self.layer, self.w_router, self.bias, self.fetch = layer, w_router, bias, fetch
        self.first = first_expert  # global id of this rank's local expert 0

    def route(self, x: torch.Tensor):
        r = oracle.route(_np_bits(x), self.w_router, self.layer, self.bias)
        return torch.from_numpy(r["ids"]), torch.from_numpy(r["weight"])

    def permute(self, ids: torch.Tensor):
        p = oracle.permute(ids.numpy(), self.layer["n_experts"])
        return {k: torch.from_numpy(v) for k, v in p.items()}, p["counts"].tolist()

    def gather_rows(self, x: torch.Tensor, dest_row: torch.Tensor):
        k = self.layer["topk"]
        out = torch.empty(x.shape[0] * k, x.shape[1], dtype=x.dtype)
        out[dest_row.long()] = x.repeat_interleave(k, dim=0)
        return out

    def expert_rows(self, x_rows: torch.Tensor, row_expert):
        xb = _np_bits(x_rows)
        re = np.asarray(row_expert, dtype=np.int64)
        out = np.zeros((xb.shape[0], xb.shape[1]), dtype=np.float64)
        for e in np.unique(re):
            rows = np.nonzero(re == e)[0]
            out[rows] = oracle.expert_mlp(np.ascontiguousarray(xb[rows]), *self.fetch(self.first + int(e)))
        return torch.from_numpy(out)

    def combine(self, o_back: torch.Tensor, perm: dict, w: torch.Tensor):
        T, k = w.shape
        per_slot = o_back.numpy()[perm["dest_row"].numpy()].reshape(T, k, -1)
        return torch.from_numpy(oracle.combine(per_slot, w.numpy(), self.layer["routed_scale"]))
