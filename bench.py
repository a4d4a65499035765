#!/usr/bin/env python
"""Benchmark of the Beam MoE block forward pass (group-limited routing + 8 SwiGLU experts) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill] [--impl ours|reference]

One step = one beam_moe_forward call over one batch (router, dispatch, gather, gate/up + SwiGLU
GEMM, down GEMM, combine) with inputs and the 20.1 GB of expert weights already resident in HBM.
The default workload is the T=4096 prefill chunk at Beam shapes.  Under torchrun each rank runs an
independent replica (the path has no exchange step on one layer); value = tokens of all ranks /
max-over-ranks device time.  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (plain FP64 C, the test oracle) on a bounded token sample of the
same workload on this host's cores; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import beam_synth as bs  # noqa: E402

METRIC = "MoE-layer tokens/s (Beam shape, BF16, T=4096) and % of tensor/HBM roofline"
METRIC_FP8 = "MoE-layer tokens/s (Beam shape, MXFP8 expert weights, T=4096) and % of tensor/HBM roofline"
METRIC_W4A4 = ("MoE-layer tokens/s (Beam shape, NVFP4 expert weights and activations on block-scaled tensor cores, "
               "T=4096) and % of tensor/HBM roofline")
METRIC_MXFP8 = ("MoE-layer tokens/s (Beam shape, MXFP8 expert weights and activations on block-scaled tensor cores, "
                "T=4096) and % of tensor/HBM roofline")
METRIC_NVFP4 = "MoE-layer tokens/s (Beam shape, NVFP4 expert weights, T=4096) and % of tensor/HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant kernel, keyed by
# (kernel, workload).  Taken with ncu on a 32-expert case with the same rows per expert as the workload
# (decode: T=32, prefill: T=512, long: T=8192; one launch each) and scaled by 256/32 = 8 to the full
# layer: each expert's weights and rows are its own traffic, so reads grow in proportion.  Writes of the
# small case partly stay in the 126 MB L2, so the scaled figure understates full-size writes by up to
# the kernel's output size.  An entry counts only while the sources it was captured from hash the same;
# otherwise the JSON line reports null.
_CSRC = os.path.join(ROOT, "group_limited_routing_router_b200", "csrc")
_BF16_SRC = ("gemm.cuh", "gemm_2sm.cuh", "common.cuh", "beam_moe.cu")  # beam_moe.cu picks the variants
_MX_SRC = ("gemm_mx8.cuh", "gemm.cuh", "common.cuh", "beam_moe.cu")
_H1, _H2 = "c93cc758952df2fd", "c38934599f27bc8c"
NCU_TRAFFIC = {
    ("gate_up_swiglu", "decode"): {"bytes": 8 * (1678104832 + 400896), "files": _BF16_SRC, "hash": _H1},
    ("gate_up_swiglu", "prefill"): {"bytes": 8 * (1748065536 + 4208640), "files": _BF16_SRC, "hash": _H1},
    ("gate_up_swiglu", "long"): {"bytes": 8 * (6605592576 + 331901184), "files": _BF16_SRC, "hash": _H1},
    ("down", "decode"): {"bytes": 8 * (840216064 + 3623680), "files": _BF16_SRC, "hash": _H1},
    ("down", "prefill"): {"bytes": 8 * (863484160 + 33014272), "files": _BF16_SRC, "hash": _H1},
    ("down", "long"): {"bytes": 8 * (1509199360 + 1311041024), "files": _BF16_SRC, "hash": _H1},
    ("gate_up_swiglu_w4a4", "decode"): {"bytes": 8 * (472080384 + 357120), "files": _MX_SRC, "hash": _H2},
    ("gate_up_swiglu_w4a4", "prefill"): {"bytes": 8 * (483272192 + 3281408), "files": _MX_SRC, "hash": _H2},
    ("down_w4a4", "decode"): {"bytes": 8 * (236404224 + 1159168), "files": _MX_SRC, "hash": _H2},
    ("down_w4a4", "prefill"): {"bytes": 8 * (241893632 + 25558272), "files": _MX_SRC, "hash": _H2},
    ("gate_up_swiglu_mxfp8", "decode"): {"bytes": 8 * (865321216 + 864768), "files": _MX_SRC, "hash": _H2},
    ("gate_up_swiglu_mxfp8", "prefill"): {"bytes": 8 * (887475712 + 1669632), "files": _MX_SRC, "hash": _H2},
    ("down_mxfp8", "decode"): {"bytes": 8 * (433307392 + 1774592), "files": _MX_SRC, "hash": _H2},
    ("down_mxfp8", "prefill"): {"bytes": 8 * (444443392 + 5229312), "files": _MX_SRC, "hash": _H2},
}


def traffic_of(kernel, fmt, workload):
    tr = NCU_TRAFFIC.get((kernel + ("" if fmt == "bf16" else "_" + fmt), workload))
    return tr["bytes"] if tr and files_hash(tr["files"]) == tr["hash"] else None


def files_hash(names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(_CSRC, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill", choices=["decode", "prefill", "skew", "long"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--also", default=None,
                    help="comma-separated workloads timed after the headline one in the same process "
                         "(default: decode,skew,long for bf16, decode for --fp8/--mxfp8/--nvfp4, none for --block)")
    ap.add_argument("--cpu-sample", type=int, default=1024, help="tokens in the CPU-oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--experts", type=int, default=None,
                    help="profiling only: a reduced Beam-shaped layer with this many experts (8 groups, keep 4, top 8)")
    ap.add_argument("--tokens", type=int, default=None, help="profiling only: override the workload's T")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism over the N ranks (E/N experts each, all-to-all dispatch and combine); "
                         "each rank brings its own batch of the workload (weak scaling)")
    ap.add_argument("--dense", action="store_true",
                    help="time the dense SwiGLU MLP of Beam's first layers (T=4096, intermediate 20480)")
    ap.add_argument("--block", action="store_true",
                    help="time the MoE sublayer on the residual stream (pre-norm, block, post-norm, residual)")
    ap.add_argument("--nvfp4", action="store_true",
                    help="NVFP4 expert weights (E2M1 + E4M3 scale per 16 K elements + FP32 per-matrix scale)")
    ap.add_argument("--fp8", action="store_true",
                    help="MXFP8 expert weights (E4M3 + one power-of-two scale per 32 K elements)")
    ap.add_argument("--w4a4", action="store_true",
                    help="the 4-bit path: NVFP4 weights and activations, block-scaled tcgen05 MMA")
    ap.add_argument("--mxfp8", action="store_true",
                    help="the native FP8 path: MXFP8 weights and activations, block-scaled tcgen05 MMA")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "group_limited_routing_router_b200", "csrc")
    for n in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# ------------------------------------------------------------------------------------------------
# algorithmic work (bytes the method must move, flops it must do), per step
def algorithmic(wl: bs.Workload, n_act: int, fmt: str = "bf16") -> dict:
    """The layer's algorithmic work and each stage's share of it.

    Layer bytes = each active expert's weights once + W_r + x in + y out + ids and weights; the
    dispatch copies (x_perm), h and the FP32 expert outputs are implementation choices and count in
    no stage's algorithmic bytes (they appear in the ncu traffic).  Stage shares: router = x, W_r
    and its ids/weights out; gate/up = its weights + x; down = its weights; combine = y out + the
    ids/weights it reads; dispatch and gather = the ids they read.
    fmt "fp8": expert weights are 1-byte E4M3 codes plus one 1-byte scale code per 32 elements;
    "nvfp4": half-byte E2M1 codes plus one 1-byte scale code per 16 elements (the per-matrix FP32
    scales are negligible)."""
    T, H, I, E, k = wl.T, wl.hidden, wl.inter, wl.n_experts, wl.topk
    R = T * k
    wb = {"bf16": 2.0, "fp8": 1.0 + 1.0 / 32, "mxfp8": 1.0 + 1.0 / 32, "nvfp4": 0.5 + 1.0 / 16,
          "w4a4": 0.5 + 1.0 / 16}[fmt]  # bytes per expert weight element
    w_expert = 3 * H * I * wb
    return dict(
        layer_flops=T * (2 * H * E + k * 6 * H * I),
        layer_bytes=n_act * w_expert + E * H * 4 + 2 * T * H * 2 + T * k * 8,
        stage_bytes={
            "router": T * H * 2 + E * H * 4 + T * k * 8,
            "dispatch": T * k * 4,
            "gather": T * k * 4,
            "gate_up_swiglu": n_act * 2 * I * H * wb + T * H * 2,
            "down": n_act * H * I * wb,
            "combine": T * H * 2 + T * k * 8,
        },
        stage_flops={"router": 2 * T * H * E, "gate_up_swiglu": 4 * R * H * I, "down": 2 * R * H * I},
    )


# ------------------------------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clock / throttle samples every 200 ms while the GPU works."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        self.gpu = vis.split(",")[local_rank] if vis else str(local_rank)
        self.file = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
        self.proc = None
        self.marks = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                                          "-i", self.gpu, "-lms", "200"], stdout=self.file,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.5)

    def n_samples(self) -> int:
        self.file.flush()
        with open(self.file.name) as f:
            return sum(1 for ln in f if ln.strip())

    def mark(self):
        self.marks.append(self.n_samples())

    def stop(self) -> dict:
        """Stops sampling; returns the summary of every sample taken."""
        self.rows = []
        if self.proc is not None:
            self.proc.terminate()
            self.proc.wait()
            with open(self.file.name) as f:
                self.rows = [ln.strip().split(", ") for ln in f if ln.strip()]
        return self.summary(0, len(self.rows))

    def summary(self, lo: int, hi: int) -> dict:
        """Median SM clock, max clock, throttle reasons and peak power over samples [lo, hi)."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        sel = self.rows[lo:hi] if hi > lo else self.rows
        sm = [float(r[1]) for r in sel if len(r) > 1 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in sel if len(r) > 2 and r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in sel for i in range(4) if len(r) > 5 + i and r[5 + i] == "Active"})
        power = [float(r[3]) for r in sel if len(r) > 3 and r[3].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(sel), "power_w_max": max(power) if power else None}

    def cleanup(self):
        try:
            os.unlink(self.file.name)
        except OSError:
            pass


# ------------------------------------------------------------------------------------------------
def bf16_fetch(wg, wu, wd):
    """One expert's weights for the oracle: bf16 bits from one host copy of the layer (made on first use)."""
    host = []

    def fetch(e):
        if not host:
            host.extend(t.cpu().view(torch.int16).numpy().view(np.uint16) for t in (wg, wu, wd))
        return host[0][e], host[1][e], host[2][e]
    return fetch


def fp8_fetch(w8):
    """One expert's weights for the oracle: MXFP8 codes dequantised on the host by the oracle."""
    import oracle
    return lambda e: tuple(oracle.dequant_mxfp8(w8["q_" + n][e].cpu().numpy(), w8["s_" + n][e].cpu().numpy())
                           for n in ("gate", "up", "down"))


def nvfp4_fetch(w4):
    """One expert's weights for the oracle: NVFP4 codes dequantised to FP64 on the host by the oracle."""
    import oracle
    return lambda e: tuple(oracle.dequant_nvfp4(w4["q_" + n][e].cpu().numpy(), w4["s_" + n][e].cpu().numpy(),
                                                float(w4["g_" + n][e].cpu())) for n in ("gate", "up", "down"))


def cpu_oracle_rate(wl, x_cpu, W, bias, fetch, n_sample: int, route_all: bool = True, fmt: str = "bf16") -> dict:
    """Time the CPU oracle: routing (FP64 scores + selection) and the expert half on a token sample.
    fetch(e) gives one expert's bf16 weight bits on the host; it runs outside the timed sections."""
    import oracle
    xb = oracle.bf16_bits(x_cpu)
    b = None if bias is None else bias.cpu().numpy()
    Wn = W.cpu().numpy()
    T = wl.T
    tok = bs.sample_tokens(wl, n_sample)
    t0 = time.perf_counter()
    if route_all:
        r = oracle.route(xb, Wn, wl.layer, b)
        ids, wts = r["ids"][tok], r["weight"][tok]
        t_route_tok = (time.perf_counter() - t0) / T
    else:
        r = oracle.route(np.ascontiguousarray(xb[tok]), Wn, wl.layer, b)
        ids, wts = r["ids"], r["weight"]
        t_route_tok = (time.perf_counter() - t0) / len(tok)
    xs = np.ascontiguousarray(xb[tok])
    out = np.zeros((len(tok), wl.topk, wl.hidden))
    t_exp = 0.0
    for e in range(wl.n_experts):
        rows, slots = np.nonzero(ids == e)
        if rows.size == 0:
            continue
        w3 = fetch(e)
        t1 = time.perf_counter()
        expert = {"nvfp4": oracle.expert_mlp_f64, "mxfp8": oracle.expert_mlp_mx8,
                  "w4a4": oracle.expert_mlp_w4a4}.get(fmt, oracle.expert_mlp)
        out[rows, slots, :] = expert(xs[rows], *w3)
        t_exp += time.perf_counter() - t1
    t1 = time.perf_counter()
    y = oracle.combine(out, wts, wl.routed_scale)
    t_exp += time.perf_counter() - t1
    secs = t_route_tok * len(tok) + t_exp
    return {"value": len(tok) / secs, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "seconds": secs, "tok": tok, "ids": ids, "y": y,
            "sample": (f"router + group-limited selection on {'all ' + str(T) if route_all else len(tok)} tokens, "
                       f"SwiGLU experts + combine on {len(tok)} seeded tokens of the {wl.name} batch; "
                       "tokens/s = sample / (per-token routing time x sample + expert time)")}


def parity_of(y_gpu, ids_gpu, tok, ids_oracle, y_oracle) -> dict:
    """Raw output error of the timed forward pass on the CPU baseline's token sample (the oracle's
    routing and outputs): the tokens whose GPU expert set is the oracle's are compared; the others
    (decision margins below 1e-6) are counted."""
    yg = y_gpu[torch.from_numpy(np.asarray(tok)).to(y_gpu.device)].float().cpu().numpy().astype(np.float64)
    ig = ids_gpu[torch.from_numpy(np.asarray(tok)).to(ids_gpu.device)].cpu().numpy()
    same = np.array([set(a.tolist()) == set(b.tolist()) for a, b in zip(ig, ids_oracle)])
    yo = y_oracle[same]
    err = np.abs(yg[same] - yo)
    rms = float(np.sqrt(np.mean(yo ** 2)))
    row_rms = np.sqrt(np.mean(yo ** 2, axis=1))
    return {"tokens": int(same.sum()), "tokens_other_expert_set": int((~same).sum()),
            "max_abs_err_over_rms": float(err.max() / rms),
            "worst_row_max_err_over_row_rms": float((err.max(axis=1) / row_rms).max()),
            "note": "raw figures on the oracle's sample; the tests' pass rule is per token, 2e-2 x the row RMS "
                    "where BF16 spacing allows and as the distance to the BF16 rounding interval everywhere"}


# ------------------------------------------------------------------------------------------------
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = bs.get(args.workload)
    torch.cuda.set_device(0)
    x = bs.make_x(wl)
    W = bs.make_router(wl)
    bias = bs.load_bias(wl)
    wg, wu, wd = bs.make_experts(wl, device="cuda")
    # one host copy of the layer (the oracle reads each expert it needs from it, untimed)
    host = tuple(t.cpu().view(torch.int16).numpy().view(np.uint16) for t in (wg, wu, wd))
    del wg, wu, wd
    fetch = lambda e: (host[0][e], host[1][e], host[2][e])  # noqa: E731
    n = 32
    rates, secs = [], []
    for i in range(args.warmup + args.steps):
        r = cpu_oracle_rate(wl, x, W, bias, fetch, n, route_all=False)
        if i >= args.warmup:
            rates.append(r)
            secs.append(r["seconds"])
    tot = sum(secs)
    value = n * args.steps / tot
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(wl),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": rates[0]["cores"], "kind": "oracle",
                             "sample": f"each step: the whole block (routing + experts + combine) for {n} seeded "
                                       f"tokens of the {wl.name} batch, FP64 CPU oracle"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def config_dict(wl):
    return {"workload": f"{wl.name}: {wl.description}", "T": wl.T, "hidden": wl.hidden, "inter": wl.inter,
            "n_experts": wl.n_experts, "n_groups": wl.n_groups, "topk_groups": wl.topk_groups, "topk": wl.topk,
            "routed_scale": wl.routed_scale, "weights_bytes": 3 * wl.n_experts * wl.hidden * wl.inter * 2,
            "l2": "no flush: every step streams the 20.1 GB of expert weights (> 126 MB L2)",
            "parallelism": "replicas (one independent layer instance per GPU)"}


def launches_per_step(wl: bs.Workload, block: bool, fmt: str = "bf16") -> int:
    """Kernels one forward launches: the router (the direct kernel below 2048 tokens; from 2048 the
    screened router's five: plane split, tensor-core projection, screen, exact path, finish),
    3 dispatch kernels, [row gather for wide tiles], [activation quantiser on the block-scaled paths],
    gate/up, down, combine; the sublayer adds the pre-norm (its combine is the fused post-norm kernel)."""
    wide = wl.T * wl.topk / wl.n_experts > 12.0
    screened = wl.T >= 2048 and wl.n_experts <= 256 and wl.topk <= 8 and wl.n_groups <= 32
    return (5 if screened else 1) + 6 + (1 if wide else 0) + (1 if block else 0) + (1 if fmt in ("mxfp8", "w4a4") else 0)


class Ranks:
    """One process per GPU: barrier, max-over-ranks and the whole-job rate of independent replicas.

    backend "nccl" on GPUs; "gloo" works the same way on CPU (used by the multi-rank tests)."""

    def __init__(self, backend: str = "nccl", timeout_s: int = 120):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.dist = None
        if self.world > 1:
            import datetime

            import torch.distributed as dist
            kw = {"device_id": torch.device("cuda", self.local)} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
            self.dist = dist

    def _sync_device(self):
        if self.backend == "nccl" and torch.cuda.is_available():
            torch.cuda.synchronize()

    def barrier(self):
        """Device synchronize, then a barrier over all ranks, then synchronize again."""
        self._sync_device()
        if self.dist is not None:
            self.dist.barrier()
        self._sync_device()

    def max(self, v: float) -> float:
        if self.dist is None:
            return v
        dev = "cuda" if self.backend == "nccl" else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def rate(self, units_per_rank: float, ms_this_rank: float) -> float:
        """Whole-job units/s: all ranks' units over the slowest rank's time."""
        return self.world * units_per_rank / (self.max(ms_this_rank) / 1e3)

    def close(self):
        if self.dist is not None:
            self.dist.barrier()
            self.dist.destroy_process_group()
            self.dist = None


def reduced(wl, args):
    """The workload with --experts / --tokens applied (profiling cases: a few GB instead of 20)."""
    import dataclasses
    kw = {}
    if args.experts:
        kw["n_experts"] = args.experts
    if args.tokens:
        kw["T"] = args.tokens
    if kw:
        kw["name"] = f"{wl.name}_E{args.experts or wl.n_experts}_T{args.tokens or wl.T}"
        kw["description"] = (f"profiling case: Beam shapes with {args.experts or wl.n_experts} experts, "
                             f"T={args.tokens or wl.T}")
        kw["bias"] = "zero"
        return dataclasses.replace(wl, **kw)
    return wl


def layer_inputs(wl):
    """x, W_r and bias of a workload: host copies and device tensors."""
    x_cpu = bs.make_x(wl)
    W_cpu = bs.make_router(wl)
    b_cpu = bs.load_bias(wl)
    return dict(x_cpu=x_cpu, W_cpu=W_cpu, b_cpu=b_cpu, x=x_cpu.cuda(), W=W_cpu.cuda(),
                bias=None if b_cpu is None else b_cpu.cuda())


def roofline_of(wl, fmt, stage_ms, n_act, ms_step, pk, pk_kind):
    """Layer roofline and the dominant kernel's roofline (HBM GB/s or tensor TFLOP/s, whichever
    bounds it at this workload) from the measured stage times."""
    alg = algorithmic(wl, n_act, fmt)
    # the expert products run on the tensor cores at their own dtype's rate (nominal ratio to bf16:
    # 2x for FP8, 4x for FP4 operands; the weight-only low-precision paths multiply in bf16); the router
    # projection is counted at the bf16 rate
    ratio = {"mxfp8": 2.0, "w4a4": 4.0}.get(fmt, 1.0)
    router_flops = alg["stage_flops"]["router"]
    t_tensor = (router_flops + (alg["layer_flops"] - router_flops) / ratio) / (pk["bf16_tflops"] * 1e12)
    t_hbm = alg["layer_bytes"] / (pk["hbm_gbs"] * 1e9)
    t_roof = max(t_tensor, t_hbm)
    layer = {"bound": "hbm" if t_hbm >= t_tensor else "tensor", "roofline_ms": t_roof * 1e3,
             "roofline_tokens_s": wl.T / t_roof, "frac": t_roof / (ms_step / 1e3),
             "tensor_ms": t_tensor * 1e3, "tensor_peak_ratio_to_bf16": ratio, "hbm_ms": t_hbm * 1e3,
             "active_experts": n_act,
             "achieved_tflops": alg["layer_flops"] / (ms_step / 1e3) / 1e12,
             "achieved_gbs": alg["layer_bytes"] / (ms_step / 1e3) / 1e9}
    dom = max(stage_ms, key=stage_ms.get)
    sec = stage_ms[dom] / 1e3
    by = alg["stage_bytes"][dom]
    fl = alg["stage_flops"].get(dom, 0.0)
    t_b = by / (pk["hbm_gbs"] * 1e9)
    t_f = fl / (pk["bf16_tflops"] * 1e12)
    if dom in ("gate_up_swiglu", "down") and t_f > t_b and fmt == "bf16":
        # a tensor-bound launch runs milliseconds inside a long step under the power cap: the sustained
        # peak is its denominator (the burst one is reported beside it)
        peak = pk["bf16_tflops_sustained"]
        roof = {"bound": "tensor", "kernel": dom, "achieved": fl / sec / 1e12, "peak": peak,
                "unit": "TFLOP/s", "frac": fl / sec / 1e12 / peak, "peak_kind": pk_kind + " sustained",
                "frac_of_burst_peak": fl / sec / 1e12 / pk["bf16_tflops"],
                "algorithmic_flops_per_launch": fl, "launch_ms": stage_ms[dom]}
    else:
        roof = {"bound": "hbm", "kernel": dom, "achieved": by / sec / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": by / sec / 1e9 / pk["hbm_gbs"], "peak_kind": pk_kind, "algorithmic_bytes_per_launch": by,
                "launch_ms": stage_ms[dom]}
    return layer, roof


def run_ours(args):
    import group_limited_routing_router_b200 as bm

    ranks = Ranks("nccl")
    world, rank, local = ranks.world, ranks.rank, ranks.local
    torch.cuda.set_device(local)
    barrier = ranks.barrier

    wl = reduced(bs.get(args.workload), args)
    layer = wl.layer
    T, H = wl.T, wl.hidden
    fmt = ("nvfp4" if args.nvfp4 else "fp8" if args.fp8 else "mxfp8" if args.mxfp8 else "w4a4" if args.w4a4
           else "bf16")
    if args.also is None:
        also = [] if args.block else (["decode", "skew", "long"] if fmt == "bf16" else ["decode"])
    else:
        also = [n for n in args.also.split(",") if n]
    if (args.experts or args.tokens) and args.also is None:
        also = []
    also = [n for n in also if n != wl.name]
    wg, wu, wd = bs.make_experts(wl, device="cuda")
    w8 = None
    if fmt != "bf16":
        if args.block:
            raise SystemExit("--fp8/--nvfp4 and --block: the sublayer entry point takes bf16 expert weights")
        w8 = bs.quantize_experts_nvfp4(wg, wu, wd) if fmt in ("nvfp4", "w4a4") else bs.quantize_experts(wg, wu, wd)
        del wg, wu, wd
        wg = wu = wd = None
        torch.cuda.empty_cache()
    T_max = max([T] + [bs.get(n).T for n in also])
    ws = torch.empty(bm.workspace_size(layer, T_max, bm.WS_FORWARD), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def make_step(inp, y, ids, w):
        x, W, bias = inp["x"], inp["W"], inp["bias"]
        if args.block:
            g_pre = torch.ones(H, dtype=torch.float32, device="cuda")
            g_post = torch.ones(H, dtype=torch.float32, device="cuda")
            ws_blk = torch.empty(bm.workspace_size(layer, x.shape[0], bm.WS_BLOCK), dtype=torch.uint8, device="cuda")
            block_step = 2 * 3 + 3  # the MoE sublayer of the first MoE layer (layer 3)
            return lambda: bm.block_forward(layer, x, g_pre, g_post, 1e-6, block_step, W, bias, wg, wu, wd,
                                            stream_out=y, ids=ids, w=w, ws=ws_blk)
        if fmt == "fp8":
            return lambda: bm.forward_fp8(layer, x, W, bias, w8, y=y, ids=ids, w=w, ws=ws)
        if fmt == "mxfp8":
            return lambda: bm.forward_mxfp8(layer, x, W, bias, w8, y=y, ids=ids, w=w, ws=ws)
        if fmt == "w4a4":
            return lambda: bm.forward_w4a4(layer, x, W, bias, w8, y=y, ids=ids, w=w, ws=ws)
        if fmt == "nvfp4":
            return lambda: bm.forward_nvfp4(layer, x, W, bias, w8, y=y, ids=ids, w=w, ws=ws)
        return lambda: bm.forward(layer, x, W, bias, wg, wu, wd, y=y, ids=ids, w=w, ws=ws)

    def profiled(inp, y, ids, w, ev):
        x, W, bias = inp["x"], inp["W"], inp["bias"]
        if fmt == "fp8":
            bm.forward_fp8(layer, x, W, bias, w8, y=y, ids=ids, w=w, ws=ws, events=ev)
        elif fmt == "mxfp8":
            bm.forward_mxfp8(layer, x, W, bias, w8, y=y, ids=ids, w=w, ws=ws, events=ev)
        elif fmt == "w4a4":
            bm.forward_w4a4(layer, x, W, bias, w8, y=y, ids=ids, w=w, ws=ws, events=ev)
        elif fmt == "nvfp4":
            bm.forward_nvfp4(layer, x, W, bias, w8, y=y, ids=ids, w=w, ws=ws, events=ev)
        else:
            bm.forward_profiled(layer, x, W, bias, wg, wu, wd, ev, y, ids, w, ws)

    clocks = ClockSampler(local)
    clocks.start()
    pk, pk_kind = peaks()

    def measure(wlx, steps, warmup, headline):
        """Device time of `steps` calls (max over ranks), stage times from profiled calls, routing stats."""
        inp = layer_inputs(wlx)
        y = torch.empty(wlx.T, H, dtype=torch.bfloat16, device="cuda")
        ids = torch.empty(wlx.T, wlx.topk, dtype=torch.int32, device="cuda")
        w = torch.empty(wlx.T, wlx.topk, dtype=torch.float32, device="cuda")
        step = make_step(inp, y, ids, w)
        for _ in range(warmup):
            step()
        assert bm.device_status() == bm.OK
        barrier()
        mark0 = clocks.n_samples()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(steps):
            step()
        ev1.record(stream)
        barrier()
        # keep the GPU busy (untimed) until the sampler has seen at least 3 samples under load
        t_extra = time.time()
        while clocks.n_samples() - mark0 < 3 and time.time() - t_extra < 2.0:
            for _ in range(10):
                step()
            torch.cuda.synchronize()
        span = (mark0, clocks.n_samples())
        ms_this = ev0.elapsed_time(ev1)
        ms_step = ranks.max(ms_this) / steps
        value = ranks.rate(wlx.T * steps, ms_this)
        counts = torch.bincount(ids.flatten().long(), minlength=wlx.n_experts)
        n_act = int((counts > 0).sum().item())
        # per-stage device time from events recorded between the launches (same stream)
        n_prof = min(steps, 20)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(n_prof)]
        for i in range(n_prof):
            profiled(inp, y, ids, w, evs[i])
        torch.cuda.synchronize()
        stage_ms = {name: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs)
                    for j, name in enumerate(bm.STAGES)}
        layer_roof, roof = roofline_of(wlx, fmt, stage_ms, n_act, ms_step, pk, pk_kind)
        out = dict(value=value, ms_per_step=ms_step, steps=steps, warmup=warmup, layer_roofline=layer_roof,
                   roofline=roof, stage_ms=stage_ms, clock_span=span,
                   load={"max_over_mean": float(counts.max().item() / counts.float().mean().item()),
                         "experts_with_no_token": int((counts == 0).sum().item())})
        if headline:
            out["inp"], out["step"], out["y"], out["ids"] = inp, step, y, ids
        return out

    head = measure(wl, args.steps, args.warmup, True)
    others = {}
    for n in also:
        wlx = bs.get(n)
        k_steps = max(3, min(args.steps, int(2000.0 / max(head["ms_per_step"] * wlx.T / T, 1e-3))))
        others[n] = measure(wlx, k_steps, max(3, min(args.warmup, 5)), False)

    # end to end through the public API with host buffers: every step copies its input from pinned host
    # memory and reads its output back.  The copies run on their own streams, double-buffered, so step
    # i + 1's upload and step i - 1's download overlap step i's forward pass (compute stays ordered on
    # one stream, so the shared workspace is safe); the timed region runs from before the first upload
    # to after the last download.
    inp, step, y, ids_gpu = head.pop("inp"), head.pop("step"), head.pop("y"), head.pop("ids")
    x_host = inp["x_cpu"].pin_memory()
    xs = [inp["x"], torch.empty_like(inp["x"])]
    ys = [y, torch.empty_like(y)]
    y_hosts = [torch.empty(T, H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    k_top = layer["topk"]
    steps_b = [make_step(dict(inp, x=xs[b]), ys[b],
                         torch.empty(T, k_top, dtype=torch.int32, device="cuda"),
                         torch.empty(T, k_top, dtype=torch.float32, device="cuda")) for b in range(2)]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        b = i & 1
        up.wait_event(ev_comp[b])  # step i - 2 has finished reading this input buffer
        with torch.cuda.stream(up):
            xs[b].copy_(x_host, non_blocking=True)
        ev_up[b].record(up)
        stream.wait_event(ev_up[b])
        stream.wait_event(ev_down[b])  # step i - 2's output has been read back
        steps_b[b]()
        ev_comp[b].record(stream)
        down.wait_event(ev_comp[b])
        with torch.cuda.stream(down):
            y_hosts[b].copy_(ys[b], non_blocking=True)
        ev_down[b].record(down)

    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_event(e0)
    for i in range(args.steps):
        e2e_step(i)
    stream.wait_event(ev_down[(args.steps - 1) & 1])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_value = ranks.rate(T * args.steps, e0.elapsed_time(e1))
    assert bm.device_status() == bm.OK
    clk_all = clocks.stop()
    clk = clocks.summary(*head.pop("clock_span"))
    for n in others:
        others[n]["clocks"] = clocks.summary(*others[n].pop("clock_span"))
    clocks.cleanup()

    roofline = head["roofline"]
    roofline["traffic"] = traffic_of(roofline["kernel"], fmt, wl.name)
    for n in others:
        others[n]["roofline"]["traffic"] = traffic_of(others[n]["roofline"]["kernel"], fmt, n)
    src_hash = kernel_source_hash()

    cpu = parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        fetch = {"bf16": lambda: bf16_fetch(wg, wu, wd), "fp8": lambda: fp8_fetch(w8), "mxfp8": lambda: fp8_fetch(w8),
                 "w4a4": lambda: nvfp4_fetch(w8),
                 "nvfp4": lambda: nvfp4_fetch(w8)}[fmt]()
        cpu = cpu_oracle_rate(wl, inp["x_cpu"], inp["W_cpu"], inp["b_cpu"], fetch, args.cpu_sample,
                              fmt=fmt)
        cpu.pop("seconds", None)
        parity = parity_of(y, ids_gpu, cpu.pop("tok"), cpu.pop("ids"), cpu.pop("y"))

    cfg = config_dict(wl)
    if fmt == "w4a4":
        cfg["weights"] = ("NVFP4 experts (E2M1 + E4M3 per 16 K + FP32 per matrix, 0.5625 B/weight) and NVFP4 "
                          "activations (x per token with a power-of-two scale, h per row) on tcgen05 "
                          "kind::mxf4nvf4; router FP32")
        cfg["weights_bytes"] = int(3 * wl.n_experts * wl.hidden * wl.inter * (0.5 + 1 / 16))
        cfg["l2"] = "no flush: every step streams the 5.7 GB of NVFP4 expert weights and scales (> 126 MB L2)"
    if fmt == "mxfp8":
        cfg["weights"] = ("MXFP8 experts: E4M3 codes + UE8M0 scale per 32 K elements (1.03 B/weight) and MXFP8 "
                          "activations (x, h per row, blocks of 32) on tcgen05 kind::mxf8f6f4; router FP32")
        cfg["weights_bytes"] = int(3 * wl.n_experts * wl.hidden * wl.inter * (1 + 1 / 32))
        cfg["l2"] = "no flush: every step streams the 10.4 GB of FP8 expert weights and scales (> 126 MB L2)"
    if fmt == "fp8":
        cfg["weights"] = ("MXFP8 experts: E4M3 codes + UE8M0 scale per 32 K elements (1.03 B/weight), rebuilt "
                          "as bf16 in a TMEM ring; router FP32")
        cfg["weights_bytes"] = int(3 * wl.n_experts * wl.hidden * wl.inter * (1 + 1 / 32))
        cfg["l2"] = "no flush: every step streams the 10.4 GB of FP8 expert weights and scales (> 126 MB L2)"
    elif fmt == "nvfp4":
        cfg["weights"] = ("NVFP4 experts: E2M1 code pairs + E4M3 scale per 16 K elements + FP32 per-matrix scale "
                          "(0.5625 B/weight), rebuilt as bf16 in a TMEM ring; router FP32")
        cfg["weights_bytes"] = int(3 * wl.n_experts * wl.hidden * wl.inter * (0.5 + 1 / 16))
        cfg["l2"] = "no flush: every step streams the 5.7 GB of NVFP4 expert weights and scales (> 126 MB L2)"
    metric = {"bf16": METRIC, "fp8": METRIC_FP8, "mxfp8": METRIC_MXFP8, "nvfp4": METRIC_NVFP4, "w4a4": METRIC_W4A4}[fmt]
    dtype = {"bf16": "bf16", "fp8": "fp8-e4m3 weights, bf16 MMA", "mxfp8": "fp8-e4m3 weights and activations",
             "nvfp4": "nvfp4-e2m1 weights, bf16 MMA", "w4a4": "nvfp4-e2m1 weights and activations"}[fmt]
    n_launch = launches_per_step(wl, args.block, fmt)
    line = {"metric": metric, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": dtype,
            "data": "synthetic", "config": cfg,
            "roofline": roofline, "layer_roofline": head["layer_roofline"], "stage_ms": head["stage_ms"],
            "load": head["load"], "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": T * H * 2,
                    "d2h_bytes_per_step": T * H * 2},
            "clocks": clk, "clocks_whole_run": clk_all,
            "gpu_launches": n_launch * args.steps, "kernel_source": src_hash}
    if parity is not None:
        line["parity"] = parity
    if others:
        line["workloads"] = {n: {"T": bs.get(n).T, "tokens_s": o["value"], "ms_per_step": o["ms_per_step"],
                                 "steps": o["steps"], "warmup": o["warmup"], "layer_roofline": o["layer_roofline"],
                                 "roofline": o["roofline"], "stage_ms": o["stage_ms"], "load": o["load"],
                                 "clocks": o["clocks"], "workload": config_dict(bs.get(n))["workload"]}
                             for n, o in others.items()}
    if args.block:
        line["config"]["block"] = ("sublayer step: RMSNorm pre-norm + MoE block + fused post-norm and scaled residual "
                                   "(step k=9); stage_ms/roofline are from the plain block's profiled launches")
    if rank == 0:
        print(json.dumps(line))
    ranks.close()


def run_dense(args):
    """Dense SwiGLU MLP line: tokens/s and the tensor-core roofline of the whole call."""
    import group_limited_routing_router_b200 as bm
    ranks = Ranks("nccl")
    torch.cuda.set_device(ranks.local)
    wl = bs.DENSE["dense_prefill"]
    T, H, I = wl.T, wl.hidden, wl.inter
    x = bs.make_x(wl).cuda()
    wg, wu, wd = (t[0].contiguous() for t in bs.make_experts(wl, device="cuda"))
    y = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(bm.dense_workspace_size(H, I, T), dtype=torch.uint8, device="cuda")
    clocks = ClockSampler(ranks.local)
    clocks.start()
    for _ in range(args.warmup):
        bm.dense_swiglu(x, wg, wu, wd, y=y, ws=ws)
    ranks.barrier()
    clocks.mark()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        bm.dense_swiglu(x, wg, wu, wd, y=y, ws=ws)
    e1.record()
    ranks.barrier()
    clocks.mark()
    clocks.stop()
    clk = clocks.summary(clocks.marks[0], clocks.marks[-1])
    clocks.cleanup()
    assert bm.device_status() == bm.OK
    ms = ranks.max(e0.elapsed_time(e1)) / args.steps
    flops = 6.0 * T * H * I
    pk, kind = peaks()
    achieved = flops / (ms / 1e3) / 1e12
    line = {"metric": "dense SwiGLU MLP tokens/s (Beam first layers, T=4096, intermediate 20480)",
            "value": ranks.world * T / (ms / 1e3), "unit": "tokens/s", "n_gpus": ranks.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"dense_prefill: {wl.description}", "T": T, "hidden": H, "inter": I},
            "roofline": {"bound": "tensor", "kernel": "dense call (gate/up + down GEMMs)",
                         "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / pk["bf16_tflops"], "traffic": None, "peak_kind": kind},
            "clocks": clk, "gpu_launches": 3 * args.steps}
    if ranks.rank == 0:
        print(json.dumps(line))
    ranks.close()


def run_ep(args):
    """Expert-parallel line: N ranks, each with E/N experts and its own batch; tokens/s of all ranks
    over the slowest rank's device time.  One rank runs the same code with a trivial exchange."""
    import group_limited_routing_router_b200 as bm
    from group_limited_routing_router_b200 import ep

    ranks = Ranks("nccl")
    torch.cuda.set_device(ranks.local)
    wl = bs.get(args.workload)
    part = ep.Partition(wl.n_experts, ranks.world)
    own = part.experts_of(ranks.rank)
    full = bs.make_experts(wl, device="cuda")  # drawn per expert from its own sub-seed: keep this rank's slice
    wg, wu, wd = (t[own.start:own.stop].contiguous() for t in full)
    del full
    torch.cuda.empty_cache()
    import dataclasses
    inp = layer_inputs(dataclasses.replace(wl, seed=wl.seed + 7919 * ranks.rank))
    rank = ep.Rank(part, ranks.rank, ep.GpuOps(wl.layer, inp["W"], inp["bias"], wg, wu, wd))
    group = ranks.dist.group.WORLD if ranks.dist is not None else None

    def step():
        if ranks.dist is None:
            return ep.forward_emulated([rank], [inp["x"]])[0]
        return ep.forward(rank, inp["x"], group)

    for _ in range(args.warmup):
        step()
    assert bm.device_status() == bm.OK
    ranks.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    ranks.barrier()
    ms = e0.elapsed_time(e1)
    value = ranks.rate(wl.T * args.steps, ms)
    line = {"metric": METRIC + " [expert parallel]", "value": value, "unit": "tokens/s", "n_gpus": ranks.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ranks.max(ms) / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**config_dict(wl), "parallelism": f"expert parallel: {part.per_rank} experts per rank",
                       "note": "host-synchronising exchange (split sizes read back); every rank its own batch"}}
    if ranks.rank == 0:
        print(json.dumps(line))
    ranks.close()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.ep:
        run_ep(args)
    elif args.dense:
        run_dense(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
