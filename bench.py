#!/usr/bin/env python3
"""Benchmark: batch-1 MoE decode through the A3B-shaped stack.

Workload: 40 MoE layers, hidden 2048, 256 routed SwiGLU experts (top-8,
intermediate 512) plus one shared expert (intermediate 512), bf16 weights
N(0, 0.02) drawn per layer (64.7 GB resident), router scaled for near-uniform
routing, 256 decode tokens x ~ N(0, 1). One step = one token through all 40
layers = one persistent kernel launch (router, top-k, routed + shared experts,
weighted sum, residual for every layer).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). With N > 1 (torchrun) every rank runs its own
replica of the stack on its own token stream (replicas only: the decode path
has no exchange step), timed on the device, max over ranks.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE decode layer tok/s at B=1; achieved HBM GB/s vs peak on routed bytes"
WORKLOAD = "a3b_bf16"
NOMINAL_HBM_GBS = 8000.0  # the ~8 TB/s nominal B200 figure quoted for this metric
FALLBACK_HBM_GBS = 6650.0


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------- distributed plumbing


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(ws, backend):
    import torch.distributed as dist
    if ws > 1 and not dist.is_initialized():
        from datetime import timedelta
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=300))
    return dist


def max_over_ranks(value: float, ws: int, device) -> float:
    """Max of a per-rank float over all ranks (identity when ws == 1)."""
    if ws <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while active."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.idx)], stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or self.path is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- workloads
#
# Each workload sets up its synthetic inputs on the device and provides:
#   step(i)      one step on device-resident inputs (the timed unit)
#   e2e_step(i)  the same through host (pinned) buffers: input H2D, output D2H
#   nbytes(i)    algorithmic bytes the step must read (router, routed experts
#                or kept channels, shared expert; exact routing of that step)
# plus tokens per step, launches per step and a config description.


def a3b_config(name, w, B, layers=None):
    return {"workload": name + ("" if B == 1 else f"_b{B}"), "layers": layers or w["layers"], "hidden": w["H"],
            "experts": w["E"], "top_k": w["k"], "expert_intermediate": w["I"], "shared_intermediate": w["I_shared"],
            "batch": B, "pre_norm": "rms", "l2": "inputs larger than L2 (weights of 40 layers, tens of GB)"}


class A3BStack:
    """40-layer A3B-shaped SwiGLU stack (bf16 or int4 experts), batch B, pre-norm."""

    def __init__(self, torch, M, S, device, rank, wtype="bf16", B=1, steps=0, layers=0):
        self.torch, self.M, self.S, self.dev = torch, M, S, device
        self.name = "a3b_bf16" if wtype == "bf16" else "a3b_int4"
        w = S.WORKLOADS[self.name]
        self.w = w
        H, E, I, k, I_sh, nl = w["H"], w["E"], w["I"], w["k"], w["I_shared"], layers or w["layers"]
        self.H, self.E, self.I, self.k, self.I_sh, self.nl, self.B = H, E, I, k, I_sh, nl, B
        gen = S.swiglu_layer_bf16 if wtype == "bf16" else S.swiglu_layer_int4
        self.layers = [gen(H, E, I, I_sh, seed=S.weight_seed(w["cfg"], l), device=device,
                           router_scale=w["router_scale"]) for l in range(nl)]
        kw = {} if wtype == "bf16" else {"wtype": M.MOE_W_INT4_G64}
        self.descs = []
        for L in self.layers:
            extra = {} if wtype == "bf16" else {"gate_s": L["gate_s"], "up_s": L["up_s"], "down_s": L["down_s"]}
            self.descs.append(M.make_desc(H, E, I, k, router=L["router"], gate=L["gate"], up=L["up"],
                                          down_t=L["down_t"], sh_gate=L["sh_gate"], sh_up=L["sh_up"],
                                          sh_down_t=L["sh_down_t"], **kw, **extra))
        self.ntok = 256
        self.xs = S.tokens(self.ntok * B, H, seed=S.act_seed(w["cfg"]) + 97 * rank, device=device)
        self.ws = M.alloc_workspace(self.descs[0], B, device)
        self.x_out = torch.empty((B, H), dtype=torch.bfloat16, device=device)
        self.ids_hist = torch.zeros((max(steps, 1), nl, B, k), dtype=torch.int32, device=device)
        self.w_hist = torch.zeros((max(steps, 1), nl, B, k), dtype=torch.float32, device=device)
        self.expert_bytes = 3 * I * H * 2 if wtype == "bf16" else 3 * I * H // 2 + 3 * I * (H // 64) * 2
        self.tokens_per_step = B
        self.launches_per_step = 1
        self.kernel = f"decode_kernel<layers,B{B},{wtype},planar>"
        self.sources = DECODE_KERNEL_SOURCES
        self.dtype = "bf16" if wtype == "bf16" else "int4"
        self.wtype = wtype
        self.record = 0

    def _x(self, i):
        j = i % self.ntok
        return self.xs[j * self.B:(j + 1) * self.B]

    def step(self, i, stream):
        r = self.record
        kw = {"ids_hist": self.ids_hist[r], "w_hist": self.w_hist[r]} if r < self.ids_hist.shape[0] else {}
        self.M.moe_stack_forward(self.descs, self._x(i), self.x_out, self.ws, flags=self.M.MOE_STACK_PRE_RMSNORM,
                                 stream=stream, **kw)

    def host_buffers(self):
        t = self.torch
        self.x_host = self.xs.cpu().pin_memory()
        self.out_host = t.empty((self.B, self.H), dtype=t.bfloat16).pin_memory()
        self.x_dev = t.empty((self.B, self.H), dtype=t.bfloat16, device=self.dev)
        return self.B * self.H * 2, self.B * self.H * 2

    def e2e_step(self, i, stream):
        j = i % self.ntok
        self.x_dev.copy_(self.x_host[j * self.B:(j + 1) * self.B], non_blocking=True)
        self.M.moe_stack_forward(self.descs, self.x_dev, self.x_out, self.ws, flags=self.M.MOE_STACK_PRE_RMSNORM,
                                 stream=stream)
        self.out_host.copy_(self.x_out, non_blocking=True)

    def nbytes(self, r):
        """Bytes of timed step r: per layer router + touched experts + shared."""
        ids = self.ids_hist[r].cpu()
        total = 0
        for l in range(self.nl):
            touched = len(set(ids[l].reshape(-1).tolist()))
            total += 2 * self.E * self.H + touched * self.expert_bytes + 3 * self.I_sh * self.H * 2
        return total

    def config(self):
        return a3b_config(self.name, self.w, self.B, self.nl)

    def oracle_sample(self, budget_s):
        """The fp64 oracle on whole layers of this stack (batch 1 token by token)."""
        tps, done, dt = oracle_rate(self.layers, self.w, self.xs, budget_s=budget_s, wtype=self.wtype)
        return {"value": tps, "unit": "tok/s", "cores": blas_threads(), "kind": "oracle",
                "sample": f"{done} layer passes of one token in {dt:.1f} s, scaled to tokens through "
                          f"{self.nl} layers (fp64; the router, shared and routed experts' slices copied "
                          "from the device; RMS pre-norm as on the device)"}


class ChannelStack:
    """48-layer channel-major stack, batch 1, channel top-k keep over given
    scores, or (screen=True) over scores the kernel computes per layer from
    the weight-only sketch of each layer (the screen inside the stack)."""

    def __init__(self, torch, M, S, device, rank, frac=0.13, steps=0, layers=0, screen=False):
        self.torch, self.M, self.S, self.dev = torch, M, S, device
        w = S.WORKLOADS["channel_topk"]
        H, E, I, k, nl = w["H"], w["E"], w["I"], w["k"], layers or w["layers"]
        self.H, self.E, self.I, self.k, self.nl = H, E, I, k, nl
        self.keep = S.keep_count(frac, k, I)
        self.frac = frac
        self.layers = [S.channel_major_layer(H, E, I, seed=S.weight_seed(5, l), device=device) for l in range(nl)]
        self.descs = [M.make_desc(H, E, I, k, layout=M.MOE_LAYOUT_CHANNEL_MAJOR, router=L["router"], gate=L["cm"])
                      for L in self.layers]
        scale = [S.channel_scale(E, I, seed=S.weight_seed(5, l) + 7, device=device) for l in range(nl)]
        self.nsc = 16  # distinct per-token score sets
        self.scores = torch.stack([torch.cat([S.channel_scores(1, E, I, scale[l], seed=S.act_seed(5, l) + 1000 * t,
                                                               device=device) for l in range(nl)])
                                   for t in range(self.nsc)])
        self.xs = S.tokens(256, H, seed=S.act_seed(5) + 97 * rank, device=device)
        self.ws = M.alloc_workspace(self.descs[0], 1, device)
        self.x_out = torch.empty((1, H), dtype=torch.bfloat16, device=device)
        self.sectors = torch.empty((nl,), dtype=torch.int64, device=device)
        self.tokens_per_step = 1
        self.launches_per_step = 1
        self.kernel = "decode_kernel<layers,B1,bf16,channel-major>" + (" + in-kernel screen" if screen else "")
        self.sources = DECODE_KERNEL_SOURCES
        self.dtype = "bf16"
        self.screen = screen
        self.sketches = None
        if screen:
            self.signs = S.reader_signs(H, seed=S.weight_seed(5, 0) + 11, device=device)
            shp = M.reader_sketch_shapes(self.descs[0])
            self.sk_bufs = []
            for d in self.descs:
                codes = torch.empty(shp["codes"], dtype=torch.int32, device=device)
                scales = torch.empty(shp["scales"], dtype=torch.int16, device=device)
                rho = torch.empty(shp["rho"], dtype=torch.float32, device=device)
                dnorm = torch.empty(shp["dnorm"], dtype=torch.float32, device=device)
                M.moe_reader_build(d, self.signs, codes, scales, rho, dnorm)
                self.sk_bufs.append((codes, scales, dnorm))
                del rho
            self.sketches = [M.make_sketch(c, sc, dn) for (c, sc, dn) in self.sk_bufs]
            torch.cuda.synchronize()

    def _scores(self, i):
        return None if self.screen else self.scores[i % self.nsc]

    def step(self, i, stream):
        self.M.moe_channel_stack_forward(self.descs, self.xs[i % 256:][:1], self._scores(i), self.keep,
                                         self.x_out, self.sectors, self.ws, flags=self.M.MOE_STACK_PRE_RMSNORM,
                                         sketches=self.sketches, signs=self.signs if self.screen else None,
                                         stream=stream)

    def host_buffers(self):
        t = self.torch
        self.x_host = self.xs.cpu().pin_memory()
        self.out_host = t.empty((1, self.H), dtype=t.bfloat16).pin_memory()
        self.x_dev = t.empty((1, self.H), dtype=t.bfloat16, device=self.dev)
        return self.H * 2, self.H * 2

    def e2e_step(self, i, stream):
        self.x_dev.copy_(self.x_host[i % 256:][:1], non_blocking=True)
        self.M.moe_channel_stack_forward(self.descs, self.x_dev, self._scores(i), self.keep, self.x_out,
                                         self.sectors, self.ws, flags=self.M.MOE_STACK_PRE_RMSNORM,
                                         sketches=self.sketches, signs=self.signs if self.screen else None,
                                         stream=stream)
        self.out_host.copy_(self.x_out, non_blocking=True)

    def nbytes(self, r):
        # router + kept channels (gate row, up row, down column) + the 8 score rows read;
        # screened: + the routed experts' codes, scales and down-column norms
        b = 2 * self.E * self.H + self.keep * 3 * self.H * 2 + self.k * self.I * 4
        if self.screen:
            b += self.k * self.I * (2 * (self.H // 4 + 2 * (self.H // 128)) + 4)
        return self.nl * b

    def oracle_sample(self, budget_s):
        """The fp64 oracle's channel-stack layer, token 0 through the layers in order."""
        from oracle import moe_oracle as O

        def f64(t):
            return t.detach().cpu().float().double().numpy()
        t0 = time.perf_counter()
        x = f64(self.xs[0])
        done = 0
        sg = f64(self.signs) if self.screen else None
        while True:
            l = done % self.nl
            cm = self.layers[l]["cm"]
            R = f64(self.layers[l]["router"])
            if self.screen:
                # the screen from the oracle's own sketch of the routed experts' channels
                u = O.rmsnorm_bf16(x)
                ids, w, _, _ = O.route_topk(u, R, self.k)

                def sketch(e, c, cm=cm):
                    g, v, d = f64(cm[e, c])
                    cg, scg, _ = O.reader_sketch_row(g, sg)
                    cv, scv, _ = O.reader_sketch_row(v, sg)
                    return cg, scg, cv, scv, float(np.sqrt(np.sum(d ** 2)))
                o_sc, _ = O.reader_screen(u, ids.tolist(), w, sketch, self.I, sg)
                sc = np.full((self.E, self.I), -np.inf)
                for t, e in enumerate(ids.tolist()):
                    sc[e] = o_sc[t]
            else:
                sc = f64(self.scores[0, l])
            x, *_ = O.channel_stack_layer(x, R, lambda e, c, cm=cm: f64(cm[e, c]), sc, self.k, self.keep, self.I)
            done += 1
            if time.perf_counter() - t0 >= budget_s:
                break
        dt = time.perf_counter() - t0
        return {"value": (done / self.nl) / dt, "unit": "tok/s", "cores": blas_threads(), "kind": "oracle",
                "sample": f"{done} channel-sparse layer passes of one token in {dt:.1f} s, scaled to tokens "
                          f"through {self.nl} layers (fp64; kept channels copied from the device"
                          + ("; scores from the oracle's own screen)" if self.screen else ")")}

    def config(self):
        return {"workload": f"channel_topk_{int(round(100 * self.frac))}pct" + ("_screened" if self.screen else ""),
                "scores": "computed in the kernel from per-layer sketches" if self.screen else "input",
                "layers": self.nl, "hidden": self.H,
                "experts": self.E, "top_k": self.k, "channels": self.I, "keep": self.keep, "batch": 1,
                "pre_norm": "rms", "l2": "inputs larger than L2 (58 GB of channel-major weights)"}


class BatchSweep:
    """64 experts of one 8192 x 8192 bf16 matrix, top-3 uniform ids, batch B."""

    def __init__(self, torch, M, S, device, rank, B=256, steps=0, experts=0):
        self.torch, self.M, self.S, self.dev = torch, M, S, device
        w = S.WORKLOADS["batch_sweep"]
        H, E, k = w["H"], experts or w["E"], w["k"]
        self.H, self.E, self.k, self.B = H, E, k, B
        self.W = S.linear_experts(E, H, seed=S.weight_seed(3, 0), device=device)
        self.desc = M.make_desc(H, E, H, k, kind=M.MOE_EXPERT_LINEAR, gate=self.W)
        self.nsets = 16
        self.xs = [S.tokens(B, H, seed=S.act_seed(3) + 31 * t + 97 * rank, device=device) for t in range(self.nsets)]
        self.ids = [S.uniform_ids(B, E, k, seed=S.act_seed(3) + 1000 + 31 * t + 97 * rank, device=device)
                    for t in range(self.nsets)]
        self.wts = torch.ones((B, k), device=device)
        self.ws = M.alloc_workspace(self.desc, B, device)
        self.y = torch.empty((B, H), dtype=torch.float32, device=device)
        self.touched = [len(set(i.reshape(-1).tolist())) for i in self.ids]
        self.tokens_per_step = B
        self.launches_per_step = 4  # plan, gather, GEMV engine, tensor-core engine (+ a memset)
        self.kernel = "linear plan+gather+gemv+tcgen05"
        self.sources = LINEAR_KERNEL_SOURCES
        self.dtype = "bf16"
        self.record = 0

    def step(self, i, stream):
        t = i % self.nsets
        self.M.moe_expert_forward(self.desc, self.xs[t], self.ids[t], self.wts, self.y, self.ws, stream=stream)

    def host_buffers(self):
        t = self.torch
        self.x_host = [x.cpu().pin_memory() for x in self.xs]
        self.id_host = [i.cpu().pin_memory() for i in self.ids]
        self.y_host = t.empty((self.B, self.H), dtype=t.float32).pin_memory()
        self.x_dev = t.empty((self.B, self.H), dtype=t.bfloat16, device=self.dev)
        self.id_dev = t.empty((self.B, self.k), dtype=t.int32, device=self.dev)
        return self.B * self.H * 2 + self.B * self.k * 4, self.B * self.H * 4

    def e2e_step(self, i, stream):
        t = i % self.nsets
        self.x_dev.copy_(self.x_host[t], non_blocking=True)
        self.id_dev.copy_(self.id_host[t], non_blocking=True)
        self.M.moe_expert_forward(self.desc, self.x_dev, self.id_dev, self.wts, self.y, self.ws, stream=stream)
        self.y_host.copy_(self.y, non_blocking=True)

    def nbytes(self, r):
        return self.touched[r % self.nsets] * self.H * self.H * 2

    def touched_record(self):
        """Touched experts of the step inputs against E[1 - (1 - k/E)^B]."""
        return {"mean_touched": statistics.mean(self.touched), "expected": self.E * (1 - (1 - self.k / self.E) ** self.B),
                "input_sets": self.nsets}

    def oracle_sample(self, budget_s):
        """The fp64 oracle on whole tokens of step 0 (each token through its k experts)."""
        from oracle import moe_oracle as O
        t0 = time.perf_counter()
        x = self.xs[0].detach().cpu().float().double().numpy()
        ids = self.ids[0].cpu().numpy()
        done = 0
        while True:
            b = done % self.B
            O.linear_experts(x[b], lambda e: self.W[e].detach().cpu().float().double().numpy(),
                             ids[b].tolist(), [1.0] * self.k)
            done += 1
            if time.perf_counter() - t0 >= budget_s:
                break
        dt = time.perf_counter() - t0
        return {"value": done / dt, "unit": "tok/s", "cores": blas_threads(), "kind": "oracle",
                "sample": f"{done} tokens of one batch in {dt:.1f} s, each through its {self.k} experts of "
                          f"{self.H} x {self.H} (fp64; expert matrices copied from the device)"}

    def config(self):
        return {"workload": f"batch_sweep_b{self.B}", "experts": self.E, "top_k": self.k, "hidden": self.H,
                "batch": self.B, "expected_touched": self.E * (1 - (1 - self.k / self.E) ** self.B),
                "l2": "inputs larger than L2 (8.6 GB of expert matrices)"}


class ChannelBatch:
    """Channel-sparse layers of the 48-layer channel-major stack at batch B
    (4 or 8): per layer, B tokens with their own routed experts (k distinct
    uniform ids) and scores select their kept channels, and the batch reads
    the union of the kept channels once (one launch per layer). The bytes of
    a step are the union's 32-byte sectors the kernel reports, plus the
    score rows; they are compared with reading the touched experts whole
    (the full-read column of the pages' Table 7)."""

    def __init__(self, torch, M, S, device, rank, B=4, frac=0.13, steps=0, layers=0):
        self.torch, self.M, self.S, self.dev = torch, M, S, device
        w = S.WORKLOADS["channel_topk"]
        H, E, I, k, nl = w["H"], w["E"], w["I"], w["k"], layers or w["layers"]
        self.H, self.E, self.I, self.k, self.nl, self.B, self.frac = H, E, I, k, nl, B, frac
        self.keep = S.keep_count(frac, k, I)
        self.layers = [S.channel_major_layer(H, E, I, seed=S.weight_seed(5, l), device=device) for l in range(nl)]
        self.descs = [M.make_desc(H, E, I, k, layout=M.MOE_LAYOUT_CHANNEL_MAJOR, router=L["router"], gate=L["cm"])
                      for L in self.layers]
        self.nsets = 4
        scale = [S.channel_scale(E, I, seed=S.weight_seed(5, l) + 7, device=device) for l in range(nl)]
        self.scores = [[S.channel_scores(B, E, I, scale[l], seed=S.act_seed(5, l) + 1000 * t + 97 * rank,
                                         device=device) for l in range(nl)] for t in range(self.nsets)]
        self.ids = [[S.uniform_ids(B, E, k, seed=S.act_seed(5, l) + 2000 + 1000 * t + 97 * rank, device=device)
                     for l in range(nl)] for t in range(self.nsets)]
        self.wts = [torch.softmax(torch.randn((B, k), device=device), dim=1) for _ in range(nl)]
        self.xs = [S.tokens(B, H, seed=S.act_seed(5) + 31 * t + 97 * rank, device=device) for t in range(self.nsets)]
        self.ws = M.alloc_workspace(self.descs[0], B, device)
        self.y = torch.empty((B, H), dtype=torch.float32, device=device)
        self.sec = torch.empty((B,), dtype=torch.int64, device=device)
        self.ucount = torch.zeros((max(steps, 1), nl), dtype=torch.int32, device=device)
        self.usec = torch.zeros((max(steps, 1), nl), dtype=torch.int64, device=device)
        self.tokens_per_step = B
        self.launches_per_step = nl
        self.kernel = f"channel_batch_kernel<B{B}> x {nl} layers"
        self.sources = DECODE_KERNEL_SOURCES + ("channel_batch.cuh",)
        self.dtype = "bf16"
        self.record = 0

    def step(self, i, stream):
        t = i % self.nsets
        r = self.record
        for l in range(self.nl):
            kw = {"union_count": self.ucount[r, l:l + 1], "union_sectors": self.usec[r, l:l + 1]} \
                if r < self.ucount.shape[0] else {}
            self.M.moe_channel_topk_forward(self.descs[l], self.xs[t], self.ids[t][l], self.wts[l], self.scores[t][l],
                                            self.keep, self.y, self.sec, self.ws, stream=stream, **kw)

    def host_buffers(self):
        return 0, 0

    def e2e_step(self, i, stream):
        self.step(i, stream)

    def nbytes(self, r):
        """Union sectors x 32 (what the batch read) + the B x k score rows read."""
        return int(self.usec[r].sum().item()) * 32 + self.nl * self.B * self.k * self.I * 4

    def touched_record(self):
        """Bytes per layer of the union read against reading the touched
        experts whole (the pages' Table 7 full-read column)."""
        import statistics as st
        u = self.ucount[: min(self.ucount.shape[0], 1 << 30)].float()
        touched = [len(set(self.ids[t][l].reshape(-1).tolist())) for t in range(self.nsets) for l in range(self.nl)]
        full_mb = st.mean(touched) * self.I * 3 * self.H * 2 / 1e6
        union_mb = float(u[u > 0].mean().item()) * 3 * self.H * 2 / 1e6 if bool((u > 0).any()) else 0.0
        return {"union_channels_per_layer": float(u[u > 0].mean().item()) if bool((u > 0).any()) else 0.0,
                "kept_per_token": self.keep, "union_mb_per_layer": union_mb, "full_read_mb_per_layer": full_mb,
                "union_share_of_full": union_mb / full_mb if full_mb else None,
                "table7_reference_share": {"B4": 49.9 / 229.1, "B8": 92.3 / 359.3}}

    def oracle_sample(self, budget_s):
        from oracle import moe_oracle as O

        def f64(t):
            return t.detach().cpu().float().double().numpy()
        t0 = time.perf_counter()
        done = 0
        while True:
            l = done % self.nl
            cm = self.layers[l]["cm"]
            for b in range(self.B):
                ids = self.ids[0][l][b].tolist()
                kept = O.channel_topk_select(f64(self.scores[0][l][b]), ids, self.keep)
                O.channel_sparse_forward(f64(self.xs[0][b]), lambda e, c: f64(cm[e, c]), ids, f64(self.wts[l][b]),
                                         kept, self.I)
            done += 1
            if time.perf_counter() - t0 >= budget_s:
                break
        dt = time.perf_counter() - t0
        return {"value": done * self.B / self.nl / dt, "unit": "tok/s", "cores": blas_threads(), "kind": "oracle",
                "sample": f"{done} layers of a batch of {self.B} in {dt:.1f} s, scaled to tokens through "
                          f"{self.nl} layers (fp64; kept channels copied from the device)"}

    def config(self):
        return {"workload": f"channel_topk_{int(round(100 * self.frac))}pct_b{self.B}", "layers": self.nl,
                "hidden": self.H, "experts": self.E, "top_k": self.k, "channels": self.I, "keep": self.keep,
                "batch": self.B, "routing": "k distinct uniform ids per token and layer",
                "l2": "inputs larger than L2 (58 GB of channel-major weights)"}


def make_workload(name, torch, M, S, device, rank, args):
    if name == "a3b_bf16":
        return A3BStack(torch, M, S, device, rank, "bf16", args.batch or 1, steps=args.steps, layers=args.layers)
    if name == "a3b_int4":
        return A3BStack(torch, M, S, device, rank, "int4", args.batch or 1, steps=args.steps, layers=args.layers)
    if name == "channel_topk":
        return ChannelStack(torch, M, S, device, rank, args.keep_frac, steps=args.steps, layers=args.layers,
                            screen=getattr(args, "screen", False))
    if name == "batch_sweep":
        return BatchSweep(torch, M, S, device, rank, args.batch or 256, steps=args.steps, experts=args.experts)
    if name == "channel_batch":
        return ChannelBatch(torch, M, S, device, rank, args.batch or 4, args.keep_frac, steps=args.steps,
                            layers=args.layers)
    raise SystemExit(f"unknown workload {name}")


# ---------------------------------------------------------------- CPU oracle timing


def oracle_rate(layers, w, xs, budget_s=12.0, max_layers=None, start_token=0, wtype="bf16"):
    """Time the fp64 oracle (as it stands) layer by layer on whole tokens.

    Token t goes through layers 0..L-1 (RMS pre-norm, MoE, residual: the same
    stack the device runs); per layer the oracle copies the router, the shared expert and only the routed experts'
    weights to the host, converts them to fp64 and computes. Stops after the
    budget (at least one layer). Returns (tok/s, layers done, seconds)."""
    from oracle import moe_oracle as O

    def f64(t):
        return t.detach().cpu().float().double().numpy()

    k, nl = w["k"], len(layers)
    t0 = time.perf_counter()
    done = 0
    tok = start_token
    x = f64(xs[tok % xs.shape[0]])
    while True:
        Ld = layers[done % nl]
        R = f64(Ld["router"])
        shared = (f64(Ld["sh_gate"]), f64(Ld["sh_up"]), f64(Ld["sh_down_t"]))
        if wtype == "bf16":
            experts = lambda e, Ld=Ld: (f64(Ld["gate"][e]), f64(Ld["up"][e]), f64(Ld["down_t"][e]))
        else:
            experts = lambda e, Ld=Ld: (
                O.dequant_rows_int4(Ld["gate"][e].cpu().numpy(), f64(Ld["gate_s"][e])),
                O.dequant_rows_int4(Ld["up"][e].cpu().numpy(), f64(Ld["up_s"][e])),
                O.dequant_down_t_int4(Ld["down_t"][e].cpu().numpy(), f64(Ld["down_s"][e])))
        x, *_ = O.stack_layer(x, R, experts, k, shared=shared, pre_norm=True)
        done += 1
        if done % nl == 0:
            tok += 1
            x = f64(xs[tok % xs.shape[0]])
        if time.perf_counter() - t0 >= budget_s or (max_layers and done >= max_layers):
            break
    dt = time.perf_counter() - t0
    return (done / nl) / dt, done, dt


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=1)
    except Exception:
        return os.cpu_count() or 1


# ---------------------------------------------------------------- arms


def run_reference(args):
    """The oracle arm: the fp64 CPU oracle timed on this host's cores.

    One step of this arm is one token through one layer of the stack (a
    bounded sample: 1/40 of a token), so that K steps take seconds rather
    than the tens of minutes 40-layer tokens would; ms_per_step is the time
    of one such step and steps x ms_per_step is the time actually spent.
    The value is scaled to the metric's unit: tok/s = 1 / (layers x step time).
    """
    ws_n, rank, local = dist_env()
    if rank != 0:
        return 0
    if args.workload != WORKLOAD or (args.batch or 1) != 1:
        print(json.dumps({"impl": "reference", "unavailable": "the oracle arm is timed on the default workload "
                          f"({WORKLOAD}, batch 1) only"}), flush=True)
        return 0
    import torch
    from oracle import moe_oracle as O
    from mixture_experts_decode_moe_b200 import synth as S
    w = S.WORKLOADS[WORKLOAD]
    H, E, I, k, I_sh, nl = w["H"], w["E"], w["I"], w["k"], w["I_shared"], w["layers"]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    # one CPU copy of the stack would be 64 GB: keep it on the device when
    # there is one and let the oracle fetch the slices it reads
    layers = [S.swiglu_layer_bf16(H, E, I, I_sh, seed=S.weight_seed(w["cfg"], l), device=dev,
                                  router_scale=w["router_scale"]) for l in range(nl)]
    xs = S.tokens(w["tokens"], H, seed=S.act_seed(w["cfg"]), device=dev)

    def f64(t):
        return t.detach().cpu().float().double().numpy()

    x = f64(xs[0])
    tok = 0
    secs = []
    for i in range(args.warmup + args.steps):
        l = i % nl
        if i and l == 0:
            tok += 1
            x = f64(xs[tok % xs.shape[0]])
        Ld = layers[l]
        t0 = time.perf_counter()
        R = f64(Ld["router"])
        shared = (f64(Ld["sh_gate"]), f64(Ld["sh_up"]), f64(Ld["sh_down_t"]))
        experts = lambda e, Ld=Ld: (f64(Ld["gate"][e]), f64(Ld["up"][e]), f64(Ld["down_t"][e]))
        x, *_ = O.stack_layer(x, R, experts, k, shared=shared, pre_norm=True)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            secs.append(dt)
    step_s = sum(secs) / len(secs)
    value = 1.0 / (nl * step_s)
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * step_s, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "step_unit": f"one token through one layer of the {nl}-layer stack",
        "config": dict(a3b_config(WORKLOAD, w, 1), parallelism="single"),
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} timed layer passes (after {args.warmup} untimed), one token "
                                   f"through the layers in order, scaled to tokens through {nl} layers; "
                                   "router, shared and routed-expert slices fetched from the device"},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def nvtx_push(torch, name):
    """Mark a region for profiler filtering (a no-op where NVTX is unavailable)."""
    try:
        torch.cuda.nvtx.range_push(name)
    except Exception:
        pass


def nvtx_pop(torch):
    try:
        torch.cuda.nvtx.range_pop()
    except Exception:
        pass


def measure(torch, M, wl, args, stream, ws_n, device, local, nvtx_name="timed"):
    """W untimed warm-up steps, then K steps timed with CUDA events on the
    launching stream (barrier + synchronize on both sides), clocks sampled
    during the timed region. Returns the timing record of the workload."""
    wl.record = 10 ** 9  # no routing record during warm-up
    for i in range(args.warmup):
        wl.step(i, stream)
    torch.cuda.synchronize()
    st = M.moe_get_status(wl.ws, stream)
    if st != M.MOE_OK:
        raise SystemExit(f"device status after warm-up: {M.moe_status_string(st)}")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(ws_n)
    torch.cuda.synchronize()
    nvtx_push(torch, nvtx_name)
    with ClockSampler(local) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            wl.record = i
            ev[i][0].record(stream)
            wl.step(args.warmup + i, stream)
            ev[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    nvtx_pop(torch)
    barrier(ws_n)
    wl.record = 10 ** 9
    if M.moe_get_status(wl.ws, stream) != M.MOE_OK:
        raise SystemExit("device status error in timed region")
    return {"total_ms": max_over_ranks(t0.elapsed_time(t1), ws_n, device),
            "launch_ms": [a.elapsed_time(b) for a, b in ev],
            "step_bytes": [wl.nbytes(i) for i in range(args.steps)],
            "clocks": clk.summary()}


def roofline(wl, t):
    """Roofline record of a workload: algorithmic bytes of each step / that
    step's device time, averaged; peak = measured HBM copy bandwidth."""
    hbm, hbm_kind = peaks()
    achieved = statistics.mean(b / (ms * 1e-3) / 1e9 for b, ms in zip(t["step_bytes"], t["launch_ms"]))
    rec = recorded_profile(wl)
    r = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
         "traffic": rec.get("dram_bytes_per_launch"), "peak_kind": hbm_kind,
         "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS, "kernel": wl.kernel,
         "algorithmic_bytes_per_launch": statistics.mean(t["step_bytes"])}
    if getattr(wl, "launches_per_step", 1) > 1:
        r["timed_unit"] = f"whole step ({wl.launches_per_step} launches)"
    if "tensor_pipe_active_pct" in rec:
        r["tensor_pipe_active_pct"] = rec["tensor_pipe_active_pct"]
    return r


# Every other configuration of the workload list, timed after the headline in
# the default run (each built, timed and freed in turn).
EXTRA_WORKLOADS = ([("a3b_int4", {"batch": 1}), ("a3b_int4", {"batch": 8}),
                    ("channel_topk", {"keep_frac": 0.13}), ("channel_topk", {"keep_frac": 0.18})] +
                   [("batch_sweep", {"batch": b}) for b in (1, 4, 16, 64, 256)] +
                   [("channel_batch", {"batch": 4, "keep_frac": 0.13}), ("channel_batch", {"batch": 8, "keep_frac": 0.18}),
                    ("channel_topk", {"keep_frac": 0.13, "screen": True})])


def run_ours(args):
    import torch
    ws_n, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(ws_n, "nccl")
    from mixture_experts_decode_moe_b200 import build as Bld
    Bld.build()
    from mixture_experts_decode_moe_b200 import moedec as M
    from mixture_experts_decode_moe_b200 import synth as S

    wl = make_workload(args.workload, torch, M, S, device, rank, args)
    stream = torch.cuda.current_stream(device)
    torch.cuda.synchronize()

    # ---- device-timed region: inputs resident in HBM (larger than L2)
    t = measure(torch, M, wl, args, stream, ws_n, device, local)
    total_ms = t["total_ms"]

    # ---- end to end through the C ABI with host buffers (pinned), copies timed
    h2d, d2h = wl.host_buffers()
    barrier(ws_n)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    nvtx_push(torch, "e2e")
    e0.record(stream)
    for i in range(args.steps):
        wl.e2e_step(args.warmup + i, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    nvtx_pop(torch)
    barrier(ws_n)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), ws_n, device)

    tokens_total = args.steps * wl.tokens_per_step * ws_n
    value = tokens_total / (total_ms * 1e-3)
    cfg = wl.config()
    cfg["parallelism"] = f"replicas{ws_n}" if ws_n > 1 else "single"
    line = {
        "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": ws_n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else wl.dtype,
        "data": "synthetic", "config": cfg,
        "roofline": roofline(wl, t),
        "e2e": {"value": tokens_total / (e2e_ms * 1e-3), "unit": "tok/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * wl.launches_per_step,
        "clocks": t["clocks"],
    }
    if rank == 0 and ws_n == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = wl.oracle_sample(args.cpu_budget)

    # ---- the other configurations (one GPU): same timing, each freed in turn
    if ws_n == 1 and args.workload == WORKLOAD and not args.no_workloads:
        del wl
        import gc
        gc.collect()
        torch.cuda.empty_cache()
        entries = []
        for name, over in EXTRA_WORKLOADS:
            a = argparse.Namespace(**vars(args))
            for key, v in over.items():
                setattr(a, key, v)
            w2 = make_workload(name, torch, M, S, device, rank, a)
            t2 = measure(torch, M, w2, a, stream, ws_n, device, local, nvtx_name="timed_" + name)
            c2 = w2.config()
            e = {"workload": c2["workload"], "value": a.steps * w2.tokens_per_step / (t2["total_ms"] * 1e-3),
                 "unit": "tok/s", "ms_per_step": t2["total_ms"] / a.steps, "steps": a.steps, "warmup": a.warmup,
                 "tokens_per_step": w2.tokens_per_step, "dtype": w2.dtype, "roofline": roofline(w2, t2),
                 "gpu_launches": a.steps * w2.launches_per_step, "clocks": t2["clocks"], "config": c2}
            if hasattr(w2, "touched_record"):
                e["touched"] = w2.touched_record()
            if not args.no_cpu_baseline:
                e["cpu_baseline"] = w2.oracle_sample(args.extra_cpu_budget)
            entries.append(e)
            del w2
            gc.collect()
            torch.cuda.empty_cache()
        line["workloads"] = entries
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws_n > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# the sources decode_kernel is compiled from: a recorded DRAM traffic figure
# stays valid while these are unchanged
DECODE_KERNEL_SOURCES = ("common.cuh", "decode.cuh", "screen_lut.cuh", "decode_kernel.cuh")
LINEAR_KERNEL_SOURCES = ("common.cuh", "small_kernels.cuh", "linear.cuh")


def source_hash(sources=DECODE_KERNEL_SOURCES):
    import hashlib
    h = hashlib.sha256()
    cs = os.path.join(ROOT, "mixture_experts_decode_moe_b200", "csrc")
    for f in sources:
        with open(os.path.join(cs, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_profile(wl):
    """The ncu figures recorded for this workload's kernel (DRAM bytes per
    launch, tensor-pipe activity), valid only while the kernel's sources hash
    to the value recorded with them; {} otherwise."""
    tfile = os.path.join(ROOT, "profiles", f"traffic_{wl.config()['workload']}.json")
    try:
        with open(tfile) as f:
            tj = json.load(f)
    except Exception:
        return {}
    return tj if tj.get("kernel_source_hash") == source_hash(wl.sources) else {}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--extra-cpu-budget", type=float, default=4.0,
                    help="seconds of oracle time per extra configuration's cpu_baseline")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time the headline configuration only (no workloads array)")
    ap.add_argument("--workload", default=WORKLOAD, choices=["a3b_bf16", "a3b_int4", "channel_topk", "batch_sweep",
                                                            "channel_batch"])
    ap.add_argument("--batch", type=int, default=0, help="batch (a3b_int4: 1 or 8; batch_sweep: 1..256)")
    ap.add_argument("--layers", type=int, default=0,
                    help="fewer stack layers (profiling captures only; the metric is quoted on the full stack)")
    ap.add_argument("--experts", type=int, default=0,
                    help="fewer batch-sweep experts (profiling captures only; the sweep is quoted on 64)")
    ap.add_argument("--keep-frac", type=float, default=0.13, help="channel_topk budget (0.13 or 0.18)")
    ap.add_argument("--screen", action="store_true",
                    help="channel_topk: scores computed in the kernel from per-layer sketches")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
