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


def algorithmic_layer_bytes(H, E, I, k, I_sh):
    """Bytes one batch-1 token must read in one layer: router [E,H] + k routed
    SwiGLU experts (3*I*H) + the shared expert (3*I_sh*H), all bf16."""
    return 2 * (E * H + k * 3 * I * H + 3 * I_sh * H)


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


# ---------------------------------------------------------------- model setup


def build_stack(torch, M, S, device):
    w = S.WORKLOADS[WORKLOAD]
    H, E, I, k, I_sh, nl = w["H"], w["E"], w["I"], w["k"], w["I_shared"], w["layers"]
    layers, descs = [], []
    for l in range(nl):
        Ld = S.swiglu_layer_bf16(H, E, I, I_sh, seed=S.weight_seed(w["cfg"], l), device=device,
                                 router_scale=w["router_scale"])
        layers.append(Ld)
        descs.append(M.make_desc(H, E, I, k, router=Ld["router"], gate=Ld["gate"], up=Ld["up"],
                                 down_t=Ld["down_t"], sh_gate=Ld["sh_gate"], sh_up=Ld["sh_up"],
                                 sh_down_t=Ld["sh_down_t"]))
    return w, layers, descs


# ---------------------------------------------------------------- CPU oracle timing


def oracle_rate(layers, w, xs, budget_s=12.0, max_layers=None, start_token=0):
    """Time the fp64 oracle (as it stands) layer by layer on whole tokens.

    Token t goes through layers 0..L-1 (residual between layers); per layer the
    oracle copies the router, the shared expert and only the routed experts'
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
        experts = lambda e, Ld=Ld: (f64(Ld["gate"][e]), f64(Ld["up"][e]), f64(Ld["down_t"][e]))
        y, *_ = O.moe_layer(x, R, experts, k, shared=shared)
        x = O.residual_bf16(x, y)
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
    """The oracle arm: the fp64 CPU oracle timed on this host's cores."""
    ws_n, rank, local = dist_env()
    if rank != 0:
        return 0
    import torch
    from mixture_experts_decode_moe_b200 import synth as S
    w = S.WORKLOADS[WORKLOAD]
    H, E, I, k, I_sh, nl = w["H"], w["E"], w["I"], w["k"], w["I_shared"], w["layers"]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    # one CPU copy of the stack would be 64 GB: keep it on the device when
    # there is one and let the oracle fetch the slices it reads
    layers = [S.swiglu_layer_bf16(H, E, I, I_sh, seed=S.weight_seed(w["cfg"], l), device=dev,
                                  router_scale=w["router_scale"]) for l in range(nl)]
    xs = S.tokens(w["tokens"], H, seed=S.act_seed(w["cfg"]), device=dev)
    per_step = max(0.2, 90.0 / max(1, args.steps + args.warmup))
    secs, n_layers = [], 0
    for i in range(args.warmup + args.steps):
        tps, done, dt = oracle_rate(layers, w, xs, budget_s=per_step, start_token=i)
        if i >= args.warmup:
            secs.append(1.0 / tps)
            n_layers += done
    sec = sum(secs) / len(secs)
    value = 1.0 / sec
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sec, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "layers": nl, "hidden": H, "experts": E, "top_k": k,
                   "expert_intermediate": I, "shared_intermediate": I_sh, "batch": 1},
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step >= {per_step:.2f} s of whole layers ({n_layers} layer passes "
                                   f"timed in all), scaled to tokens through {nl} layers; routed-expert "
                                   "slices fetched from the device"},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


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

    w, layers, descs = build_stack(torch, M, S, device)
    H, E, I, k, I_sh, nl = w["H"], w["E"], w["I"], w["k"], w["I_shared"], w["layers"]
    B = 1
    xs = S.tokens(w["tokens"], H, seed=S.act_seed(w["cfg"]) + 97 * rank, device=device)
    ws = M.alloc_workspace(descs[0], B, device)
    x_out = torch.empty((B, H), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)
    torch.cuda.synchronize()

    def step(i):
        M.moe_stack_forward(descs, xs[i % w["tokens"]:][:B], x_out, ws, flags=M.MOE_STACK_PRE_RMSNORM,
                            stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    st = M.moe_get_status(ws, stream)
    if st != M.MOE_OK:
        raise SystemExit(f"device status after warm-up: {M.moe_status_string(st)}")

    # ---- device-timed region: inputs resident in HBM
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(ws_n)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step(args.warmup + i)
            ev[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(ws_n)
    total_ms = max_over_ranks(t0.elapsed_time(t1), ws_n, device)
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    kern_ms = statistics.mean(launch_ms)
    clocks = clk.summary()
    if M.moe_get_status(ws, stream) != M.MOE_OK:
        raise SystemExit("device status error in timed region")

    # ---- end to end through the C ABI with host buffers (pinned), copies timed
    x_host = xs.cpu().pin_memory()
    out_host = torch.empty((B, H), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty((B, H), dtype=torch.bfloat16, device=device)
    barrier(ws_n)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        j = (args.warmup + i) % w["tokens"]
        x_dev.copy_(x_host[j:j + B], non_blocking=True)
        M.moe_stack_forward(descs, x_dev, x_out, ws, flags=M.MOE_STACK_PRE_RMSNORM, stream=stream)
        out_host.copy_(x_out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(ws_n)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), ws_n, device)

    layer_bytes = algorithmic_layer_bytes(H, E, I, k, I_sh)
    launch_bytes = layer_bytes * nl * B
    hbm, hbm_kind = peaks()
    achieved = launch_bytes / (kern_ms * 1e-3) / 1e9
    traffic = None
    tfile = os.path.join(ROOT, "profiles", "decode_kernel_a3b_bf16_traffic.json")
    if os.path.exists(tfile):
        try:
            with open(tfile) as f:
                tj = json.load(f)
            if tj.get("kernel_source_hash") == source_hash():
                traffic = tj.get("dram_bytes_per_launch")
        except Exception:
            traffic = None

    tokens_total = args.steps * B * ws_n
    value = tokens_total / (total_ms * 1e-3)
    line = {
        "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": ws_n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "layers": nl, "hidden": H, "experts": E, "top_k": k,
                   "expert_intermediate": I, "shared_intermediate": I_sh, "batch": B,
                   "parallelism": f"replicas{ws_n}" if ws_n > 1 else "single",
                   "l2": "inputs larger than L2: 64.7 GB of weights, each token reads 2.31 GB"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": traffic, "peak_kind": hbm_kind,
                     "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                     "kernel": "decode_kernel<1,bf16,planar>", "algorithmic_bytes_per_launch": launch_bytes},
        "e2e": {"value": tokens_total / (e2e_ms * 1e-3), "unit": "tok/s", "h2d_bytes_per_step": B * H * 2,
                "d2h_bytes_per_step": B * H * 2},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    if rank == 0 and ws_n == 1 and not args.no_cpu_baseline:
        tps, done, dt = oracle_rate(layers, w, xs, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": tps, "unit": "tok/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"{done} layer passes of the stack in {dt:.1f} s, scaled to tokens "
                                          f"through {nl} layers (fp64; routed-expert slices copied from the device)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws_n > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def source_hash():
    import hashlib
    h = hashlib.sha256()
    cs = os.path.join(ROOT, "mixture_experts_decode_moe_b200", "csrc")
    for f in sorted(os.listdir(cs)):
        with open(os.path.join(cs, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
