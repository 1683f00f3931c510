#!/usr/bin/env python
"""Benchmark of the routed-MoE decode path on B200.

One step = one token through the whole hot path of a 40-layer stack shaped
like Qwen3.6-35B-A3B (H=2048, 256 experts, top-8, I=Is=512, 4-bit affine
groups of 64 with bf16 scales/biases, packed gate/up): router + softmax
top-k, the 8 selected experts' gate/up + SwiGLU + down, the sigmoid-gated
shared expert, the weighted combine and the residual/RMSNorm glue, for all
40 layers (moe_stack_forward, T=1). Each step feeds a new token, so the
selected experts change every step; the 18.1 GB expert stack is far larger
than L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0). With N > 1 (torchrun) every rank runs an
independent replica on its own tokens: the path has no exchange step.
`--impl reference` times the CPU oracle instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_routed_expert_bit_b200 import moe, synth  # noqa: E402

METRIC = "MoE-layer decode tokens/s and achieved HBM GB/s (% of 8 TB/s) at 1 B200"
SHAPE_KEY = "35b"
NOMINAL_HBM_GBS = 8000.0
# DRAM traffic of the persistent decode kernel per layer (dram__bytes_read.sum +
# dram__bytes_write.sum from one ncu capture of the first 4 layers of the workload, divided by 4).
# Each layer reads its own weights once, so the traffic of a launch over L layers is L times this.
# Keyed by the workload and a hash of the kernel's source files: a capture of another revision of
# the kernel is not reported (traffic null).
KERNEL_SOURCES = ("stack_split.cu", "decode_common.cuh", "moe_common.cuh", "moe_launch.h")
DECODE_TRAFFIC_PER_LAYER = {}


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "quantized_routed_expert_bit_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]
FALLBACK_HBM_GBS = 6650.0


def touched_bytes_per_token(shape: synth.MoEShape) -> int:
    """Algorithmic bytes of one token through the stack: per layer the k
    selected experts and the shared expert (packed codes + bf16 scales and
    biases), the router E*H*2, the shared gate H*2 and the router bias E*4."""
    per_layer = shape.top_k * shape.expert_bytes() + shape.expert_bytes(shape.shared_inter)
    per_layer += shape.num_experts * shape.hidden * 2 + (shape.hidden * 2 if shape.shared_inter > 0 else 0)
    if shape.router_bias:
        per_layer += shape.num_experts * 4
    return per_layer * shape.layers


def touched_bytes_batched(shape, layers_dev, tokens, T, steps):
    """Algorithmic bytes of a batched step: per layer every distinct expert the
    batch selects (read once), the shared expert, the router and w_sg. The
    selection is recomputed per layer on the host side from the library's
    own routing of the stack (trace), averaged over the timed steps."""
    cfg = moe.make_config(shape)
    ws = moe.Workspace(cfg, T, L=shape.layers)
    arr = moe.make_layer_array([moe.make_layer_weights(lw, cfg) for lw in layers_dev])
    ti = torch.empty(shape.layers, T, shape.top_k, dtype=torch.int32, device="cuda")
    xo = torch.empty(T, shape.hidden, dtype=torch.bfloat16, device="cuda")
    distinct = 0
    for s in range(steps):
        tr = moe.Trace(0, ti.data_ptr(), 0, 0, 0)
        moe.moe_stack_forward(cfg, arr, tokens[s * T:(s + 1) * T], xo, ws, trace=tr)
        torch.cuda.synchronize()
        for l in range(shape.layers):
            distinct += int(torch.unique(ti[l]).numel())
    per_layer_fixed = (shape.expert_bytes(shape.shared_inter) + shape.num_experts * shape.hidden * 2 +
                       (shape.hidden * 2 if shape.shared_inter > 0 else 0))
    return (distinct / steps) * shape.expert_bytes() + shape.layers * per_layer_fixed


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 8:
                self.rows.append(parts)

    def __exit__(self, *a):
        time.sleep(0.2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


def dist_setup(n_gpus: int, backend: str = "nccl"):
    """One process per GPU (torchrun sets RANK/LOCAL_RANK/WORLD_SIZE/MASTER_*). The
    ranks are independent replicas: the process group only carries the barrier
    and the max-over-ranks of the timed region. `backend="gloo"` (CPU) serves tests."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
        return dist, dist.get_rank(), world, local
    return None, 0, 1, 0


def barrier_max(dist, value: float, device: str = "cuda") -> float:
    """The largest of the ranks' values (the job's time is its slowest rank's)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_token_ids(rank: int, n: int):
    """Token seeds of one rank: every rank decodes its own tokens (disjoint streams)."""
    return [rank * 100000 + i for i in range(n)]


def job_tokens_per_s(steps: int, world: int, T: int, ms: float) -> float:
    """Whole-job throughput: the tokens all ranks processed over the slowest rank's time."""
    return steps * world * T / (ms / 1e3)


def host_layers_for(shape, layers_dev, tokens_bits):
    """Host copies (outside any timing) of what the oracle needs for these tokens."""
    import oracle
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from parity import DeviceLayer  # host view of device weights
    hosts = []
    for lw in layers_dev:
        h = DeviceLayer(shape, lw)
        for x in tokens_bits:
            lg = oracle.router_logits(x, h.router_w, h.router_bias)
            for e in oracle.softmax_topk(lg[0], shape.top_k)[0]:
                h.expert(int(e))
        hosts.append(h)
    return hosts


def cpu_oracle_tokens_per_s(shape, layers_dev, x_tokens, threads: int, budget_s: float = 12.0):
    """The oracle (as it stands) on a bounded sample of the workload: tokens
    through all layers, one layer at a time, until `budget_s` of CPU time is
    spent. Only the oracle calls are timed. Returns (tokens/s, evaluations, seconds)."""
    import oracle
    spent, evals = 0.0, 0
    for i in range(x_tokens.shape[0]):
        x = synth.bf16_bits(x_tokens[i:i + 1])
        for l0 in range(0, shape.layers, 8):
            hosts = host_layers_for(shape, layers_dev[l0:l0 + 8], [x])
            for h in hosts:
                t0 = time.perf_counter()
                oracle.layer_forward(h, x, threads=threads)
                spent += time.perf_counter() - t0
                evals += 1
            if spent >= budget_s:
                break
        if spent >= budget_s:
            break
    per_token = spent / evals * shape.layers
    return 1.0 / per_token, evals, spent


def run_reference(args):
    """Reference arm: the CPU oracle timed on this host (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    shape = synth.SHAPES[SHAPE_KEY]
    threads = os.cpu_count() or 1
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    threads = min(threads, shape.top_k + 1)  # the oracle runs one expert per thread
    n_layers = 2
    layers = [synth.make_layer(shape, l, dev) for l in range(n_layers)]
    tokens = synth.make_tokens(shape, list(range(args.warmup + args.steps)), dev)
    xs = [synth.bf16_bits(tokens[i:i + 1]) for i in range(tokens.shape[0])]
    hosts = host_layers_for(shape, layers, xs)
    for i in range(args.warmup):
        for h in hosts:
            oracle.layer_forward(h, xs[i], threads=threads)
    t0 = time.perf_counter()
    for i in range(args.warmup, args.warmup + args.steps):
        for h in hosts:
            oracle.layer_forward(h, xs[i], threads=threads)
    dt = time.perf_counter() - t0
    sec_per_token = dt / args.steps * (shape.layers / n_layers)
    value = 1.0 / sec_per_token
    sample = f"1 token x {n_layers} of {shape.layers} layers per step, scaled to {shape.layers}"
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec_per_token * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(shape),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def workload_config(shape):
    return {"workload": f"{shape.name}: T={shape.tokens} through {shape.layers} stacked MoE layers "
                        f"(H={shape.hidden}, E={shape.num_experts}, top-{shape.top_k}, I=Is={shape.inter}, "
                        f"{shape.bits}-bit affine g{shape.group}, bf16 scale/bias, packed gate/up)",
            "tokens_per_step": shape.tokens, "layers": shape.layers,
            "l2": f"inputs larger than L2: {shape.layers * shape.num_experts * shape.expert_bytes() / 1e9:.1f} GB "
                  "resident expert stack, a new token (new experts) every step"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=0,
                    help="profile a shorter stack (small ncu case); the default is the full stack")
    ap.add_argument("--workload", default=SHAPE_KEY, choices=sorted(synth.SHAPES),
                    help="35b (default, the headline), 80b, 35b8, or the batched 35b_t64 / 35b_t512")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
        return

    dist, rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    key = args.workload
    shape = synth.SHAPES[key]
    if args.layers:
        import dataclasses
        shape = dataclasses.replace(shape, layers=args.layers, name=shape.name + f"-first{args.layers}")
    cfg = moe.make_config(shape)
    layers = [synth.make_layer(shape, l, "cuda", seed_id=synth.SHAPE_SEED_ID[key])
              for l in range(shape.layers)]
    arr = moe.make_layer_array([moe.make_layer_weights(lw, cfg) for lw in layers])
    T = shape.tokens
    ws = moe.Workspace(cfg, T, L=shape.layers)
    nsteps = args.warmup + args.steps
    # each rank its own tokens (independent replicas); a step is one batch of T tokens
    if T == 1:
        tokens = synth.make_tokens(shape, rank_token_ids(rank, nsteps), "cuda", seed_id=synth.SHAPE_SEED_ID[key])
    else:
        tokens = torch.cat([synth.make_batch(shape, T, i, "cuda", seed_id=synth.SHAPE_SEED_ID[key])
                            for i in rank_token_ids(rank, nsteps)])
    xout = torch.empty(T, shape.hidden, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    def step(i):
        moe.moe_stack_forward(cfg, arr, tokens[i * T:(i + 1) * T], xout, ws, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == moe.MOE_OK

    # ---- device-timed region: inputs resident in HBM
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for i in range(args.warmup, nsteps):
            step(i)
        ev1.record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
    ms = ev0.elapsed_time(ev1)
    ms = barrier_max(dist, ms)
    status = moe.moe_get_device_status(ws)

    # ---- the same steps again, each bracketed by its own events: the spread of a step
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    evs[0].record(stream)
    for i in range(args.warmup, nsteps):
        step(i)
        evs[i - args.warmup + 1].record(stream)
    torch.cuda.synchronize()
    per = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps))
    pct = {f"p{q}": per[min(len(per) - 1, int(q / 100 * len(per)))] for q in (10, 50, 90)}

    # ---- end to end: host tokens in pinned memory, result read back every step
    host_tok = tokens.cpu().pin_memory()
    host_out = torch.empty(T, shape.hidden, dtype=torch.bfloat16).pin_memory()
    xin = torch.empty(T, shape.hidden, dtype=torch.bfloat16, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(args.warmup, nsteps):
        xin.copy_(host_tok[i * T:(i + 1) * T], non_blocking=True)
        moe.moe_stack_forward(cfg, arr, xin, xout, ws, stream=stream)
        host_out.copy_(xout, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = barrier_max(dist, e0.elapsed_time(e1))

    launches_per_step = moe.moe_stack_kernel_launches(cfg, T, shape.layers)
    path = moe.moe_stack_path_name(cfg, T, shape.layers)
    persistent = launches_per_step < shape.layers
    if T == 1:
        bytes_step = touched_bytes_per_token(shape)
    else:
        bytes_step = touched_bytes_batched(shape, layers, tokens[args.warmup * T:nsteps * T], T, args.steps)
    total_tokens = args.steps * world * T
    tok_s = job_tokens_per_s(args.steps, world, T, ms)
    per_step_s = ms / 1e3 / args.steps
    gbs = bytes_step / per_step_s / 1e9
    peak, peak_src = peaks()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and T == 1:
        threads = min(os.cpu_count() or 1, shape.top_k + 1)  # one expert per thread
        v, evals, dt = cpu_oracle_tokens_per_s(shape, layers, tokens, threads)
        cpu = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{evals} (token, layer) evaluations of the bench tokens, {dt:.1f} s of oracle time, "
                         f"scaled to {shape.layers} layers per token; expert copies to the host untimed"}

    traffic = None
    src_hash = kernel_source_hash()
    if persistent and (key, src_hash) in DECODE_TRAFFIC_PER_LAYER:
        traffic = DECODE_TRAFFIC_PER_LAYER[(key, src_hash)] * shape.layers
    if rank == 0:
        out = {
            "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "weights": f"u{shape.bits} affine g{shape.group}, bf16 scale/bias",
            "data": "synthetic", "config": workload_config(shape),
            "hbm_gbs": gbs, "hbm_frac_of_8tbs": gbs / NOMINAL_HBM_GBS,
            "roofline": {"bound": "hbm",
                         "kernel": (f"{path} (the whole stack, one launch per step)" if persistent
                                    else f"moe_stack_forward step on the {path} path (all its kernels)"),
                         "achieved": gbs, "peak": peak, "peak_source": peak_src, "unit": "GB/s",
                         "frac": gbs / peak, "traffic": traffic,
                         "bytes_per_step": bytes_step,
                         "note": "achieved = algorithmic bytes per step / device time per step (CUDA events "
                                 "on the launch stream around the timed steps)"},
            "cpu_baseline": cpu,
            "e2e": {"value": total_tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": T * shape.hidden * 2, "d2h_bytes_per_step": T * shape.hidden * 2},
            "step_ms": pct,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(),
            "device_status": moe.status_string(status),
        }
        print(json.dumps(out), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
