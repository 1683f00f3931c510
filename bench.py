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
# dram__bytes_read.sum + dram__bytes_write.sum per layer of decode_split_kernel from the 4-layer
# capture in profiles/decode_split_kernel_35b_l4_full.md, keyed by workload and kernel source hash
DECODE_TRAFFIC_PER_LAYER = {("35b", "afa65bc43f7fbf78"): (68_041_728 + 1_808_384) / 4}


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


def traced_stack(shape, cfg, arr, ws, x0):
    """One token through the stack with a trace: the GPU's own input, selection and output of
    every layer (outside any timing)."""
    L, H, k = shape.layers, shape.hidden, shape.top_k
    tx = torch.empty(L, 1, H, dtype=torch.bfloat16, device="cuda")
    ti = torch.empty(L, 1, k, dtype=torch.int32, device="cuda")
    tw = torch.empty(L, 1, k, dtype=torch.float32, device="cuda")
    ty = torch.empty(L, 1, H, dtype=torch.bfloat16, device="cuda")
    xo = torch.empty(1, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_stack_forward(cfg, arr, x0, xo, ws, trace=moe.Trace(tx.data_ptr(), ti.data_ptr(), tw.data_ptr(),
                                                               ty.data_ptr()))
    torch.cuda.synchronize()
    return synth.bf16_bits(tx), ti.cpu().numpy(), tw.cpu().numpy(), synth.bf16_bits(ty)


def cpu_oracle_leg(shape, cfg, arr, ws, layers_dev, x_tokens, threads: int, budget_s: float = 12.0):
    """The oracle (as it stands) on a bounded sample of the workload, timed on the host cores:
    (token, layer) evaluations on the GPU's own input of that layer (from a traced run of the
    same token), until `budget_s` of oracle time is spent. Only the oracle calls are timed.
    Each evaluation is also compared with the GPU's output of that layer: the same three checks
    the GPU tests apply (expert set where the k-th/(k+1)-th logit gap exceeds 1e-4, weights within
    1e-5, bf16 output within max-abs 2e-2 and rel-L2 1e-3 of the oracle's rounded output).
    Returns (tokens/s, evaluations, seconds, parity summary)."""
    import numpy as np
    import oracle
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from parity import GAP_MIN, W_TOL, Y_MAX_ABS, Y_REL_L2, y_errors
    spent, evals = 0.0, 0
    par = {"pairs": 0, "gap_excluded": 0, "index_mismatch": 0, "max_w_err": 0.0, "max_abs": 0.0,
           "max_rel_l2": 0.0}
    for i in range(x_tokens.shape[0]):
        tx, ti, tw, ty = traced_stack(shape, cfg, arr, ws, x_tokens[i:i + 1])
        for l0 in range(0, shape.layers, 8):
            hosts = host_layers_for(shape, layers_dev[l0:l0 + 8], [tx[l] for l in range(l0, min(l0 + 8, shape.layers))])
            for dl, h in enumerate(hosts):
                l = l0 + dl
                t0 = time.perf_counter()
                ref = oracle.layer_forward(h, tx[l], threads=threads)
                spent += time.perf_counter() - t0
                evals += 1
                par["pairs"] += 1
                gi = ti[l][0].astype(np.int64)
                if ref["gap"][0] > GAP_MIN:
                    if set(gi.tolist()) != set(ref["idx"][0].tolist()):
                        par["index_mismatch"] += 1
                    else:
                        rw = dict(zip(ref["idx"][0].tolist(), ref["w"][0].tolist()))
                        par["max_w_err"] = max(par["max_w_err"], max(abs(float(tw[l][0][j]) - rw[int(gi[j])])
                                                                     for j in range(len(gi))))
                else:
                    par["gap_excluded"] += 1
                    ref = oracle.layer_forward(h, tx[l], force_idx=ti[l], threads=threads)
                ma, rel, _ = y_errors(ty[l][0], ref)
                par["max_abs"] = max(par["max_abs"], ma)
                par["max_rel_l2"] = max(par["max_rel_l2"], rel)
            if spent >= budget_s:
                break
        if spent >= budget_s:
            break
    par["pass"] = bool(par["index_mismatch"] == 0 and par["max_w_err"] <= W_TOL and par["max_abs"] <= Y_MAX_ABS
                       and par["max_rel_l2"] <= Y_REL_L2)
    per_token = spent / evals * shape.layers
    return 1.0 / per_token, evals, spent, par


def run_reference(args):
    """Reference arm: the CPU oracle timed on this host (rank 0 only). Each step is a bounded
    sample of the workload (one token through `n_layers` of its layers); `ms_per_step` is the
    measured time of that sample and `value` scales it to the whole stack."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    shape = synth.SHAPES[SHAPE_KEY]
    cores = os.cpu_count() or 1
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    threads = min(cores, shape.top_k + 1)  # the oracle runs one expert per thread
    n_layers = 2
    layers = [synth.make_layer(shape, l, dev) for l in range(n_layers)]
    tokens = synth.make_tokens(shape, list(range(args.warmup + args.steps)), dev)
    xs = [synth.bf16_bits(tokens[i:i + 1]) for i in range(tokens.shape[0])]
    hosts = host_layers_for(shape, layers, xs)
    for i in range(args.warmup):
        for h in hosts:
            oracle.layer_forward(h, xs[i], threads=threads)
    per = []
    for i in range(args.warmup, args.warmup + args.steps):
        t0 = time.perf_counter()
        for h in hosts:
            oracle.layer_forward(h, xs[i], threads=threads)
        per.append(time.perf_counter() - t0)
    dt = sum(per)
    sample_ms = dt / args.steps * 1e3
    scale = shape.layers / n_layers
    value = 1.0 / (dt / args.steps * scale)
    sample = (f"1 token x {n_layers} of {shape.layers} layers per step (measured {sample_ms:.1f} ms per step); "
              f"value scaled by {scale:.0f} to the whole stack")
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sample_ms,
        "ms_per_step_note": f"measured time of one sampled step ({n_layers} of {shape.layers} layers); "
                            f"the whole-stack time per token is {sample_ms * scale:.1f} ms",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(shape),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "threads": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "step_ms_raw": [round(x * 1e3, 3) for x in per],
        "seeds": seeds_desc(SHAPE_KEY, list(range(args.warmup, args.warmup + args.steps))),
    }
    print(json.dumps(out), flush=True)


def workload_config(shape, stock=False):
    layout = "stock gate/up (separate gate and up tensors)" if stock else "packed gate/up"
    return {"workload": f"{shape.name}: T={shape.tokens} through {shape.layers} stacked MoE layers "
                        f"(H={shape.hidden}, E={shape.num_experts}, top-{shape.top_k}, I=Is={shape.inter}, "
                        f"{shape.bits}-bit affine g{shape.group}, bf16 scale/bias, {layout})",
            "tokens_per_step": shape.tokens, "layers": shape.layers,
            "l2": f"inputs larger than L2: {shape.layers * shape.num_experts * shape.expert_bytes() / 1e9:.1f} GB "
                  "resident expert stack, a new token (new experts) every step"}


def seeds_desc(key, token_ids):
    cid = synth.SHAPE_SEED_ID[key]
    return {"weights": f"tensor t of layer l: {cid}*1000003 + l*1009 + t (synth.layer_seed)",
            "tokens": f"token i: {cid}*1000003 + 999983 + i (synth.token_seed), batch b: token_seed(1000000 + b)",
            "token_ids": [token_ids[0], token_ids[-1]] if token_ids else []}


# The GPU tests that check each workload's path element by element against the oracle.
PARITY_TESTS = {
    "35b": "tests/test_gpu_stack.py::test_decode_stack_parity[35b]",
    "80b": "tests/test_gpu_stack.py::test_decode_stack_parity[80b]",
    "35b8": "tests/test_gpu_stack.py::test_decode_stack_parity[35b8]",
    "35b_t64": "tests/test_gpu_stack.py::test_batched_stack_parity[35b_t64-grouped_gemv]",
    "35b_t512": "tests/test_gpu_stack.py::test_batched_stack_parity[35b_t512-batched]",
}


class Workload:
    """One workload's stack on the device, ready to step: weights (with their decode-ready
    copies), a workspace and the tokens of `nsteps` steps."""

    def __init__(self, key, nsteps, rank=0, layers=0, stock=False):
        self.key = key
        self.stock = stock
        shape = synth.SHAPES[key]
        if layers:
            import dataclasses
            shape = dataclasses.replace(shape, layers=layers, name=shape.name + f"-first{layers}")
        self.shape = shape
        self.cfg = moe.make_config(shape)
        sid = synth.SHAPE_SEED_ID[key]
        self.layers = [synth.make_layer(shape, l, "cuda", seed_id=sid) for l in range(shape.layers)]
        if stock:  # the stock gate/up layout: separate gate and up tensors (the packed copies freed)
            self.layers = [synth.stock_layer(lw) for lw in self.layers]
            torch.cuda.empty_cache()
        self.arr = moe.make_layer_array([moe.make_layer_weights(lw, self.cfg) for lw in self.layers])
        self.T = shape.tokens
        self.ws = moe.Workspace(self.cfg, self.T, L=shape.layers)
        self.token_ids = rank_token_ids(rank, nsteps)
        if self.T == 1:
            self.tokens = synth.make_tokens(shape, self.token_ids, "cuda", seed_id=sid)
        else:
            self.tokens = torch.cat([synth.make_batch(shape, self.T, i, "cuda", seed_id=sid) for i in self.token_ids])
        self.xout = torch.empty(self.T, shape.hidden, dtype=torch.bfloat16, device="cuda")

    def step(self, i, stream):
        T = self.T
        moe.moe_stack_forward(self.cfg, self.arr, self.tokens[i * T:(i + 1) * T], self.xout, self.ws, stream=stream)

    def path(self):
        p = moe.moe_stack_path_name(self.cfg, self.T, self.shape.layers)
        return "grouped_gemv" if (self.stock and p == "batched") else p  # the tensor cores read packed only

    def launches(self):
        n = moe.moe_stack_kernel_launches(self.cfg, self.T, self.shape.layers)
        return 1 + 6 * self.shape.layers if (self.stock and self.path() != moe.moe_stack_path_name(
            self.cfg, self.T, self.shape.layers)) else n

    def bytes_per_step(self, warmup, steps):
        if self.T == 1:
            return touched_bytes_per_token(self.shape)
        T = self.T
        return touched_bytes_batched(self.shape, self.layers, self.tokens[warmup * T:(warmup + steps) * T], T, steps)


def per_step_ms(wl, first, steps, stream):
    """Each step between its own events (device time): the raw per-step list."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    evs[0].record(stream)
    for i in range(first, first + steps):
        wl.step(i, stream)
        evs[i - first + 1].record(stream)
    torch.cuda.synchronize()
    return [evs[i].elapsed_time(evs[i + 1]) for i in range(steps)]


def pct(v):
    v = sorted(v)
    return {f"p{q}": v[min(len(v) - 1, int(q / 100 * len(v)))] for q in (10, 50, 90)}


def secondary(keys, steps, warmup, peak, budget_s=150.0):
    """The other workloads, each timed like the headline on its own stack (made, timed and
    freed in turn), within about budget_s of wall time: tokens/s, algorithmic GB/s and the
    fraction of the measured copy peak, the per-step spread, the path and its launches."""
    out = {}
    t_start = time.time()
    stream = torch.cuda.current_stream()
    for key in keys:
        if time.time() - t_start > budget_s:
            out[key] = {"skipped": "time budget of the secondary block spent"}
            continue
        wl = Workload(key, warmup + steps)
        for i in range(warmup):
            wl.step(i, stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(warmup, warmup + steps):
            wl.step(i, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        status = moe.moe_get_device_status(wl.ws)
        raw = per_step_ms(wl, warmup, steps, stream)
        b = wl.bytes_per_step(warmup, steps)
        gbs = b / (ms / 1e3 / steps) / 1e9
        out[key] = {"workload": workload_config(wl.shape)["workload"], "tokens_per_s": steps * wl.T / (ms / 1e3),
                    "ms_per_step": ms / steps, "bytes_per_step": b, "hbm_gbs": gbs, "frac_of_measured_peak": gbs / peak,
                    "frac_of_8tbs": gbs / NOMINAL_HBM_GBS, "step_ms": pct(raw),
                    "step_ms_raw": [round(x, 4) for x in raw], "path": wl.path(), "launches_per_step": wl.launches(),
                    "steps": steps, "warmup": warmup, "device_status": moe.status_string(status),
                    "parity_test": PARITY_TESTS.get(key), "seeds": seeds_desc(key, wl.token_ids)}
        del wl
        torch.cuda.empty_cache()
    return out


def dispatch_sweep(steps=8, warmup=3, Ts=(1, 2, 3, 4, 6, 8, 12, 16, 24, 32, 48, 64, 96, 128, 192, 256, 512), key=None):
    """The multi-token paths for T tokens through a stack (the persistent decode kernel a token at a
    time, up to 16 tokens; the per-token kernels; the grouped GEMV; the batched tensor-core path;
    moe_set_decode_max_tokens / moe_set_gemv_min_tokens / moe_set_batched_min_tokens pick one; one
    token through a stack always runs the persistent decode kernel): one JSON line per (T, path)
    with its device time per step, then the fastest path per T."""
    key = key or SHAPE_KEY
    shape = synth.SHAPES[key]
    cfg = moe.make_config(shape)
    sid = synth.SHAPE_SEED_ID[key]
    layers = [synth.make_layer(shape, l, "cuda", seed_id=sid) for l in range(shape.layers)]
    arr = moe.make_layer_array([moe.make_layer_weights(lw, cfg) for lw in layers])
    stream = torch.cuda.current_stream()
    best = {}
    # (path, GEMV threshold, tensor-core threshold, decode threshold)
    paths = (("decode_split_kernel", 1 << 30, 1 << 30, 1 << 30), ("per_layer", 1 << 30, 1 << 30, 1),
             ("grouped_gemv", 1, 1 << 30, 1), ("batched", 1 << 30, 1, 1))
    for T in Ts:
        x = [synth.make_tokens(shape, [i], "cuda", seed_id=sid) if T == 1 else
             synth.make_batch(shape, T, i, "cuda", seed_id=sid) for i in range(warmup + steps)]
        xo = torch.empty(T, shape.hidden, dtype=torch.bfloat16, device="cuda")
        ws = moe.Workspace(cfg, T, L=shape.layers)
        for path, gthr, bthr, dthr in paths:
            pg, pb = moe.moe_set_gemv_min_tokens(gthr), moe.moe_set_batched_min_tokens(bthr)
            pd = moe.moe_set_decode_max_tokens(dthr)
            try:
                name = moe.moe_stack_path_name(cfg, T, shape.layers)
                launches = moe.moe_stack_kernel_launches(cfg, T, shape.layers)
                if T > 1 and (name != path or (path.startswith("decode") and T > 16)):
                    continue  # (a token at a time on the decode kernel is timed up to 16 tokens)
                for i in range(warmup):
                    moe.moe_stack_forward(cfg, arr, x[i], xo, ws, stream=stream)
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for i in range(warmup, warmup + steps):
                    moe.moe_stack_forward(cfg, arr, x[i], xo, ws, stream=stream)
                e1.record(stream)
                torch.cuda.synchronize()
            finally:
                moe.moe_set_gemv_min_tokens(pg)
                moe.moe_set_batched_min_tokens(pb)
                moe.moe_set_decode_max_tokens(pd)
            assert moe.moe_get_device_status(ws) == moe.MOE_OK
            ms = e0.elapsed_time(e1) / steps
            rec = {"sweep": "dispatch", "workload": shape.name, "T": T, "path": name, "ms_per_step": ms,
                   "tokens_per_s": T / (ms / 1e3), "launches_per_step": launches}
            print(json.dumps(rec), flush=True)
            if T not in best or ms < best[T][1]:
                best[T] = (name, ms)
            if T == 1:
                break  # one token: the persistent kernel whatever the thresholds
        del ws
    print(json.dumps({"sweep": "dispatch", "workload": shape.name,
                      "fastest_path": {str(T): b[0] for T, b in best.items()}}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true", help="skip the other workloads' block")
    ap.add_argument("--sweep", action="store_true",
                    help="time the per-token kernels, the grouped GEMV and the tensor-core path for "
                         "T = 1..512 tokens and exit")
    ap.add_argument("--stock", action="store_true",
                    help="the stock (unpacked) gate/up layout: each expert's gate and up rows in separate "
                         "tensors, the A/B baseline of the packed layout")
    ap.add_argument("--path", default=None, choices=["decode", "per_layer", "grouped_gemv", "batched"],
                    help="pin the multi-token path (moe_set_gemv_min_tokens / moe_set_batched_min_tokens); "
                         "the default is the library's choice for the token count")
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

    if args.sweep:
        dispatch_sweep(key=args.workload)
        return
    if args.path is not None:  # process-wide dispatch thresholds
        gthr, bthr, dthr = {"decode": (1 << 30, 1 << 30, 1 << 30), "per_layer": (1 << 30, 1 << 30, 1),
                            "grouped_gemv": (2, 1 << 30, 1), "batched": (1 << 30, 2, 1)}[args.path]
        moe.moe_set_gemv_min_tokens(gthr)
        moe.moe_set_batched_min_tokens(bthr)
        moe.moe_set_decode_max_tokens(dthr)
    dist, rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    key = args.workload
    nsteps = args.warmup + args.steps
    # each rank its own tokens (independent replicas); a step is one batch of T tokens
    wl = Workload(key, nsteps, rank, args.layers, stock=args.stock)
    shape, T = wl.shape, wl.T
    stream = torch.cuda.current_stream()

    for i in range(args.warmup):
        wl.step(i, stream)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(wl.ws) == moe.MOE_OK

    # ---- device-timed region: inputs resident in HBM
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for i in range(args.warmup, nsteps):
            wl.step(i, stream)
        ev1.record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
    ms = ev0.elapsed_time(ev1)
    ms = barrier_max(dist, ms)
    status = moe.moe_get_device_status(wl.ws)

    # ---- the same steps again, each bracketed by its own events: the spread of a step
    raw = per_step_ms(wl, args.warmup, args.steps, stream)

    # ---- end to end: host tokens in pinned memory, result read back every step
    host_tok = wl.tokens.cpu().pin_memory()
    host_out = torch.empty(T, shape.hidden, dtype=torch.bfloat16).pin_memory()
    xin = torch.empty(T, shape.hidden, dtype=torch.bfloat16, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(args.warmup, nsteps):
        xin.copy_(host_tok[i * T:(i + 1) * T], non_blocking=True)
        moe.moe_stack_forward(wl.cfg, wl.arr, xin, wl.xout, wl.ws, stream=stream)
        host_out.copy_(wl.xout, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = barrier_max(dist, e0.elapsed_time(e1))

    launches_per_step = wl.launches()
    path = wl.path()
    persistent = launches_per_step < shape.layers
    bytes_step = wl.bytes_per_step(args.warmup, args.steps)
    total_tokens = args.steps * world * T
    tok_s = job_tokens_per_s(args.steps, world, T, ms)
    per_step_s = ms / 1e3 / args.steps
    gbs = bytes_step / per_step_s / 1e9
    peak, peak_src = peaks()

    cpu = None
    # (the stock layout is an A/B variant of the same workload: its line carries no oracle leg)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.stock and T == 1:
        cores = os.cpu_count() or 1
        threads = min(cores, shape.top_k + 1)  # one expert per thread
        v, evals, dt, par = cpu_oracle_leg(shape, wl.cfg, wl.arr, wl.ws, wl.layers, wl.tokens[:4], threads)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "threads": threads, "kind": "oracle",
               "sample": f"{evals} (token, layer) evaluations of the first bench tokens on the GPU's own per-layer "
                         f"inputs, {dt:.1f} s of oracle time, scaled to {shape.layers} layers per token; expert "
                         "copies to the host untimed",
               "parity": par}

    traffic = None
    src_hash = kernel_source_hash()
    if persistent and (key, src_hash) in DECODE_TRAFFIC_PER_LAYER:
        traffic = DECODE_TRAFFIC_PER_LAYER[(key, src_hash)] * shape.layers
    sec = None
    if world == 1 and not args.no_secondary and not args.layers and not args.stock and key == SHAPE_KEY:
        del wl
        torch.cuda.empty_cache()
        sec = secondary([k for k in ("80b", "35b8", "35b_t64", "35b_t512") if k != key], 32, args.warmup, peak)
    if rank == 0:
        out = {
            "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "weights": f"u{shape.bits} affine g{shape.group}, bf16 scale/bias",
            "arithmetic": "exact integer byte dot products (dp4a) of the codes with a 22-bit fixed-point copy of the "
                          "activations, fp32 scale/bias and sums" if path == "decode_split_kernel" else "fp32",
            "data": "synthetic", "config": workload_config(shape, args.stock),
            "hbm_gbs": gbs, "hbm_frac_of_8tbs": gbs / NOMINAL_HBM_GBS,
            "roofline": {"bound": "hbm",
                         "kernel": (f"{path} (the whole stack, one launch per step)" if persistent
                                    else f"moe_stack_forward step on the {path} path (all its kernels)"),
                         "achieved": gbs, "peak": peak, "peak_source": peak_src, "unit": "GB/s",
                         "frac": gbs / peak, "traffic": traffic,
                         "traffic_note": None if traffic is not None else
                         f"no ncu capture of this kernel revision (source hash {src_hash})",
                         "bytes_per_step": bytes_step,
                         "note": "achieved = algorithmic bytes per step / device time per step (CUDA events "
                                 "on the launch stream around the timed steps)"},
            "cpu_baseline": cpu,
            "e2e": {"value": total_tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": T * shape.hidden * 2, "d2h_bytes_per_step": T * shape.hidden * 2},
            "step_ms": pct(raw),
            "step_ms_raw": [round(x, 4) for x in raw],
            "seeds": seeds_desc(key, wl.token_ids if sec is None else rank_token_ids(rank, nsteps)),
            "parity_test": PARITY_TESTS.get(key),
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(),
            "device_status": moe.status_string(status),
            "secondary": sec,
        }
        print(json.dumps(out), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
