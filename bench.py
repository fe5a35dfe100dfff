#!/usr/bin/env python
"""Benchmark of the low-rank decode path on B200.

Headline workload (one "step"): one decode token through a LLaMA-7B-shaped
stack of 32 layers whose Q/K/V/O projections are truncated-SVD factorised
(bf16, hidden 4096, seeded non-uniform ranks in [512, 1536] at 40 % parameter
reduction, batch 1).  Per layer, Q, K and V are computed from the layer input
x; the O projection reads the V output (single-token attention returns V
exactly) and its output is the next layer's input.  The whole stack is one
lr_linear_chain call: one persistent launch per step, two chain steps per
layer (Q/K/V; O), each waiting only for the step it reads.

The 32 layers hold 2.58 GB of factors, far above the 126 MB L2, so every step
streams them from HBM (no L2 flush needed).  Timing: W untimed warm-up steps,
then exactly K steps of a captured CUDA graph of the step, bracketed by a
barrier and a device synchronisation, measured with CUDA events, max over
ranks.  With --gpus N > 1 (torchrun), every rank runs its own replica of the
workload on its own GPU (independent requests; weak scaling, no data-path
collective).

At N = 1 the same JSON line carries `rows`: every configuration of the path,
each with its own CUDA-event time, roofline, CPU-oracle baseline and an
end-to-end time through the C ABI with host buffers:
  c1        single fp32 low-rank linear, 256 x 256, rank 32, one token
  c2b4/b16  the headline stack at batch 4 and 16
  c3b1/8/32 hybrid int8 SwiGLU FFN (7B shapes), batch 1, 8, 32
  c4k4/16/32 latent-KV flash decoding, batch 8, 32 heads, rank 32, ctx 4K/16K/32K
  c5        W8A8 prefill of one 13B layer (7 projections), 2048 tokens
and the uncompressed baselines the pages compare against, with the speed-up
of the low-rank path over each:
  c2dense   dense bf16 Q/K/V/O stack, 32 layers, batch 1
  c3dense   dense int8 SwiGLU FFN (all 11008 channels dense), batch 1
  c4full*   flash decoding over full K/V reconstructed from the same latents
and  c4q8k*   the latent decode over int8 caches with per-position scales,
     c4rk*    the latent decode with keys reconstructed on the tensor cores and
              rotated (rotary base 10000), ctx 4K/16K/32K,
     c4app    the latent producer writing one token's per-head latents.

`--impl reference` times the CPU oracle (the float64 reference
implementation) on the headline workload instead, on the host cores.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode-layer µs & achieved HBM GB/s (% of B200 roofline) at batch 1; tokens/s"
LAYERS, HIDDEN = 32, 4096
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
TC_MIN = [4, 1]   # smallest batch on the tensor-core path (linears, FFN): the library's defaults
ROW_IDS = ("c1", "c2b4", "c2b16", "c2dense", "c3b1", "c3b8", "c3b32", "c3dense", "c4k4", "c4k16", "c4k32",
           "c4rk4", "c4rk16", "c4rk32", "c4app", "c4full4", "c4full16", "c4full32", "c4q8k4", "c4q8k16", "c4q8k32",
           "c5")


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true", help="headline only (no per-configuration rows)")
    ap.add_argument("--only", default="", help="comma list of row ids to run (" + ",".join(ROW_IDS) + ")")
    ap.add_argument("--layers", type=int, default=LAYERS,
                    help="layers in the stack (default 32; fewer only for profiling small cases)")
    ap.add_argument("--tc-min-batch", default="",
                    help="LINEAR,FFN: smallest batch on the tensor-core path (lr_set_tensor_core_min_batch)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# distributed plumbing (timing only: no data-path collective)
# ---------------------------------------------------------------------------
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def dist_init(backend: str):
    import datetime

    import torch.distributed as dist
    rank, _, world = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=120))
    return world


def reduce_max(value: float, device=None) -> float:
    """Max of a per-rank float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_throughput(world: int, batch: int, ms_step_max: float) -> float:
    """Tokens/s of the whole job: every rank decodes `batch` tokens per step
    (independent replicas, no data-path collective), and the step time is the
    slowest rank's."""
    return world * batch / (ms_step_max * 1e-3)


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------
# peaks, DRAM traffic records
# ---------------------------------------------------------------------------
def measured_peaks() -> dict:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except (OSError, ValueError):
        return {}


def hbm_peak():
    p = measured_peaks()
    if "hbm_gbs" in p:
        return float(p["hbm_gbs"]), "of measured"
    return FALLBACK_HBM_GBS, "of fallback"


def int8_peak_tops():
    """int8 dense tensor peak: the measured bf16 burst figure times the nominal int8/bf16 ratio (2)."""
    p = measured_peaks()
    if "bf16_tflops" in p:
        return 2.0 * float(p["bf16_tflops"]), "of measured bf16 burst x 2 (nominal int8/bf16 ratio)"
    return 2.0 * FALLBACK_BF16_TFLOPS, "of fallback bf16 x 2 (nominal int8/bf16 ratio)"


# DRAM bytes (read + write) per algorithmic byte, from one ncu capture of the
# kernel named, valid only while its sources hash to the recorded value (the
# figure is dropped, as null, as soon as the kernel changes).  Filled from
# the profiles of the current sources.
TRAFFIC_RECORDS = {
    # ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch of the first 2 layers of the
    # stack (bench.py --layers 2; median of 3 launches): 160,054,784 bytes for 159,481,856 algorithmic bytes
    "chain_kernel<bf16,1,1>": {"sources_sha1": "400999462a321c4881a8610ba98da80fb1b2b09d", "per_alg_byte": 160054784 / 159481856},
}
KERNEL_SOURCES = {"chain_kernel<bf16,1,1>": ("chain.cu", "common.cuh")}


def sources_sha1(files) -> str:
    h = hashlib.sha1()
    for name in files:
        with open(os.path.join(ROOT, "decode_lr_linear_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic_for(kernel: str, alg_bytes: float):
    rec = TRAFFIC_RECORDS.get(kernel)
    if not rec or rec["sources_sha1"] != sources_sha1(KERNEL_SOURCES[kernel]):
        return None
    return round(rec["per_alg_byte"] * alg_bytes)


class ClockSampler:
    """nvidia-smi clock/throttle sampling while the GPU runs the timed work."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.proc, self.out = index, None, None

    def start(self):
        try:
            self.out = open(f"/tmp/lr_clocks_{os.getpid()}.csv", "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "50", "-i", str(self.index)], stdout=self.out,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def wait_first_sample(self, limit_s: float = 5.0):
        """Return once nvidia-smi has written a sample (its start-up takes a while)."""
        if self.proc is None:
            return
        t0 = time.time()
        while time.time() - t0 < limit_s:
            self.out.flush()
            if os.path.getsize(self.out.name) > 0:
                return
            time.sleep(0.02)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.out.name) as f:
            for line in f:
                p = [c.strip() for c in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
        os.unlink(self.out.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------
def time_graph(fn, iters: int, warmup: int = 3) -> float:
    """Mean ms per call of fn(i): `iters` calls captured in one CUDA graph (no
    host time between launches), replayed once after warm-up, CUDA events on
    the replay stream."""
    import torch
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(iters):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / iters


def time_e2e(step, iters: int, warmup: int = 3) -> float:
    """Mean ms per step of step(): each step copies its inputs from pinned host
    memory, calls the C ABI entry point, copies the result back to pinned host
    memory and waits for it on the host.  CUDA events around all steps."""
    import torch
    s = torch.cuda.current_stream()
    for _ in range(warmup):
        step()
        s.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        step()
        s.synchronize()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters


def cpu_timed(fn, budget_s: float, max_calls: int = 1000):
    """Calls fn() until budget_s of host time is spent (at least once); returns (s per call, calls)."""
    n, t = 0, 0.0
    while (t < budget_s or n == 0) and n < max_calls:
        t0 = time.perf_counter()
        fn()
        t += time.perf_counter() - t0
        n += 1
    return t / n, n


def check_device(lr) -> None:
    err = lr.lr_check_device_error()
    if err != 0:
        raise SystemExit(f"a kernel gave up a bounded wait during the timed work (device error {err}); "
                         "no number is reported")


def stream_ptr() -> int:
    import torch
    return torch.cuda.current_stream().cuda_stream


# ---------------------------------------------------------------------------
# headline workload
# ---------------------------------------------------------------------------
def algorithmic_bytes_per_step(ranks, batch: int, layers: int) -> int:
    """Factor bytes (bf16) of all the layers' projections plus activation reads/writes."""
    factor = int(sum(int(r) * (HIDDEN + HIDDEN) * 2 for r in ranks[:layers].reshape(-1)))
    act = layers * batch * HIDDEN * 2 * (2 + 4)  # reads: x (shared by Q/K/V), v; writes: q, k, v, o
    return factor + act


def build_layers(device, layers: int):
    from decode_lr_linear_b200 import synth
    import decode_lr_linear_b200 as lr
    ranks = synth.attention_ranks(0)
    out = []
    for l in range(layers):
        L = synth.make_attention_layer(l, ranks, seed=0)
        out.append({n: lr.Factor(L[n]["At"].to(device), L[n]["B"].to(device)) for n in synth.ATTN_PROJ})
    return ranks, out


def stack_steps(lr, layers, batch, device, split_v: bool = False):
    """The decode stack as one chain: per layer Q/K/V in one step (input: the previous O), then O
    (input: V).  split_v: three steps per layer instead, V, then Q and K, then O (reads V), so O waits
    only for V; measured slower on B200 (0.97 against 0.80 ms per step at batch 1: the third step's
    input round trip and latent hand-off cost more than the wait it hides), kept for comparison."""
    import torch

    def out():
        return torch.empty(batch, HIDDEN, dtype=torch.bfloat16, device=device)
    steps = []
    for l, L in enumerate(layers):
        if split_v:
            src = -1 if l == 0 else 3 * l - 1
            steps.append(lr.ChainStep([L["v"]], src, 0, [out()]))
            steps.append(lr.ChainStep([L["q"], L["k"]], src, 0, [out(), out()]))
            steps.append(lr.ChainStep([L["o"]], 3 * l, 0, [out()]))
        else:
            steps.append(lr.ChainStep([L["q"], L["k"], L["v"]], -1 if l == 0 else 2 * l - 1, 0,
                                      [out(), out(), out()]))
            steps.append(lr.ChainStep([L["o"]], 2 * l, 2, [out()]))
    return steps


def oracle_layer(L, x):
    """The CPU oracle on one layer of the chain: Q, K, V from x; O from V."""
    from oracle import lowrank
    outs = {n: lowrank.lr_linear(x, L[n]["At"].double().numpy().T, L[n]["B"].double().numpy())
            for n in ("q", "k", "v")}
    return lowrank.lr_linear(outs["v"], L["o"]["At"].double().numpy().T, L["o"]["B"].double().numpy())


def cpu_baseline_stack(batch: int, budget_s: float, layers_in_sample: int = 2) -> dict:
    """The oracle as it stands, timed on the host cores over a bounded sample
    of the stack (whole passes over the first layers), scaled to 32 layers."""
    from decode_lr_linear_b200 import synth
    ranks = synth.attention_ranks(0)
    cpu = [synth.make_attention_layer(l, ranks, seed=0) for l in range(layers_in_sample)]
    x = synth.make_activations(batch, HIDDEN, seed=0, key=(90,)).double().numpy()

    def one_pass():
        y = x
        for L in cpu:
            y = oracle_layer(L, y)

    per_pass, n = cpu_timed(one_pass, budget_s, 64)
    per_step = per_pass / layers_in_sample * LAYERS
    return {"value": batch / per_step, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
            "sample": f"{n} pass(es) over layers 0..{layers_in_sample - 1} of the 32-layer stack at batch {batch} "
                      f"(float64 numpy, {per_pass * n:.1f} s), scaled to 32 layers"}


def headline_config(world: int, batch: int, ranks) -> dict:
    return {"workload": "llama7b-lowrank-qkvo-decode", "layers": LAYERS, "hidden": HIDDEN, "batch": batch,
            "ranks": f"seeded non-uniform in [512,1536], mean {float(ranks.mean()):.2f}, 40% reduction",
            "l2": "inputs larger than L2 (2.58 GB of factors streamed per step)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def run_ours(args) -> None:
    global LAYERS
    LAYERS = args.layers
    import torch

    import decode_lr_linear_b200 as lr
    from decode_lr_linear_b200 import _lib as L
    from decode_lr_linear_b200 import synth

    rank, local, world = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init("nccl")
    batch = args.batch
    if args.tc_min_batch:
        lin, ffn = (int(v) for v in args.tc_min_batch.split(","))
        lr.lr_set_tensor_core_min_batch(lin, ffn)
        TC_MIN[0], TC_MIN[1] = lin or 4, ffn or 1
    only = set(filter(None, args.only.split(",")))
    want_headline = not only or "headline" in only
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline

    ranks, layers = build_layers(device, LAYERS)
    out = None
    if want_headline:
        x0 = synth.make_activations(batch, HIDDEN, seed=0, key=(90,)).to(device)
        steps = stack_steps(lr, layers, batch, device)
        ws = lr.workspace(lr.lr_linear_chain_workspace_size(steps, batch), device)

        def step():
            lr.lr_linear_chain(steps, x0, ws=ws)

        launches_per_step = (batch + 7) // 8
        step()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        torch.cuda.synchronize()

        clocks = ClockSampler(device.index).start()
        clocks.wait_first_sample()
        for _ in range(args.warmup):
            g.replay()
        torch.cuda.synchronize()
        barrier(device)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        barrier(device)
        torch.cuda.synchronize()
        ms_total = e0.elapsed_time(e1)
        # a short timed region gets no clock sample of its own: keep the same
        # load running (untimed) until the sampler has seen it for 0.3 s
        t_extra = time.time()
        while ms_total < 300.0 and time.time() - t_extra < 0.3:
            for _ in range(50):
                g.replay()
            torch.cuda.synchronize()
        clk = clocks.stop()
        if ms_total < 300.0:
            clk["window"] = "timed region plus untimed replays of the same step up to 0.3 s"
        check_device(lr)
        ms_step = reduce_max(ms_total, device) / args.steps

        # end to end through the C ABI: each step copies x from pinned host
        # memory, calls lr_linear_chain (descriptors prepared once, as a caller
        # keeps them), and copies the last layer's output back to the host
        x_host = synth.make_activations(batch, HIDDEN, seed=0, key=(90,)).pin_memory()
        y_host = torch.empty(batch, HIDDEN, dtype=torch.bfloat16).pin_memory()
        arr = lr.ops._chain_array(steps)
        lib = L.load()
        nbytes = ws.numel()
        y_last = steps[-1].ys[0]

        def e2e_step():
            x0.copy_(x_host, non_blocking=True)
            L.check("lr_linear_chain", lib.lr_linear_chain(arr, len(steps), x0.data_ptr(), batch, ws.data_ptr(),
                                                           nbytes, stream_ptr()))
            y_host.copy_(y_last, non_blocking=True)

        barrier(device)
        ms_e2e = reduce_max(time_e2e(e2e_step, max(3, min(args.steps, 200))), device)
        check_device(lr)
        del g

        bytes_step = algorithmic_bytes_per_step(ranks, batch, LAYERS)
        peak, peak_kind = hbm_peak()
        achieved = bytes_step / (ms_step * 1e-3) / 1e9
        out = {
            "metric": METRIC, "value": whole_job_throughput(world, batch, ms_step), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": headline_config(world, batch, ranks),
            "layer_us": ms_step * 1e3 / LAYERS,
            "hbm_gbs": achieved,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": traffic_for("chain_kernel<bf16,1,1>", bytes_step) if batch == 1 else None,
                         "peak_source": peak_kind,
                         "kernel": "chain_kernel<bf16, batch 1> (the decode engine)",
                         "algorithmic_bytes": bytes_step,
                         "note": "the step is one launch of this kernel per 8 batch rows, so its launch duration "
                                 "is the event-timed step time"},
            "gpu_launches": launches_per_step * args.steps,
            "e2e": {"value": whole_job_throughput(world, batch, ms_e2e), "unit": "tokens/s",
                    "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
                    "d2h_bytes_per_step": int(y_host.numel() * y_host.element_size()),
                    "path": "lr_linear_chain through the C ABI every step, pinned host x in, last output out"},
            "clocks": clk,
        }
        if want_cpu:
            out["cpu_baseline"] = cpu_baseline_stack(batch, 12.0)
        del steps, ws

    if rank == 0 and world == 1 and not args.no_rows:
        rows = run_rows(args, lr, L, synth, device, ranks, layers, only)
        dense = [r for r in rows if r["row"] == "c2dense"]
        if out is not None and dense:
            out["speedup_vs_uncompressed"] = out["value"] / dense[0]["value"]
        if out is None:
            for r in rows:
                print(json.dumps(r), flush=True)
            return
        out["rows"] = rows
    if rank == 0 and out is not None:
        print(json.dumps(out), flush=True)


# ---------------------------------------------------------------------------
# rows: every configuration of the path at N = 1
# ---------------------------------------------------------------------------
def _roof_hbm(alg_bytes: float, ms: float, note: str = "") -> dict:
    peak, kind = hbm_peak()
    gbs = alg_bytes / (ms * 1e-3) / 1e9
    r = {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak, "peak_source": kind,
         "algorithmic_bytes": int(alg_bytes), "traffic": None}
    if note:
        r["note"] = note
    return r


def row_c1(lr, L, synth, device, want_cpu):
    import torch
    from oracle import lowrank
    d = synth.make_single_linear(0)
    f = lr.Factor(d["At"].to(device), d["B32"].to(device))
    x = d["x"].to(device)
    y = torch.empty(1, 256, dtype=torch.float32, device=device)
    ws = lr.workspace(lr.lr_linear_workspace_size(f, 1), device)
    ms = time_graph(lambda i: lr.lr_linear(f, x, y, ws), 200)
    alg = (32 * 256 * 2 + 256 + 256) * 4
    lib, desc = L.load(), f.desc()
    xh, yh = d["x"].pin_memory(), torch.empty(1, 256, dtype=torch.float32).pin_memory()

    def e2e():
        x.copy_(xh, non_blocking=True)
        L.check("lr_linear", lib.lr_linear(ctypes.byref(desc), x.data_ptr(), None, 1, y.data_ptr(), ws.data_ptr(),
                                           ws.numel(), stream_ptr()))
        yh.copy_(y, non_blocking=True)
    ms_e2e = time_e2e(e2e, 200)
    row = {"row": "c1", "workload": "single low-rank linear, fp32, d_in = d_out = 256, rank 32, 1 token "
                                    "(Haar U, V; sigma_i = i^-1/2)",
           "value": ms * 1e3, "unit": "µs per call", "higher_is_better": False, "launches": 1,
           "roofline": dict(_roof_hbm(alg, ms, "66 KB that stay in L2: launch-latency bound, no roofline target"),
                            bound="latency"),
           "e2e": {"value": ms_e2e * 1e3, "unit": "µs per call", "h2d_bytes_per_step": 1024,
                   "d2h_bytes_per_step": 1024, "path": "lr_linear through the C ABI"},
           "l2": "all inputs fit L2 (the configuration is the latency case)"}
    if want_cpu:
        xd = d["x"].double().numpy()
        At, B = d["At"].double().numpy().T, d["B32"].double().numpy()
        s, n = cpu_timed(lambda: lowrank.lr_linear(xd, At, B), 1.0)
        row["cpu_baseline"] = {"value": s * 1e6, "unit": "µs per call", "cores": host_cores(), "kind": "oracle",
                               "sample": f"{n} calls of the float64 oracle on the same inputs"}
    return row


def row_c2(lr, L, synth, device, ranks, layers, batch, want_cpu):
    import torch
    steps = stack_steps(lr, layers, batch, device)
    ws = lr.workspace(lr.lr_linear_chain_workspace_size(steps, batch), device)
    x0 = synth.make_activations(batch, HIDDEN, seed=0, key=(90, batch)).to(device)
    ms = time_graph(lambda i: lr.lr_linear_chain(steps, x0, ws=ws), 20)
    alg = algorithmic_bytes_per_step(ranks, batch, LAYERS)
    passes = (batch + 31) // 32
    tensor_cores = batch >= TC_MIN[0]
    launches = passes * (2 * len(steps) + 1) if tensor_cores else (batch + 7) // 8
    note = (f"{launches} launches per step: per dependent step two tcgen05 products (z = x A, y = z B, weights "
            f"as M, tokens as N; the first also finalizes the step before), one finalize at the end; every "
            f"factor byte streamed once per pass of 32 tokens"
            if tensor_cores else f"{launches} launch(es) of chain_kernel per step; each streams every factor byte once")
    arr, lib = lr.ops._chain_array(steps), L.load()
    xh = synth.make_activations(batch, HIDDEN, seed=0, key=(90, batch)).pin_memory()
    yh = torch.empty(batch, HIDDEN, dtype=torch.bfloat16).pin_memory()

    def e2e():
        x0.copy_(xh, non_blocking=True)
        L.check("lr_linear_chain", lib.lr_linear_chain(arr, len(steps), x0.data_ptr(), batch, ws.data_ptr(),
                                                       ws.numel(), stream_ptr()))
        yh.copy_(steps[-1].ys[0], non_blocking=True)
    ms_e2e = time_e2e(e2e, 20)
    row = {"row": f"c2b{batch}", "workload": f"llama7b-lowrank-qkvo-decode, 32 layers, batch {batch}",
           "value": batch / (ms * 1e-3), "unit": "tokens/s", "higher_is_better": True,
           "ms_per_step": ms, "layer_us": ms * 1e3 / LAYERS, "launches": launches,
           "roofline": _roof_hbm(alg, ms, note),
           "e2e": {"value": batch / (ms_e2e * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": batch * HIDDEN * 2,
                   "d2h_bytes_per_step": batch * HIDDEN * 2, "path": "lr_linear_chain through the C ABI"},
           "l2": "2.58 GB of factors streamed per step"}
    if want_cpu:
        row["cpu_baseline"] = cpu_baseline_stack(batch, 3.0, 1)
    return row


def row_c3(lr, L, synth, device, d, batch, want_cpu):
    import torch
    from oracle import ffn as offn
    copies = 4

    def g(t):
        return t.to(device)
    ffns = [lr.FfnWeights(d["hidden"], d["inter"], d["n_lr"], d["rank"], g(d["A_q"]), g(d["s_A"]), g(d["B_q"]),
                          g(d["s_B"]), g(d["D_q"]), g(d["s_D"]), g(d["Wd_q"]), g(d["s_d"])) for _ in range(copies)]
    w_bytes = sum(int(d[k].numel() * d[k].element_size()) for k in ("A_q", "s_A", "B_q", "s_B", "D_q", "s_D",
                                                                  "Wd_q", "s_d"))
    xc = synth.make_activations(batch, d["hidden"], seed=0, key=(30, batch), outliers=4)
    x = xc.to(device)
    y = torch.empty_like(x)
    ws = lr.workspace(lr.lr_swiglu_ffn_workspace_size(ffns[0], batch), device)
    ms = time_graph(lambda i: lr.lr_swiglu_ffn(ffns[i % copies], x, y, ws), 40)
    alg = w_bytes + 2 * batch * d["hidden"] * 2
    lib, desc = L.load(), ffns[0].desc()
    xh, yh = xc.pin_memory(), torch.empty(batch, d["hidden"], dtype=torch.bfloat16).pin_memory()

    def e2e():
        x.copy_(xh, non_blocking=True)
        L.check("lr_swiglu_ffn", lib.lr_swiglu_ffn(ctypes.byref(desc), x.data_ptr(), batch, y.data_ptr(),
                                                   ws.data_ptr(), ws.numel(), stream_ptr()))
        yh.copy_(y, non_blocking=True)
    ms_e2e = time_e2e(e2e, 40)
    if batch >= TC_MIN[1]:
        passes = math.ceil(batch / 32)
        fused = batch <= 4   # the down projection evaluates the SwiGLU while it stages h
        pieces = passes * ((4 if d["n_lr"] > 0 else 3) + (0 if fused else 1))
        note = (f"{pieces} launches: tcgen05 kind::i8 products (x A' with x D, B'^T z, W_down^T h), "
                + ("the SwiGLU evaluated while h is staged" if fused else "a SwiGLU kernel")
                + ", finalize; every weight byte streamed once per pass of 32 tokens")
    else:
        pieces = math.ceil(batch / 2) + math.ceil(batch / 4)
        note = f"{pieces} launch(es) of the CUDA-core decode engine, each streaming its phase's weight bytes"
    row = {"row": f"c3b{batch}", "workload": f"hybrid int8 SwiGLU FFN, 7B shapes (hidden 4096, inter 11008, "
                                             f"n_lr 8192, rank 1536), batch {batch}",
           "value": ms * 1e3, "unit": "µs per layer", "higher_is_better": False,
           "tokens_s_32_layers": batch / (ms * 1e-3 * 32), "launches": pieces,
           "roofline": _roof_hbm(alg, ms, note),
           "e2e": {"value": ms_e2e * 1e3, "unit": "µs per layer", "h2d_bytes_per_step": batch * d["hidden"] * 2,
                   "d2h_bytes_per_step": batch * d["hidden"] * 2, "path": "lr_swiglu_ffn through the C ABI"},
           "l2": f"{copies} weight copies rotate ({copies * w_bytes / 1e6:.0f} MB > L2)"}
    if want_cpu:
        x64 = xc.double().numpy()
        s, n = cpu_timed(lambda: offn.hybrid_swiglu_ffn(x64, d["A_q"], d["s_A"], d["B_q"], d["s_B"], d["D_q"],
                                                        d["s_D"], d["Wd_q"], d["s_d"], d["n_lr"], d["n_dense"]),
                         3.0, 20)
        row["cpu_baseline"] = {"value": s * 1e6, "unit": "µs per layer", "cores": host_cores(), "kind": "oracle",
                               "sample": f"{n} call(s) of the float64 oracle on the same layer and batch"}
    del ffns, ws
    return row


def row_c4(lr, L, synth, device, ctx, want_cpu, rope_base: float = 0.0):
    """Latent-KV decode, batch 8, 32 heads, rank 32: the absorbed form, or (rope_base > 0) keys
    reconstructed on the tensor cores and rotated (LR_KV_RECONSTRUCT)."""
    import torch
    from oracle import latent_kv as okv
    kvd = synth.make_latent_kv(batch=8, heads=32, ctx=ctx, seed=0)
    cache_bytes = int(kvd["C_K"].numel() * 2 * 2)
    copies = max(1, math.ceil(4 * 126e6 / cache_bytes)) if cache_bytes < 4 * 126e6 else 1
    rec = rope_base > 0
    kv = lr.LatentKv(8, 32, ctx, kvd["B_K"].to(device), kvd["B_V"].to(device), kvd["scale"],
                     L.LR_KV_RECONSTRUCT if rec else L.LR_KV_ABSORBED, 0, rope_base)
    caches = [(kvd["C_K"].to(device), kvd["C_V"].to(device)) for _ in range(copies)]
    q, sl = kvd["q"].to(device), kvd["seq_lens"].to(device)
    o = torch.empty(8, 32, 128, dtype=torch.bfloat16, device=device)
    ws = lr.workspace(lr.lr_latent_kv_workspace_size(kv), device)
    ms = time_graph(lambda i: lr.lr_latent_kv_decode(kv, q, caches[i % copies][0], caches[i % copies][1], sl, o, ws),
                    40)
    alg = cache_bytes + int(kvd["B_K"].numel() * 2 * 2) + 2 * q.numel() * 2
    lib, desc = L.load(), kv.desc()
    qh, oh = kvd["q"].pin_memory(), torch.empty(8, 32, 128, dtype=torch.bfloat16).pin_memory()
    CK, CV = caches[0]

    def e2e():
        q.copy_(qh, non_blocking=True)
        L.check("lr_latent_kv_decode", lib.lr_latent_kv_decode(ctypes.byref(desc), q.data_ptr(), CK.data_ptr(),
                                                               CV.data_ptr(), sl.data_ptr(), o.data_ptr(),
                                                               ws.data_ptr(), ws.numel(), stream_ptr()))
        oh.copy_(o, non_blocking=True)
    ms_e2e = time_e2e(e2e, 40)
    form = (f"keys reconstructed on the tensor cores, rotary base {rope_base:g}" if rec else "absorbed form")
    row = {"row": f"c4{'r' if rec else ''}k{ctx // 1024}",
           "workload": f"per-head latent-KV flash decoding, batch 8, 32 heads, head_dim 128, rank 32, ctx {ctx} "
                       f"({form})",
           "value": ms * 1e3, "unit": "µs per call", "higher_is_better": False,
           "tokens_s_32_layers": 8 / (ms * 1e-3 * 32), "launches": 2 if rec else 3,
           "roofline": _roof_hbm(alg, ms, ("reconstruct-and-rotate split kernel (dominant) + combine kernel" if rec
                                           else "q projection + split kernel (dominant) + combine kernel")),
           "e2e": {"value": ms_e2e * 1e3, "unit": "µs per call", "h2d_bytes_per_step": int(q.numel() * 2),
                   "d2h_bytes_per_step": int(o.numel() * 2),
                   "path": "lr_latent_kv_decode through the C ABI (the caches stay resident, as a KV cache does)"},
           "l2": f"{copies} cache cop{'y' if copies == 1 else 'ies'} ({copies * cache_bytes / 1e6:.0f} MB > L2)"}
    if want_cpu:
        pairs = [(b, h) for b in range(0, 8, 2) for h in (0, 17)]
        if rec:
            s, n = cpu_timed(lambda: okv.latent_kv_decode_rope(kvd["q"], kvd["C_K"], kvd["C_V"], kvd["B_K"],
                                                               kvd["B_V"], kvd["seq_lens"], kvd["scale"], rope_base,
                                                               pairs), 2.0, 10)
        else:
            s, n = cpu_timed(lambda: okv.latent_kv_decode(kvd["q"], kvd["C_K"], kvd["C_V"], kvd["B_K"], kvd["B_V"],
                                                          kvd["seq_lens"], kvd["scale"], pairs), 2.0, 10)
        row["cpu_baseline"] = {"value": s * 1e6 * 256 / len(pairs), "unit": "µs per call", "cores": host_cores(),
                               "kind": "oracle",
                               "sample": f"{n} call(s) of the float64 oracle on {len(pairs)} of the 256 (batch, head) "
                                         f"pairs, scaled to 256"}
    del caches, ws
    return row


def row_c5(lr, L, synth, device, want_cpu):
    import torch
    from oracle import w8a8 as ow8
    T = 2048
    shapes = synth.prefill_shapes()
    ranks = synth.prefill_ranks(0)
    projs, ops, xs = {}, 0, {}
    # distinct inputs of a layer: x (q, k, v), attention output (o), x_ffn (gate, up), h (down)
    src = {"q": 0, "k": 0, "v": 0, "o": 1, "gate": 2, "up": 2, "down": 3}
    for j, name in enumerate(synth.PREFILL_PROJ):
        d_in, d_out = shapes[name]
        r = int(ranks[0, j])
        pp = synth.make_prefill_projection(d_in, d_out, r, seed=0, key=(d_in, d_out, r))
        f = lr.Factor(pp["A_q"].to(device), pp["B_q"].to(device), pp["s_A"].to(device), pp["s_B"].to(device))
        if src[name] not in xs:
            xc = synth.make_activations(T, d_in, seed=0, key=(60, d_in, T, src[name]), outliers=max(1, d_in // 1000))
            xd = xc.to(device)
            xs[src[name]] = [xc, xd, *lr.lr_quantize_per_token(xd)]
        ws = lr.workspace(lr.lr_linear_workspace_size(f, T, w8a8=True), device)
        y = torch.empty(T, d_out, dtype=torch.bfloat16, device=device)
        projs[name] = (f, src[name], y, ws, pp)
        ops += 2 * T * r * (d_in + d_out)

    def gemms(_):
        for name, (f, s, y, ws, _) in projs.items():
            lr.lr_linear(f, xs[s][2], y, ws, x_scale=xs[s][3])

    def layer(_):
        for key, (xc, xd, xq, sx) in xs.items():
            lr.lr_quantize_per_token(xd, xq, sx)
        gemms(0)
    ms_gemm = time_graph(gemms, 10)
    ms = time_graph(layer, 10)
    tops = ops / (ms_gemm * 1e-3) / 1e12
    peak, kind = int8_peak_tops()
    host_x = {k: v[0].pin_memory() for k, v in xs.items()}
    host_y = {n: torch.empty_like(p[2], device="cpu").pin_memory() for n, p in projs.items()}

    def e2e():
        for k, (xc, xd, xq, sx) in xs.items():
            xd.copy_(host_x[k], non_blocking=True)
            lr.lr_quantize_per_token(xd, xq, sx)
        gemms(0)
        for n, p in projs.items():
            host_y[n].copy_(p[2], non_blocking=True)
    ms_e2e = time_e2e(e2e, 5, 1)
    h2d = sum(int(v.numel() * 2) for v in host_x.values())
    d2h = sum(int(v.numel() * 2) for v in host_y.values())
    row = {"row": "c5", "workload": "W8A8 prefill, one 13B layer (q, k, v, o, gate, up, down; ranks of layer 0), "
                                    "2048 tokens, int8 x int8 -> int32 on tcgen05",
           "value": ms * 1e3, "unit": "µs per layer", "higher_is_better": False,
           "tokens_s_40_layers": T / (ms * 1e-3 * 40), "launches": 4 + 7 * 3,
           "gemm_us_per_layer": ms_gemm * 1e3,
           "roofline": {"bound": "tensor", "achieved": tops, "peak": peak, "unit": "TOPS", "frac": tops / peak,
                        "peak_source": kind, "algorithmic_ops": ops, "traffic": None,
                        "note": "w8a8_gemm_kernel x2 + requant_kernel per projection (the 7 projections' GEMM time); "
                                "value adds the 4 per-token quantisations of the layer's inputs"},
           "e2e": {"value": ms_e2e * 1e3, "unit": "µs per layer", "h2d_bytes_per_step": h2d,
                   "d2h_bytes_per_step": d2h,
                   "path": "lr_quantize_per_token + lr_linear through the C ABI, bf16 inputs in, 7 outputs out"},
           "l2": f"{ops / 1e9:.0f} GOP per layer; operands re-read from L2 by the tile loop"}
    if want_cpu:
        f, s, y, ws, pp = projs["q"]
        xc = xs[s][0]

        def one():
            qx, sx = ow8.quantize_per_token(xc)
            ow8.w8a8_lr_linear(qx, sx, pp["A_q"], pp["s_A"], pp["B_q"], pp["s_B"])
        sec, n = cpu_timed(one, 3.0, 5)
        d_in, d_out = shapes["q"]
        q_ops = 2 * T * int(ranks[0, 0]) * (d_in + d_out)
        row["cpu_baseline"] = {"value": sec * 1e6 * ops / q_ops, "unit": "µs per layer", "cores": host_cores(),
                               "kind": "oracle",
                               "sample": f"{n} call(s) of the oracle's W8A8 pipeline (quantise + both integer "
                                         f"products + requant, float64 BLAS) on the q projection, scaled to the "
                                         f"layer by integer ops"}
    del projs, xs
    return row


def row_c2dense(lr, L, synth, device, want_cpu):
    """Dense bf16 Q/K/V/O stack (the uncompressed model's projections), 32 layers, batch 1."""
    import torch
    from oracle import lowrank
    gen = torch.Generator(device=device).manual_seed(0)
    Wqkv = [(torch.randn(3 * HIDDEN, HIDDEN, device=device, generator=gen) / 64).to(torch.bfloat16) for _ in range(LAYERS)]
    Wo = [(torch.randn(HIDDEN, HIDDEN, device=device, generator=gen) / 64).to(torch.bfloat16) for _ in range(LAYERS)]
    x0 = synth.make_activations(1, HIDDEN, seed=0, key=(90,)).to(device)
    qkv = [torch.empty(1, 3 * HIDDEN, dtype=torch.bfloat16, device=device) for _ in range(LAYERS)]
    outs = [torch.empty(1, HIDDEN, dtype=torch.bfloat16, device=device) for _ in range(LAYERS)]

    def step(_):
        x = x0
        for l in range(LAYERS):
            lr.lr_dense_linear(Wqkv[l], x, y=qkv[l])
            lr.lr_dense_linear(Wo[l], qkv[l][:, 2 * HIDDEN:], y=outs[l])
            x = outs[l]
    ms = time_graph(step, 5)
    alg = LAYERS * 4 * HIDDEN * HIDDEN * 2 + LAYERS * HIDDEN * 2 * 6
    lib = L.load()
    xh = synth.make_activations(1, HIDDEN, seed=0, key=(90,)).pin_memory()
    yh = torch.empty(1, HIDDEN, dtype=torch.bfloat16).pin_memory()

    def e2e():
        x0.copy_(xh, non_blocking=True)
        x = x0
        for l in range(LAYERS):
            L.check("lr_dense_linear", lib.lr_dense_linear(Wqkv[l].data_ptr(), L.LR_BF16, None, L.LR_F32, HIDDEN,
                                                           3 * HIDDEN, x.data_ptr(), 1, qkv[l].data_ptr(), stream_ptr()))
            v = qkv[l][:, 2 * HIDDEN:]
            L.check("lr_dense_linear", lib.lr_dense_linear(Wo[l].data_ptr(), L.LR_BF16, None, L.LR_F32, HIDDEN, HIDDEN,
                                                           v.data_ptr(), 1, outs[l].data_ptr(), stream_ptr()))
            x = outs[l]
        yh.copy_(outs[-1], non_blocking=True)
    ms_e2e = time_e2e(e2e, 10)
    row = {"row": "c2dense", "workload": "dense bf16 Q/K/V/O (4096 x 4096 each), 32 layers, batch 1 (the "
                                         "uncompressed baseline of the headline stack)",
           "value": 1 / (ms * 1e-3), "unit": "tokens/s", "higher_is_better": True, "ms_per_step": ms,
           "layer_us": ms * 1e3 / LAYERS, "launches": 2 * LAYERS,
           "roofline": _roof_hbm(alg, ms, "lr_dense_linear (dense dot rows), one launch for Q/K/V and one for O per "
                                          "layer"),
           "e2e": {"value": 1 / (ms_e2e * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": HIDDEN * 2,
                   "d2h_bytes_per_step": HIDDEN * 2, "path": "lr_dense_linear through the C ABI"},
           "l2": "4.3 GB of weights streamed per step"}
    if want_cpu:
        W1 = Wqkv[0].double().cpu().numpy()
        W2 = Wo[0].double().cpu().numpy()
        x64 = x0.double().cpu().numpy()
        sec, n = cpu_timed(lambda: lowrank.dense_linear(lowrank.dense_linear(x64, W1.T)[:, 2 * HIDDEN:], W2.T), 2.0)
        row["cpu_baseline"] = {"value": 1 / (sec * LAYERS), "unit": "tokens/s", "cores": host_cores(),
                               "kind": "oracle", "sample": f"{n} call(s) of the float64 oracle on one layer, scaled "
                                                          f"to 32 layers"}
    del Wqkv, Wo
    return row


def row_c4app(lr, L, synth, device, want_cpu):
    """The latent producer: one decode token of batch 8 writes its per-head key and value latents
    (32 heads, rank 32, hidden 4096) into the caches; weights of 32 layers rotate."""
    import torch
    from oracle import latent_kv as okv
    heads, rank, hidden, ctx, batch, layers = 32, 32, 4096, 4096, 8, 32
    pr = synth.make_latent_producer(heads, rank, hidden, seed=0)
    A = [pr["A_KV"].to(device) for _ in range(layers)]
    x = synth.make_activations(batch, hidden, seed=0, key=(42,)).to(device)
    pos = torch.full((batch,), ctx - 1, dtype=torch.int32, device=device)
    CK = torch.zeros(batch, heads, ctx, rank, dtype=torch.bfloat16, device=device)
    CV = torch.zeros_like(CK)
    kv = lr.LatentKv(batch, heads, ctx, torch.empty(heads, rank, 128, dtype=torch.bfloat16, device=device),
                     torch.empty(heads, rank, 128, dtype=torch.bfloat16, device=device), 128 ** -0.5)
    ws = lr.workspace(lr.lr_latent_kv_append_workspace_size(kv, hidden), device)
    ms = time_graph(lambda i: lr.lr_latent_kv_append(kv, A[i % layers], x, pos, CK, CV, ws), 64)
    alg = A[0].numel() * 2 + x.numel() * 2 + 2 * batch * heads * rank * 2
    lib, desc = L.load(), kv.desc()
    xh = x.cpu().pin_memory()
    ch = torch.empty(batch, heads, rank, dtype=torch.bfloat16).pin_memory()

    def e2e():
        x.copy_(xh, non_blocking=True)
        L.check("lr_latent_kv_append", lib.lr_latent_kv_append(ctypes.byref(desc), A[0].data_ptr(), hidden,
                                                               x.data_ptr(), pos.data_ptr(), CK.data_ptr(),
                                                               CV.data_ptr(), ws.data_ptr(), ws.numel(),
                                                               stream_ptr()))
        ch.copy_(CK[:, :, ctx - 1], non_blocking=True)
    ms_e2e = time_e2e(e2e, 40)
    row = {"row": "c4app", "workload": "latent producer: x [8, 4096] times the stacked per-head first factors "
                                       "[2 x 32 heads x rank 32, 4096] bf16, latents written into the caches",
           "value": ms * 1e3, "unit": "µs per call", "higher_is_better": False,
           "launches": 2,
           "roofline": _roof_hbm(alg, ms, "tcgen05 product (stacked first factors as M, tokens as N) + scatter into "
                                          "the caches"),
           "e2e": {"value": ms_e2e * 1e3, "unit": "µs per call", "h2d_bytes_per_step": int(x.numel() * 2),
                   "d2h_bytes_per_step": int(ch.numel() * 2), "path": "lr_latent_kv_append through the C ABI"},
           "l2": f"{layers} weight copies ({layers * A[0].numel() * 2 / 1e6:.0f} MB > L2)"}
    if want_cpu:
        xc, Ac = x.cpu(), pr["A_KV"]
        z = torch.zeros(batch, heads, 2, rank, dtype=torch.bfloat16)
        sec, n = cpu_timed(lambda: okv.append_latents(xc, Ac, heads, rank, z, z, [1] * batch), 2.0, 20)
        row["cpu_baseline"] = {"value": sec * 1e6, "unit": "µs per call", "cores": host_cores(), "kind": "oracle",
                               "sample": f"{n} call(s) of the float64 oracle (same weights and batch, 2-position "
                                         f"caches)"}
    del A, CK, CV, ws
    return row


def row_c4q8(lr, L, synth, device, ctx, want_cpu):
    """Latent-KV decode over int8 caches (one fp16 scale per position), batch 8, 32 heads, rank 32."""
    import torch
    from oracle import latent_kv as okv
    d = synth.make_latent_kv_int8(batch=8, heads=32, ctx=ctx, seed=0)
    cache_bytes = int(d["C_Kq"].numel() * 2 + d["s_K"].numel() * 2 * 2)
    copies = max(1, math.ceil(4 * 126e6 / cache_bytes)) if cache_bytes < 4 * 126e6 else 1
    kv = lr.LatentKv(8, 32, ctx, d["B_K"].to(device), d["B_V"].to(device), d["scale"])
    caches = [tuple(d[k].to(device) for k in ("C_Kq", "s_K", "C_Vq", "s_V")) for _ in range(copies)]
    q, sl = d["q"].to(device), d["seq_lens"].to(device)
    o = torch.empty(8, 32, 128, dtype=torch.bfloat16, device=device)
    ws = lr.workspace(lr.lr_latent_kv_workspace_size(kv), device)
    ms = time_graph(lambda i: lr.lr_latent_kv_decode_q8(kv, q, *caches[i % copies][:2], *caches[i % copies][2:], sl,
                                                        o, ws), 40)
    alg = cache_bytes + int(d["B_K"].numel() * 2 * 2) + 2 * q.numel() * 2
    lib, desc = L.load(), kv.desc(L.LR_F16)
    qh, oh = d["q"].pin_memory(), torch.empty(8, 32, 128, dtype=torch.bfloat16).pin_memory()
    CK, sK, CV, sV = caches[0]

    def e2e():
        q.copy_(qh, non_blocking=True)
        L.check("lr_latent_kv_decode_q8", lib.lr_latent_kv_decode_q8(
            ctypes.byref(desc), q.data_ptr(), CK.data_ptr(), sK.data_ptr(), CV.data_ptr(), sV.data_ptr(),
            sl.data_ptr(), o.data_ptr(), ws.data_ptr(), ws.numel(), stream_ptr()))
        oh.copy_(o, non_blocking=True)
    ms_e2e = time_e2e(e2e, 40)
    row = {"row": f"c4q8k{ctx // 1024}", "workload": f"latent-KV decode over int8 caches (fp16 scale per position), "
                                                    f"batch 8, 32 heads, head_dim 128, rank 32, ctx {ctx}",
           "value": ms * 1e3, "unit": "µs per call", "higher_is_better": False, "launches": 3,
           "roofline": _roof_hbm(alg, ms, "q projection + split kernel (dominant) + combine kernel"),
           "e2e": {"value": ms_e2e * 1e3, "unit": "µs per call", "h2d_bytes_per_step": int(q.numel() * 2),
                   "d2h_bytes_per_step": int(o.numel() * 2), "path": "lr_latent_kv_decode_q8 through the C ABI"},
           "l2": f"{copies} cache cop{'y' if copies == 1 else 'ies'} ({copies * cache_bytes / 1e6:.0f} MB > L2)"}
    if want_cpu:
        pairs = [(b, h) for b in range(0, 8, 2) for h in (0, 17)]
        sec, n = cpu_timed(lambda: okv.latent_kv_decode_q8(d["q"], d["C_Kq"], d["s_K"], d["C_Vq"], d["s_V"], d["B_K"],
                                                           d["B_V"], d["seq_lens"], d["scale"], pairs), 2.0, 10)
        row["cpu_baseline"] = {"value": sec * 1e6 * 256 / len(pairs), "unit": "µs per call", "cores": host_cores(),
                               "kind": "oracle", "sample": f"{n} call(s) of the float64 oracle on {len(pairs)} of "
                                                          f"the 256 (batch, head) pairs, scaled to 256"}
    del caches, ws
    return row


def row_c4full(lr, L, synth, device, ctx, want_cpu):
    """Flash decoding over full K/V reconstructed (bf16) from the latent caches of c4."""
    import torch
    from oracle import attention
    kvd = synth.make_latent_kv(batch=8, heads=32, ctx=ctx, seed=0)
    CK, CV = kvd["C_K"].to(device), kvd["C_V"].to(device)
    K = torch.einsum("bhtr,hrd->bhtd", CK.float(), kvd["B_K"].to(device).float()).to(torch.bfloat16).contiguous()
    V = torch.einsum("bhtr,hrd->bhtd", CV.float(), kvd["B_V"].to(device).float()).to(torch.bfloat16).contiguous()
    del CK, CV
    q, sl = kvd["q"].to(device), kvd["seq_lens"].to(device)
    o = torch.empty(8, 32, 128, dtype=torch.bfloat16, device=device)
    d = L.FlashDesc(8, 32, 128, ctx, float(kvd["scale"]), 0)
    n = ctypes.c_size_t(0)
    lib = L.load()
    L.check("ws", lib.lr_flash_decode_workspace_size(ctypes.byref(d), ctypes.byref(n)))
    ws = lr.workspace(n.value, device)
    ms = time_graph(lambda i: lr.lr_flash_decode(q, K, V, sl, kvd["scale"], o, ws), 20)
    alg = int(K.numel() * 2 * 2 + 2 * q.numel() * 2)
    qh, oh = kvd["q"].pin_memory(), torch.empty(8, 32, 128, dtype=torch.bfloat16).pin_memory()

    def e2e():
        q.copy_(qh, non_blocking=True)
        L.check("lr_flash_decode", lib.lr_flash_decode(ctypes.byref(d), q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                                       sl.data_ptr(), o.data_ptr(), ws.data_ptr(), ws.numel(),
                                                       stream_ptr()))
        oh.copy_(o, non_blocking=True)
    ms_e2e = time_e2e(e2e, 20)
    row = {"row": f"c4full{ctx // 1024}", "workload": f"flash decoding over full K/V (bf16, head_dim 128, "
                                                     f"reconstructed from the c4 latents), batch 8, 32 heads, ctx {ctx}",
           "value": ms * 1e3, "unit": "µs per call", "higher_is_better": False, "launches": 2,
           "roofline": _roof_hbm(alg, ms, "split kernel (dominant) + combine kernel"),
           "e2e": {"value": ms_e2e * 1e3, "unit": "µs per call", "h2d_bytes_per_step": int(q.numel() * 2),
                   "d2h_bytes_per_step": int(o.numel() * 2), "path": "lr_flash_decode through the C ABI"},
           "l2": f"{alg / 1e9:.2f} GB of K/V per call"}
    if want_cpu:
        pairs = [(b, h) for b in range(0, 8, 2) for h in (0, 17)]
        Kc, Vc = K.cpu(), V.cpu()
        sec, cnt = cpu_timed(lambda: attention.decode_attention(kvd["q"], Kc, Vc, kvd["seq_lens"], kvd["scale"], pairs),
                             2.0, 10)
        row["cpu_baseline"] = {"value": sec * 1e6 * 256 / len(pairs), "unit": "µs per call", "cores": host_cores(),
                               "kind": "oracle", "sample": f"{cnt} call(s) of the float64 oracle on {len(pairs)} of "
                                                          f"the 256 (batch, head) pairs, scaled to 256"}
    del K, V, ws
    return row


class _Nvtx:
    """An NVTX range around one row (visible in a profiler's timeline; free without one)."""

    def __init__(self, name):
        self.name = name

    def __enter__(self):
        import torch
        torch.cuda.nvtx.range_push(self.name)

    def __exit__(self, *exc):
        import torch
        torch.cuda.nvtx.range_pop()


def run_rows(args, lr, L, synth, device, ranks, layers, only) -> list:
    import torch
    want_cpu = not args.no_cpu_baseline
    sel = [r for r in ROW_IDS if not only or r in only]
    rows = []
    clocks = ClockSampler(device.index).start()
    clocks.wait_first_sample()
    for rid in sel:
        if rid.startswith("c2b"):
            with _Nvtx(rid):
                rows.append(row_c2(lr, L, synth, device, ranks, layers, int(rid[3:]), want_cpu))
    del layers
    torch.cuda.empty_cache()
    if "c1" in sel:
        rows.insert(0, row_c1(lr, L, synth, device, want_cpu))
    if "c2dense" in sel:
        with _Nvtx("c2dense"):
            rows.append(row_c2dense(lr, L, synth, device, want_cpu))
        torch.cuda.empty_cache()
    ffn = None
    for rid in sel:
        if rid.startswith("c3b"):
            ffn = ffn or synth.make_hybrid_ffn(seed=0)
            with _Nvtx(rid):
                rows.append(row_c3(lr, L, synth, device, ffn, int(rid[3:]), want_cpu))
            torch.cuda.empty_cache()
    if "c3dense" in sel:
        dense = synth.make_hybrid_ffn(seed=0, n_lr=0, rotate=False)
        r = row_c3(lr, L, synth, device, dense, 1, want_cpu)
        r["row"], r["workload"] = "c3dense", ("dense int8 SwiGLU FFN (all 11008 channels dense), 7B shapes, batch 1 "
                                              "(the uncompressed baseline of c3)")
        rows.append(r)
        del dense
        torch.cuda.empty_cache()
    for rid in sel:
        if rid.startswith("c4k"):
            with _Nvtx(rid):
                rows.append(row_c4(lr, L, synth, device, int(rid[3:]) * 1024, want_cpu))
            torch.cuda.empty_cache()
        elif rid.startswith("c4rk"):
            with _Nvtx(rid):
                rows.append(row_c4(lr, L, synth, device, int(rid[4:]) * 1024, want_cpu, rope_base=10000.0))
            torch.cuda.empty_cache()
        elif rid == "c4app":
            with _Nvtx("c4app"):
                rows.append(row_c4app(lr, L, synth, device, want_cpu))
            torch.cuda.empty_cache()
        elif rid.startswith("c4full"):
            with _Nvtx(rid):
                rows.append(row_c4full(lr, L, synth, device, int(rid[6:]) * 1024, want_cpu))
            torch.cuda.empty_cache()
        elif rid.startswith("c4q8k"):
            with _Nvtx(rid):
                rows.append(row_c4q8(lr, L, synth, device, int(rid[5:]) * 1024, want_cpu))
            torch.cuda.empty_cache()
    if "c5" in sel:
        with _Nvtx("c5"):
            rows.append(row_c5(lr, L, synth, device, want_cpu))
    clk = clocks.stop()
    check_device(lr)
    by = {r["row"]: r for r in rows}
    # speed-up of each low-rank row over its uncompressed baseline (same work, same units)
    for low, base in (("c3b1", "c3dense"), ("c4k4", "c4full4"), ("c4k16", "c4full16"), ("c4k32", "c4full32"),
                      ("c4rk4", "c4full4"), ("c4rk16", "c4full16"), ("c4rk32", "c4full32"),
                      ("c4q8k4", "c4full4"), ("c4q8k16", "c4full16"), ("c4q8k32", "c4full32")):
        if low in by and base in by:
            by[low]["speedup_vs_uncompressed"] = by[base]["value"] / by[low]["value"]
    for r in rows:
        r["clocks"] = clk
    return rows


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle
# ---------------------------------------------------------------------------
def run_reference(args) -> None:
    rank, _, world = dist_env()
    if rank != 0:
        return
    from decode_lr_linear_b200 import synth
    ranks = synth.attention_ranks(0)
    # each step: the oracle over a bounded sample of the stack (one layer, layers cycled), scaled to 32 layers
    cache = {}

    def layer(l):
        if l not in cache:
            cache.clear()
            cache[l] = synth.make_attention_layer(l, ranks, seed=0)
        return cache[l]

    x = synth.make_activations(args.batch, HIDDEN, seed=0, key=(90,)).double().numpy()
    for i in range(args.warmup):
        oracle_layer(layer(i % LAYERS), x)
    t = 0.0
    for i in range(args.steps):
        L = layer((args.warmup + i) % LAYERS)
        t0 = time.perf_counter()
        oracle_layer(L, x)
        t += time.perf_counter() - t0
    per_step = t / args.steps * LAYERS
    value = args.batch / per_step
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": headline_config(world, args.batch, ranks),
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
                            "sample": "each step: the float64 oracle over one layer's Q/K/V/O (layers cycled), "
                                      "scaled to 32 layers, so ms_per_step is 32 times the time each step ran"},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main(argv=None):
    args = parse(argv)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)
    try:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()
    except Exception:  # pragma: no cover
        pass


if __name__ == "__main__":
    main()
