#!/usr/bin/env python
"""Benchmark of the low-rank decode path on B200.

Workload (one "step"): one decode token through a LLaMA-7B-shaped stack of
32 layers whose Q/K/V/O projections are truncated-SVD factorised (bf16,
hidden 4096, seeded non-uniform ranks in [512, 1536] at 40 % parameter
reduction, batch 1).  Per layer: one grouped call computes Q, K, V from the
layer input x; the O projection reads the V output (single-token attention
returns V exactly) and its output is the next layer's input.  The
whole stack is one lr_linear_chain call: one launch per step, with one
grid-wide barrier per dependent projection inside it.

The 32 layers hold 2.58 GB of factors, far above the 126 MB L2, so every
step streams them from HBM (no L2 flush needed).  Timing: W untimed warm-up
steps, then exactly K steps of a captured CUDA graph of the step,
bracketed by a barrier and a device synchronisation, measured with CUDA
events, max over ranks.  With --gpus N > 1 (torchrun), every rank runs its
own replica of the workload on its own GPU (independent requests; weak
scaling, no data-path collective).

`--impl reference` times the CPU oracle (the float64 reference
implementation) on the same workload instead, on the host cores.
"""
from __future__ import annotations

import argparse
import json
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


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--secondary", action="store_true",
                    help="time the FFN, latent-KV and W8A8 rows instead (one JSON line each)")
    ap.add_argument("--layers", type=int, default=LAYERS,
                    help="layers in the stack (default 32; fewer only for profiling small cases)")
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
# workload
# ---------------------------------------------------------------------------
# DRAM bytes (read + write) per algorithmic byte of chain_kernel<bf16, batch 1>,
# from one ncu capture of the same kernel on the 2-layer case (163.92 MB of
# DRAM traffic for 159.48 MB of algorithmic bytes; summary and command in
# profiles/chain_kernel_bf16_b1_llama7b_2layers.md).  DRAM traffic grows with
# the factor bytes streamed, so a full launch's traffic is this ratio times its
# algorithmic bytes.  Valid for that kernel build and batch 1 only.
CHAIN_TRAFFIC_PER_ALG_BYTE = 163.92e6 / 159481856


def algorithmic_bytes_per_step(ranks, batch: int) -> int:
    """Factor bytes (bf16) of all 128 projections plus activation reads/writes."""
    factor = int(sum(int(r) * (HIDDEN + HIDDEN) * 2 for r in ranks[:LAYERS].reshape(-1)))
    act = LAYERS * batch * HIDDEN * 2 * (2 + 4)  # reads: x (shared by Q/K/V), v; writes: q, k, v, o
    return factor + act


def build_layers(device, keep_cpu: int = 0):
    from decode_lr_linear_b200 import synth
    import decode_lr_linear_b200 as lr
    ranks = synth.attention_ranks(0)
    layers, cpu = [], []
    for l in range(LAYERS):
        L = synth.make_attention_layer(l, ranks, seed=0)
        layers.append({n: lr.Factor(L[n]["At"].to(device), L[n]["B"].to(device)) for n in synth.ATTN_PROJ})
        if l < keep_cpu:
            cpu.append(L)
    return ranks, layers, cpu


def oracle_step(cpu_layers, x):
    """The CPU oracle on the same chain: Q, K, V from x; O from V; O's output feeds the next layer."""
    from oracle import lowrank
    for L in cpu_layers:
        outs = {}
        for n in ("q", "k", "v"):
            outs[n] = lowrank.lr_linear(x, L[n]["At"].double().numpy().T, L[n]["B"].double().numpy())
        x = lowrank.lr_linear(outs["v"], L["o"]["At"].double().numpy().T, L["o"]["B"].double().numpy())
    return x


def cpu_baseline(cpu_layers, batch: int, budget_s: float = 12.0) -> dict:
    """The oracle as it stands, timed on the host cores over a bounded sample of the workload."""
    from decode_lr_linear_b200 import synth
    x = synth.make_activations(batch, HIDDEN, seed=0, key=(90,)).double().numpy()
    n_done, t_total = 0, 0.0
    while t_total < budget_s and n_done < 64:
        t0 = time.perf_counter()
        oracle_step(cpu_layers, x)
        t_total += time.perf_counter() - t0
        n_done += 1
    per_layer = t_total / (n_done * len(cpu_layers))
    per_step = per_layer * LAYERS
    return {"value": batch / per_step, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
            "sample": f"{n_done} pass(es) over layers 0..{len(cpu_layers) - 1} of the 32-layer stack at batch "
                      f"{batch} (float64 numpy, {t_total:.1f} s), scaled to 32 layers"}


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""
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


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "of measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "of fallback"


def run_ours(args) -> None:
    global LAYERS
    LAYERS = args.layers
    import torch

    import decode_lr_linear_b200 as lr
    from decode_lr_linear_b200 import synth

    rank, local, world = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init("nccl")
    batch = args.batch
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    ranks, layers, cpu_layers = build_layers(device, keep_cpu=LAYERS if want_cpu else 0)

    x0 = synth.make_activations(batch, HIDDEN, seed=0, key=(90,)).to(device)
    qkv = [[torch.empty(batch, HIDDEN, dtype=torch.bfloat16, device=device) for _ in range(3)] for _ in range(LAYERS)]
    outs = [torch.empty(batch, HIDDEN, dtype=torch.bfloat16, device=device) for _ in range(LAYERS)]
    # the whole stack as one chain: step 2l = Q/K/V of layer l (input: the previous O), step 2l+1 = O (input: V)
    steps = []
    for l in range(LAYERS):
        L = layers[l]
        steps.append(lr.ChainStep([L["q"], L["k"], L["v"]], -1 if l == 0 else 2 * l - 1, 0, qkv[l]))
        steps.append(lr.ChainStep([L["o"]], 2 * l, 2, [outs[l]]))
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
    clk = clocks.stop()
    ms_total = reduce_max(e0.elapsed_time(e1), device)
    ms_step = ms_total / args.steps

    # end to end through the public API: pinned host input -> device, the step, result -> pinned host
    x_host = synth.make_activations(batch, HIDDEN, seed=0, key=(90,)).pin_memory()
    y_host = torch.empty(batch, HIDDEN, dtype=torch.bfloat16).pin_memory()
    ge = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ge):
        step()
    for _ in range(3):
        x0.copy_(x_host, non_blocking=True)
        ge.replay()
        y_host.copy_(outs[-1], non_blocking=True)
        torch.cuda.current_stream().synchronize()
    barrier(device)
    torch.cuda.synchronize()
    k_e2e = max(3, min(args.steps, 200))
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(k_e2e):
        x0.copy_(x_host, non_blocking=True)
        ge.replay()
        y_host.copy_(outs[-1], non_blocking=True)
        torch.cuda.current_stream().synchronize()
    f1.record()
    torch.cuda.synchronize()
    barrier(device)
    ms_e2e = reduce_max(f0.elapsed_time(f1), device) / k_e2e

    if rank != 0:
        return
    bytes_step = algorithmic_bytes_per_step(ranks, batch)
    peak, peak_kind = measured_hbm_peak()
    achieved = bytes_step / (ms_step * 1e-3) / 1e9
    tokens_s = whole_job_throughput(world, batch, ms_step)
    out = {
        "metric": METRIC, "value": tokens_s, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "llama7b-lowrank-qkvo-decode", "layers": LAYERS, "hidden": HIDDEN, "batch": batch,
                   "ranks": f"seeded non-uniform in [512,1536], mean {float(ranks.mean()):.2f}, 40% reduction",
                   "l2": "inputs larger than L2 (2.58 GB of factors streamed per step)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "layer_us": ms_step * 1e3 / LAYERS,
        "hbm_gbs": achieved,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": (round(CHAIN_TRAFFIC_PER_ALG_BYTE * bytes_step) if batch == 1 else None),
                     "traffic_note": "ncu dram__bytes_read.sum + dram__bytes_write.sum of a 2-layer launch, "
                                     "scaled by factor bytes to the full launch",
                     "peak_source": peak_kind,
                     "kernel": "chain_kernel<bf16, batch 1> (factorised-linear chain)",
                     "note": "the step is one launch of this kernel only, so its launch duration is the "
                             "event-timed step time"},
        "gpu_launches": launches_per_step * args.steps,
        "e2e": {"value": whole_job_throughput(world, batch, ms_e2e), "unit": "tokens/s",
                "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
                "d2h_bytes_per_step": int(y_host.numel() * y_host.element_size())},
        "clocks": clk,
    }
    if want_cpu:
        out["cpu_baseline"] = cpu_baseline(cpu_layers, batch)
    print(json.dumps(out), flush=True)


def run_reference(args) -> None:
    rank, _, world = dist_env()
    if rank != 0:
        return
    from decode_lr_linear_b200 import synth
    ranks = synth.attention_ranks(0)
    # each step: the oracle over a bounded sample of the stack (layers cycled), scaled to 32 layers
    per_step_layers = 1
    cache = {}

    def layer(l):
        if l not in cache:
            cache.clear()
            cache[l] = synth.make_attention_layer(l, ranks, seed=0)
        return cache[l]

    x = synth.make_activations(args.batch, HIDDEN, seed=0, key=(90,)).double().numpy()
    for i in range(args.warmup):
        oracle_step([layer(i % LAYERS)], x)
    t = 0.0
    for i in range(args.steps):
        L = layer((args.warmup + i) % LAYERS)
        t0 = time.perf_counter()
        oracle_step([L], x)
        t += time.perf_counter() - t0
    per_step = t / args.steps * LAYERS / per_step_layers
    value = args.batch / per_step
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": "llama7b-lowrank-qkvo-decode", "layers": LAYERS, "hidden": HIDDEN,
                      "batch": args.batch},
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
                            "sample": f"each step: the float64 oracle over one layer's Q/K/V/O (layers cycled), "
                                      f"scaled to 32 layers"},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def _time_rotating(fn, n_copies: int, iters: int, warmup: int = 3) -> float:
    """Mean ms per call of fn(i), copy i % n_copies: `iters` calls captured in
    one CUDA graph (no host time between launches), replayed after warm-up,
    timed with CUDA events on the replay stream."""
    import torch
    for i in range(warmup):
        fn(i % n_copies)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(iters):
            fn(i % n_copies)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / iters


def run_secondary(args) -> None:
    """One JSON line per further hot-path row, each against its own roofline:
    the hybrid int8 SwiGLU FFN (7B shapes, batch 1), latent-KV split-K decode
    (batch 8, 32 heads, rank 32, ctx 16384) and the W8A8 prefill projections
    of one 13B layer (2048 tokens).  Weight or cache copies rotate so the
    working set exceeds L2."""
    import torch

    import decode_lr_linear_b200 as lr
    from decode_lr_linear_b200 import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    hbm, hbm_kind = measured_hbm_peak()
    peaks = {}
    peaks_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(peaks_path):
        with open(peaks_path) as f:
            peaks = json.load(f)
    lines = []

    # ---- hybrid FFN (int8 weights + fp16 scales), 4 copies of one layer ----
    d = synth.make_hybrid_ffn(seed=0)

    def ffn_copy():
        g = lambda t: t.to(dev)
        return lr.FfnWeights(d["hidden"], d["inter"], d["n_lr"], d["rank"], g(d["A_q"]), g(d["s_A"]), g(d["B_q"]),
                             g(d["s_B"]), g(d["D_q"]), g(d["s_D"]), g(d["Wd_q"]), g(d["s_d"]))
    ffns = [ffn_copy() for _ in range(4)]
    w_bytes = sum(int(d[k].numel() * d[k].element_size()) for k in ("A_q", "s_A", "B_q", "s_B", "D_q", "s_D",
                                                                  "Wd_q", "s_d"))
    for batch in (1, 8):
        x = synth.make_activations(batch, d["hidden"], seed=0, key=(30, batch), outliers=4).to(dev)
        y = torch.empty_like(x)
        ws = lr.workspace(lr.lr_swiglu_ffn_workspace_size(ffns[0], batch), dev)
        ms = _time_rotating(lambda i: lr.lr_swiglu_ffn(ffns[i], x, y, ws), 4, 40)
        alg = w_bytes + 2 * batch * d["hidden"] * 2
        gbs = alg / (ms * 1e-3) / 1e9
        lines.append({"row": "a4-a7 hybrid int8 SwiGLU FFN", "workload": f"7B FFN (hidden 4096, inter 11008, "
                      f"n_lr 8192, rank 1536), batch {batch}", "us_per_layer": ms * 1e3,
                      "tokens_s_32_layers": batch / (ms * 1e-3 * 32),
                      "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                                   "peak_source": hbm_kind, "algorithmic_bytes": alg}})
    del ffns

    # ---- latent-KV split-K decode (absorbed), ctx 16384 ----
    kvd = synth.make_latent_kv(batch=8, heads=32, ctx=16384, seed=0)
    kv = lr.LatentKv(kvd["batch"], kvd["heads"], kvd["ctx"], kvd["B_K"].to(dev), kvd["B_V"].to(dev), kvd["scale"],
                     0, 0)
    q, CK, CV, sl = (kvd[k].to(dev) for k in ("q", "C_K", "C_V", "seq_lens"))
    out = torch.empty(kv.batch, kv.heads, kv.head_dim, dtype=torch.bfloat16, device=dev)
    kws = lr.workspace(lr.lr_latent_kv_workspace_size(kv), dev)
    ms = _time_rotating(lambda i: lr.lr_latent_kv_decode(kv, q, CK, CV, sl, out, kws), 1, 40)
    alg = int(CK.numel() * 2 + CV.numel() * 2 + kvd["B_K"].numel() * 2 + kvd["B_V"].numel() * 2)
    gbs = alg / (ms * 1e-3) / 1e9
    lines.append({"row": "a8-a10 latent-KV split-K decode", "workload": "batch 8, heads 32, rank 32, head_dim 128, "
                  "ctx 16384 (1.07 GB of latent cache, larger than L2)", "us": ms * 1e3,
                  "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                               "peak_source": hbm_kind, "algorithmic_bytes": alg}})
    del q, CK, CV, sl, kv, kvd, out, kws

    # ---- W8A8 prefill: the 7 projections of one 13B layer, 2048 tokens ----
    T = 2048
    shapes = synth.prefill_shapes()
    ranks = synth.prefill_ranks(0)
    projs, ops = [], 0
    for j, name in enumerate(synth.PREFILL_PROJ):
        d_in, d_out = shapes[name]
        r = int(ranks[0, j])
        pp = synth.make_prefill_projection(d_in, d_out, r, seed=0, key=(d_in, d_out, r))
        f = lr.Factor(pp["A_q"].to(dev), pp["B_q"].to(dev), pp["s_A"].to(dev), pp["s_B"].to(dev))
        xin = synth.make_activations(T, d_in, seed=0, key=(60, d_in, T), outliers=max(1, d_in // 1000)).to(dev)
        xq, sx = lr.lr_quantize_per_token(xin)
        ws = lr.workspace(lr.lr_linear_workspace_size(f, T, w8a8=True), dev)
        y = torch.empty(T, d_out, dtype=torch.bfloat16, device=dev)
        projs.append((f, xq, sx, y, ws))
        ops += 2 * T * r * (d_in + d_out)

    def layer(_):
        for f, xq, sx, y, ws in projs:
            lr.lr_linear(f, xq, y, ws, x_scale=sx)
    ms = _time_rotating(layer, 1, 20)
    tops = ops / (ms * 1e-3) / 1e12
    bf16 = peaks.get("bf16_tflops")
    i8_peak = 2.0 * bf16 if bf16 else 2.0 * 1590.0
    lines.append({"row": "a11-a12 W8A8 prefill (tcgen05 int8)", "workload": "one 13B layer (q,k,v,o,gate,up,down; "
                  "ranks of layer 0), 2048 tokens, int8 x int8 -> int32", "us_per_layer": ms * 1e3,
                  "tokens_s_40_layers": T / (ms * 1e-3 * 40),
                  "roofline": {"bound": "tensor", "achieved": tops, "peak": i8_peak, "unit": "TOPS",
                               "frac": tops / i8_peak, "peak_source": ("of measured bf16 x 2 (nominal int8/bf16 "
                                                                       "ratio)" if bf16 else "of fallback x 2"),
                               "algorithmic_ops": ops}})
    for ln in lines:
        print(json.dumps(ln), flush=True)


def main(argv=None):
    args = parse(argv)
    if args.impl == "reference":
        run_reference(args)
    elif args.secondary:
        run_secondary(args)
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
