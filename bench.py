"""Benchmark of the fused FP8 routed-expert MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--config large|tiny|decode|prefill|skewed|decode_w4a8|prefill_w4a8]
                    [--impl reference] [--no-cpu-baseline] [--tokens T] [--shared-expert]
                    [--recipe 0|1|2] [--gate | --gate-only] [--no-graph]

One step = one moe_forward call (route, permute, quantize, gate+up GEMM with SwiGLU and
requantization, down GEMM, combine) over one batch of seeded synthetic inputs of the named
problem, inputs resident in HBM.  The default problem is the largest one that fits one GPU, the
large prefill with biases (16384 tokens, H 4096, I 1536, 128 experts, top-8, 4.95 TFLOP per step);
its 2.4 GB of FP8 weights exceed the 126 MB L2, so every step streams them from HBM (likewise
decode, prefill and the W4A8 problems).  The timed loop replays a CUDA graph of 10 steps (--no-graph:
host launches); the e2e figure copies each step's inputs in and its output out through pinned
host memory, on copy streams that overlap the neighbouring steps.  --gate starts every step from
the gate (moe_gate) instead of router logits; --gate-only times the gate alone.

Prints one JSON line (rank 0).  Multi-GPU runs (torchrun) are independent replicas, one per
GPU, with no collective on the data path ("scaling": "weak"); timing is the max over ranks.
`--impl reference` times the CPU oracle (test infrastructure, plain C) on host cores on a
bounded token sample of the same problem.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s & FP8 TFLOPS (% of tensor/HBM roofline), 1×B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0          # nominal dense FP8 / BF16 tensor ratio (4.5 / 2.25 PFLOP/s)
SMALL_ROWS = 2048             # the library permutes up to this many routed rows in one launch


def kernels_per_step(A: int) -> int:
    # route, permute (one kernel, or histogram + scan + scatter), quantize, gemm1, gemm2, combine
    return 6 if A <= SMALL_ROWS else 8


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def describe(shape: synth.Shape) -> str:
    rt = "sigmoid" if shape.routing else "softmax"
    extra = []
    if shape.group_count > 1:
        extra.append(f"groups {shape.group_count}/{shape.k_group} mode {shape.group_select_mode}")
    if shape.renormalize:
        extra.append("renorm")
    if shape.per_expert_scale:
        extra.append("per-expert scale")
    if shape.routed_scaling_factor != 1.0:
        extra.append(f"rsf {shape.routed_scaling_factor}")
    if shape.biases:
        extra.append("biases")
    rec = {0: "E4M3 + fp32 scale per (row,128)", 1: "MXFP8 (E4M3 + UE8M0 per 32)",
           2: "W4A8 (E2M1 weights + UE8M0 per 32, MXFP8 activations)"}[shape.recipe]
    return (f"{shape.name}: {shape.num_tokens} tok, H {shape.hidden}, I {shape.inter}, "
            f"E {shape.num_experts}, top-{shape.top_k}, {rt}" + (", " + ", ".join(extra) if extra else "")
            + (" + 1 shared expert" if shape.shared_experts else "")
            + f"; {rec}")


def workload_config(shape, active, world, gate=False):
    """The `config` object of the JSON line, the same for the native and the reference arm."""
    alg = algorithmic_bytes(shape, active)
    return {"workload": describe(shape) + ("; from bf16 hidden states through the fused gate "
                                           "(RMSNorm + router matmul + top-k)" if gate else ""),
            "tokens_per_step": shape.num_tokens, "active_experts": active,
            "parallelism": f"replicas x{world}",
            "l2": "no flush; the step streams the FP8 weights, larger than L2" if alg > 126e6
                  else "working set fits L2 (latency-bound)"}


def host_sample(prob, n, seed=7):
    """A host copy of the problem cut to n seeded tokens (every weight, the sampled rows of x and
    the logits): the oracle's input for the CPU baseline.  Valid as a sample of the whole batch
    because a row's output does not depend on the other rows."""
    T = prob.shape.num_tokens
    tok = np.sort(np.random.default_rng(seed).choice(T, n, replace=False))
    ti = torch.from_numpy(tok).to(prob.x.device)
    cpu = lambda t: None if t is None else t.cpu()
    return synth.Problem(prob.shape.with_tokens(n), prob.x[ti].cpu(), prob.logits[ti].cpu(),
                         cpu(prob.per_expert_scale), cpu(prob.w13), cpu(prob.w13_scale), cpu(prob.w2),
                         cpu(prob.w2_scale), cpu(prob.w13_bias), cpu(prob.w2_bias))


def time_cpu_oracle(shape, prob, n, budget_s, threads=None, max_reps=50):
    """Repeat the oracle on n tokens until budget_s seconds have passed: (tokens/s, seconds,
    runs, threads used)."""
    import oracle
    before = oracle.num_threads()
    done = tot = 0.0
    reps = 0
    try:
        while tot < budget_s and reps < max_reps:
            _, dt, cores = run_cpu_oracle(shape, prob, n, threads)
            tot += dt
            done += n
            reps += 1
    finally:
        if threads:
            oracle.set_num_threads(before)
    return done / tot, tot, reps, cores


def flops(shape, A):
    return 6.0 * A * shape.hidden * shape.inter


def scale_bytes(shape, K, N):
    return (K // 128) * N * 4 if shape.recipe == 0 else (K // 32) * N


def code_bytes(shape, K, N):
    """Bytes of a [K, N] weight matrix's codes: one E4M3 byte each, or two E2M1 codes a byte."""
    return K * N // 2 if shape.recipe == 2 else K * N


def algorithmic_bytes(shape, active):
    """Minimum HBM bytes of one forward: each active expert's weights and scales once, plus the
    per-call tensors (x, y, logits).  Intermediates excluded."""
    H, I, E, T = shape.hidden, shape.inter, shape.num_experts, shape.num_tokens
    w = active * (code_bytes(shape, H, 2 * I) + code_bytes(shape, I, H) + scale_bytes(shape, H, 2 * I)
                  + scale_bytes(shape, I, H))
    if shape.biases:
        w += active * 2 * (2 * I + H)
    return w + 2 * T * H * 2 + 4 * T * E


def gemm1_bytes(shape, active):
    """Algorithmic bytes of one gate+up launch: active experts' W13 codes + scales, the
    quantized activations read, the requantized SwiGLU products written."""
    H, I, T, k = shape.hidden, shape.inter, shape.num_tokens, shape.top_k + shape.shared_experts
    A = T * k
    g = 128 if shape.recipe == 0 else 32
    sb = 4 if shape.recipe == 0 else 1
    return (active * (code_bytes(shape, H, 2 * I) + scale_bytes(shape, H, 2 * I)) + A * H + A * (H // g) * sb
            + A * I + A * (I // g) * sb)


def gemm2_bytes(shape, active):
    H, I, T, k = shape.hidden, shape.inter, shape.num_tokens, shape.top_k + shape.shared_experts
    A = T * k
    g = 128 if shape.recipe == 0 else 32
    sb = 4 if shape.recipe == 0 else 1
    return active * (code_bytes(shape, I, H) + scale_bytes(shape, I, H)) + A * I + A * (I // g) * sb + A * H * 4


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 50 ms in the background."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index=0):
        self.proc = None
        self.t0 = None
        try:
            props = torch.cuda.get_device_properties(device_index)
            uuid = str(getattr(props, "uuid", "")) or None
            sel = ["-i", ("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else uuid] if uuid else []
            self.path = os.path.join("/tmp", f"moefp8_clocks_{os.getpid()}.csv")
            self.proc = subprocess.Popen(
                ["nvidia-smi", *sel, f"--query-gpu=timestamp,{self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, window):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        self.proc.wait(timeout=5)
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                rows.append((ts, float(parts[1]), float(parts[2]), parts[3:]))
            except ValueError:
                continue
        os.unlink(self.path)
        t0, t1 = window
        sel = [r for r in rows if t0 - 1.0 <= r[0] <= t1 + 1.0] or rows
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in sel for n, v in zip(names, r[3][2:6]) if v.strip().lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in sel), "sm_max_mhz": max(r[2] for r in sel),
                "reasons": reasons, "samples": len(sel)}


def traffic_for(kernel: str, workload: str):
    """dram bytes per launch from a committed ncu summary, if it was taken on the current
    kernel source (matching hash); else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        ent = d.get(f"{kernel}:{workload}")
        src = os.path.join(ROOT, "mixture_experts_fp8_b200", "csrc", ent["source"])
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        return ent["dram_bytes_per_launch"] if h == ent["source_sha256_16"] else None
    except Exception:
        return None


def run_cpu_oracle(shape, prob, n_tokens, threads=None):
    import oracle
    if threads:
        oracle.set_num_threads(threads)
    ni = prob.numpy_inputs()
    c = oracle.Config(**shape.cfg())
    tok = np.linspace(0, shape.num_tokens - 1, n_tokens).astype(np.int32)
    t = time.perf_counter()
    oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"], logits=ni["logits"],
                   per_expert_scale=ni["per_expert_scale"], b13=ni["b13"], b2=ni["b2"], tokens=tok)
    dt = time.perf_counter() - t
    return n_tokens / dt, dt, oracle.num_threads()


def reduce_max(value: float, dist=None, device="cpu") -> float:
    """The largest of the ranks' values, returned on every rank (one all-reduce; the identity
    without a process group).  Multi-GPU times are the slowest rank's."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_rank: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (ms_max / 1e3)


def gate_only(args, shape, local):
    """The gate alone (moe_gate: the router matmul on the tensor core, then the RMS-Norm factor and
    the router top-k) on the problem's hidden states.  Its inputs fit in L2, so L2 is flushed
    before every launch and each launch is timed by its own CUDA events."""
    import mixture_experts_fp8_b200 as moe

    torch.cuda.set_device(local)
    dev = f"cuda:{local}"
    x, _, pes = synth.make_activations(shape, device=dev)
    nw, rw, eps = synth.make_gate(shape, device=dev)
    cfg = moe.Config(**shape.cfg())
    gw = moe.transform_gate_weights(cfg, nw, rw)
    T, H, E, k = shape.num_tokens, shape.hidden, shape.num_experts, shape.top_k
    lg = torch.empty((T, E), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)      # twice the L2
    run = lambda: moe.gate(cfg, x, gw, eps, per_expert_scale=pes, logits=lg, topk_idx=idx, topk_weights=w)
    for _ in range(args.warmup):
        flush.zero_()
        run()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    t0 = time.time()
    for a, b in evs:
        flush.zero_()
        a.record()
        run()
        b.record()
    torch.cuda.synchronize()
    t1 = time.time()
    ms = sum(a.elapsed_time(b) for a, b in evs)
    clocks = sampler.stop((t0, t1))
    pk, pk_kind = peaks()
    peak = float(pk["bf16_tflops"])          # burst: each launch is timed alone
    # three bf16 products per (token, expert, column): the split that keeps fp32 accuracy
    tc_flops = 3 * 2.0 * T * E * H
    achieved = tc_flops * args.steps / (ms / 1e3) / 1e12
    line = {
        "metric": "gate tokens/s", "value": T * args.steps / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 x3 (fp32-accurate)", "data": "synthetic",
        "config": {"workload": describe(shape) + "; the gate alone (RMSNorm + router matmul + top-k)",
                   "l2": "flushed before every launch"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None, "kernel": "k_gate_mma + k_route",
                     "peak_kind": pk_kind + " bf16 burst"},
        "hbm": {"algorithmic_bytes": 2 * T * H + 6 * E * H + 4 * T * E + 8 * T * k,
                "GB/s": (2 * T * H + 6 * E * H + 4 * T * E + 8 * T * k) * args.steps / (ms / 1e3) / 1e9},
        "clocks": clocks, "gpu_launches": 2 * args.steps,
    }
    print(json.dumps(line))


class LocalExchange:
    """The all-to-all of a single rank: every row stays home (what ep_step sees at N = 1)."""

    @staticmethod
    def all_to_all_single(out, inp, out_splits=None, in_splits=None, group=None):
        out.copy_(inp)


def ep_bench(args, shape, world, rank, local, dist):
    """Expert parallelism (mixture_experts_fp8_b200.ep): every rank owns E/N experts and routes its
    own batch of the problem's size; one step = route, dispatch, all-to-all, the expert side,
    the reverse all-to-all, combine.  Times K steps with CUDA events, max over ranks."""
    import mixture_experts_fp8_b200 as moe
    from mixture_experts_fp8_b200 import ep

    torch.cuda.set_device(local)
    dev = f"cuda:{local}"
    from dataclasses import replace
    prob = synth.make_problem(shape, device=dev)                    # the same layer on every rank
    x, logits, _ = synth.make_activations(replace(shape, seed=shape.seed + 1000 * rank), device=dev)  # its tokens
    e_loc = shape.num_experts // world
    es = slice(rank * e_loc, (rank + 1) * e_loc)
    cfg = moe.Config(**shape.cfg())
    cfg_w = ep.rows_config(cfg, world, 1)
    w_local = moe.transform_weights(cfg_w, prob.w13[es].contiguous(), prob.w13_scale[es].contiguous(),
                                    prob.w2[es].contiguous(), prob.w2_scale[es].contiguous())
    b13 = None if prob.w13_bias is None else prob.w13_bias[es].contiguous()
    b2 = None if prob.w2_bias is None else prob.w2_bias[es].contiguous()
    ws = moe.new_workspace(cfg, dev)
    exch = dist if dist is not None else LocalExchange()

    def step():
        return ep.ep_step(cfg, world, x, logits, w_local, exch, per_expert_scale=prob.per_expert_scale,
                          w13_bias_local=b13, w2_bias_local=b2, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        y, stats = step()
    b.record()
    torch.cuda.synchronize()
    ms = reduce_max(a.elapsed_time(b), dist, dev)
    if rank == 0:
        line = {"metric": "MoE-layer tokens/s, expert parallel", "value": job_tokens_per_s(world, shape.num_tokens,
                                                                                      args.steps, ms),
                "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "e4m3", "data": "synthetic",
                "config": {"workload": describe(shape) + f"; expert parallel over {world} rank(s), "
                                                         f"{e_loc} experts each",
                           "exchange": "torch.distributed all_to_all_single" if dist else "none (one rank)"},
                "ep": {"rows_sent_by_rank0": stats["sent"], "rows_received_by_rank0": stats["received"]}}
        print(json.dumps(line))


def reference_arm(args, shape, rank):
    if rank != 0:
        return
    import oracle
    prob = synth.make_problem(shape, device="cpu")
    idx, _, _ = oracle.route(oracle.Config(**shape.cfg()), prob.numpy_inputs()["logits"],
                             prob.numpy_inputs()["per_expert_scale"])
    active = int(np.unique(idx).size) + shape.shared_experts
    # tokens per step: the whole batch where one oracle call on it takes well under a second
    # (tiny, decode), else a sample sized so that a step stays near a second
    n = {"tiny": 16, "decode": 64, "decode_w4a8": 64, "skewed": 16, "prefill": 2, "large": 4}.get(shape.name, 4)
    for _ in range(args.warmup):
        run_cpu_oracle(shape, prob, 1)
    times = []
    for _ in range(args.steps):
        _, dt, cores = run_cpu_oracle(shape, prob, n)
        times.append(dt)
    tot = sum(times)
    value = n * args.steps / tot
    sample = (f"{n} of {shape.num_tokens} tokens per step, evenly spaced (a row's output does not depend on "
              f"the other rows)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(shape, active, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="large", choices=sorted(synth.SHAPES))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the problem's token count (reduced cases for profiler captures)")
    ap.add_argument("--shared-expert", action="store_true",
                    help="add a shared expert (every token, weight 1) to the problem")
    ap.add_argument("--recipe", type=int, default=None, choices=[0, 1, 2],
                    help="run the problem with another quantization recipe (0 fp32 per 128, 1 MXFP8, 2 W4A8)")
    ap.add_argument("--gate", action="store_true",
                    help="start each step from the gate (RMSNorm + router matmul + top-k, moe_gate) on "
                         "the bf16 hidden states instead of from precomputed router logits")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism: every rank owns num_experts/N experts and routes its own batch")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every kernel from the host instead of replaying a captured CUDA graph")
    ap.add_argument("--gate-only", action="store_true",
                    help="time the gate alone (no expert layer), L2 flushed before every launch")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    shape = synth.SHAPES[args.config]
    if args.tokens:
        shape = shape.with_tokens(args.tokens)
    if args.shared_expert:
        from dataclasses import replace
        shape = replace(shape, shared_experts=1)
    if args.recipe is not None and args.recipe != shape.recipe:
        from dataclasses import replace
        shape = replace(shape, recipe=args.recipe, name=f"{shape.name}_r{args.recipe}")

    if args.impl == "reference":
        reference_arm(args, shape, rank)
        return
    if args.gate_only:
        if rank == 0:
            gate_only(args, shape, local)
        return
    if args.ep:
        dist = None
        if world > 1:
            import datetime

            import torch.distributed as dist
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        try:
            ep_bench(args, shape, world, rank, local, dist)
        finally:
            if dist:
                dist.destroy_process_group()
        return

    import mixture_experts_fp8_b200 as moe

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    dev = f"cuda:{local}"
    # big problems (prefill, large): inputs drawn on the device, the fp32 weights freed after the transform
    big = shape.num_experts * shape.hidden * shape.inter >= 500_000_000
    gen_dev = dev if big else "cpu"
    prob = synth.make_problem(shape, device=gen_dev)
    d = prob.to(dev)
    cfg = moe.Config(**shape.cfg())
    weights = moe.transform_weights(cfg, d.w13, d.w13_scale, d.w2, d.w2_scale)
    # the CPU baseline's input: a host copy of a token sample with every weight, taken before the
    # device copies of the big problems' untransformed weights are freed
    cpu_n = {"tiny": 16, "decode": 64, "skewed": 64, "prefill": 4, "large": 16}.get(shape.name, 8)
    cpu_prob = None
    if world == 1 and not args.no_cpu_baseline:
        cpu_prob = prob if prob.x.device.type == "cpu" and cpu_n >= shape.num_tokens else \
            host_sample(prob, min(cpu_n, shape.num_tokens))
    if big:
        del d.w13, d.w2, prob
    ws = moe.new_workspace(cfg, dev)
    y = torch.empty((shape.num_tokens, shape.hidden), dtype=torch.bfloat16, device=dev)
    counts = torch.zeros(shape.num_experts + shape.shared_experts, dtype=torch.int32, device=dev)

    if args.gate:
        norm_w, router_w, eps = (t.to(dev) if torch.is_tensor(t) else t for t in synth.make_gate(shape))
        gate_w = moe.transform_gate_weights(cfg, norm_w, router_w)     # once per set of weights
        g_logits = torch.empty((shape.num_tokens, shape.num_experts), dtype=torch.float32, device=dev)
        g_idx = torch.empty((shape.num_tokens, shape.top_k), dtype=torch.int32, device=dev)
        g_w = torch.empty((shape.num_tokens, shape.top_k), dtype=torch.float32, device=dev)

    def step(profile=None, x=None):
        x = d.x if x is None else x
        if args.gate:      # the gate replaces the router; the forward takes its routing
            moe.gate(cfg, x, gate_w, eps, per_expert_scale=d.per_expert_scale, logits=g_logits,
                     topk_idx=g_idx, topk_weights=g_w)
            moe.forward(cfg, x, weights, topk_idx=g_idx, topk_weights=g_w, w13_bias=d.w13_bias,
                        w2_bias=d.w2_bias, y=y, expert_counts=counts, workspace=ws, profile=profile)
        else:
            moe.forward(cfg, x, weights, router_logits=d.logits, per_expert_scale=d.per_expert_scale,
                        w13_bias=d.w13_bias, w2_bias=d.w2_bias, y=y, expert_counts=counts, workspace=ws,
                        profile=profile)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = moe.read_status(ws)
    active = int((counts.cpu() > 0).sum())
    A = shape.num_tokens * (shape.top_k + shape.shared_experts)   # rows through the GEMMs

    # Several consecutive steps captured into one CUDA graph: a replay is one host call instead of
    # six to eight launches per step, and inside the graph each step's first kernel still overlaps
    # the previous step's last one (programmatic dependent launch edges).  Eager launches with
    # --no-graph, or when the capture fails (reported in the line).
    def capture(n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(n):
                step()
        return g

    def timed_steps():             # exactly args.steps steps
        for _ in range(args.steps):
            step()

    run = timed_steps
    graph_info = {"used": False, "why": "--no-graph"}
    if not args.no_graph:
        try:
            gs = 10
            y_eager = y.clone()
            g_main = capture(gs)
            g_rest = capture(args.steps % gs) if args.steps % gs else None
            y.zero_()
            g_main.replay()
            torch.cuda.synchronize()
            same = bool(torch.equal(y, y_eager))

            def run():
                for _ in range(args.steps // gs):
                    g_main.replay()
                if g_rest is not None:
                    g_rest.replay()
            graph_info = {"used": True, "steps_per_graph": gs, "same_output_as_eager": same}
        except Exception as exc:   # noqa: BLE001 - any capture failure falls back to launches
            torch.cuda.synchronize()
            graph_info = {"used": False, "why": f"capture failed: {exc}"[:300]}

    # timed region: K plain forwards (no events between the kernels, which would break their
    # programmatic-dependent-launch overlap)
    sampler = ClockSampler(local)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start.record()
    run()
    end.record()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if dist:
        dist.barrier()
    ms = start.elapsed_time(end)
    clocks = sampler.stop((t_wall0, t_wall1))
    ms = reduce_max(ms, dist, dev)
    # per-stage device times: K more forwards with CUDA events recorded by the library between the
    # stages, on the launch stream
    prof = moe.Profile()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record()
    for _ in range(args.steps):
        step(prof)
    p1.record()
    torch.cuda.synchronize()
    ms_profiled = p0.elapsed_time(p1)
    stage_ms, calls = prof.read()
    prof.close()

    # end to end: pinned host inputs -> device, forward, result -> host, every step.  The copies
    # run on their own streams into and out of two buffer slots, so step i+1's inputs arrive and
    # step i-1's result leaves while step i computes; the library call is the same.
    x_h = d.x.cpu().pin_memory()
    l_h = d.logits.cpu().pin_memory()
    NB = 2
    y_h = [torch.empty_like(y, device="cpu").pin_memory() for _ in range(NB)]
    x_d = [torch.empty_like(d.x) for _ in range(NB)]
    l_d = [torch.empty_like(d.logits) for _ in range(NB)]
    y_d = [torch.empty_like(y) for _ in range(NB)]
    s_c = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in range(NB)]
    fwd_done = [torch.cuda.Event() for _ in range(NB)]
    out_done = [torch.cuda.Event() for _ in range(NB)]
    used = [False] * NB

    def fwd(x_in, l_in, y_out):
        if args.gate:          # the gate's input is x alone
            moe.gate(cfg, x_in, gate_w, eps, per_expert_scale=d.per_expert_scale, logits=g_logits,
                     topk_idx=g_idx, topk_weights=g_w)
            moe.forward(cfg, x_in, weights, topk_idx=g_idx, topk_weights=g_w, w13_bias=d.w13_bias,
                        w2_bias=d.w2_bias, y=y_out, workspace=ws)
        else:
            moe.forward(cfg, x_in, weights, router_logits=l_in, per_expert_scale=d.per_expert_scale,
                        w13_bias=d.w13_bias, w2_bias=d.w2_bias, y=y_out, workspace=ws)

    e2e_graphs = None
    if graph_info["used"]:     # one graph per buffer slot
        try:
            e2e_graphs = []
            for b in range(NB):
                gg = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gg):
                    fwd(x_d[b], l_d[b], y_d[b])
                e2e_graphs.append(gg)
        except Exception:          # noqa: BLE001
            torch.cuda.synchronize()
            e2e_graphs = None

    def e2e_step(i):
        b = i % NB
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(fwd_done[b])          # the forward that read slot b is done
            x_d[b].copy_(x_h, non_blocking=True)
            if not args.gate:
                l_d[b].copy_(l_h, non_blocking=True)
            in_done[b].record(s_in)
        s_c.wait_event(in_done[b])
        if used[b]:
            s_c.wait_event(out_done[b])               # slot b's previous result has left
        if e2e_graphs:
            e2e_graphs[b].replay()
        else:
            fwd(x_d[b], l_d[b], y_d[b])
        fwd_done[b].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(fwd_done[b])
            y_h[b].copy_(y_d[b], non_blocking=True)
            out_done[b].record(s_out)
        used[b] = True

    gate_ms = None
    if args.gate:              # the gate kernel alone, CUDA events on the launch stream
        for _ in range(args.warmup):
            moe.gate(cfg, d.x, gate_w, eps, per_expert_scale=d.per_expert_scale, logits=g_logits,
                     topk_idx=g_idx, topk_weights=g_w)
        q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        q0.record()
        for _ in range(args.steps):
            moe.gate(cfg, d.x, gate_w, eps, per_expert_scale=d.per_expert_scale, logits=g_logits,
                     topk_idx=g_idx, topk_weights=g_w)
        q1.record()
        torch.cuda.synchronize()
        gate_ms = q0.elapsed_time(q1) / args.steps

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_c)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(args.steps):
        e2e_step(args.warmup + i)
    s_c.wait_stream(s_out)                            # every result is on the host
    e1.record(s_c)
    torch.cuda.synchronize()
    # the last result read back equals the device-timed loop's output (same inputs, same bits)
    e2e_same = bool(torch.equal(y_h[(args.warmup + args.steps - 1) % NB], y.cpu()))
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = reduce_max(e2e_ms, dist, dev)
    if dist:
        dist.barrier()

    if rank == 0:
        pk, pk_kind = peaks()
        hbm = float(pk["hbm_gbs"])
        # dense FP8 peak: the measured burst bf16 GEMM rate x the nominal FP8/BF16 ratio (the
        # higher, stricter denominator of the two measured bf16 figures)
        fp8_peak = float(pk["bf16_tflops"]) * FP8_OVER_BF16
        tok_s = job_tokens_per_s(world, shape.num_tokens, args.steps, ms)
        per_step_s = ms / 1e3 / args.steps
        fl = flops(shape, A)
        alg = algorithmic_bytes(shape, active)
        if args.gate:          # + the gate's folded router weights (the logits are written instead of read)
            alg += 6 * shape.num_experts * shape.hidden
        g1_ms = stage_ms["gemm1_swiglu_requant"] / max(calls, 1)
        g2_ms = stage_ms["gemm2"] / max(calls, 1)
        g1_bytes = gemm1_bytes(shape, active)
        g1_gbs = g1_bytes / (g1_ms / 1e3) / 1e9
        g1_tflops = 2.0 * A * shape.hidden * 2 * shape.inter / (g1_ms / 1e3) / 1e12
        compute_bound = fl / alg > (fp8_peak * 1e12) / (hbm * 1e9)
        if compute_bound:
            roof = {"bound": "tensor", "achieved": g1_tflops, "peak": fp8_peak, "unit": "TFLOP/s",
                    "frac": g1_tflops / fp8_peak}
        else:
            roof = {"bound": "hbm", "achieved": g1_gbs, "peak": hbm, "unit": "GB/s", "frac": g1_gbs / hbm}
        # the library's kernel choice: at most 32 routed rows per expert on average -> the swap-AB
        # kernels (fp32 scales: narrow; MXFP8 / W4A8: mx_narrow), else the wide ones
        few = A <= 32 * (shape.num_experts + shape.shared_experts)
        kname = ("k_grouped_gemm_mx_narrow" if few else "k_grouped_gemm_mx") if shape.recipe != 0 else \
                ("k_grouped_gemm_narrow" if few else "k_grouped_gemm")
        roof.update({"kernel": kname + "<gate+up>",
                     "traffic": traffic_for("gemm1", shape.name),
                     "peak_source": f"{pk_kind} ({'burst bf16 x2 for fp8' if compute_bound else 'copy'})",
                     "algorithmic_bytes_per_launch": g1_bytes, "ms_per_launch": g1_ms})
        layer_roof_s = max(fl / (fp8_peak * 1e12), alg / (hbm * 1e9))
        line = {
            "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
            "config": workload_config(shape, active, world, args.gate),
            "tflops": fl / per_step_s / 1e12,
            "layer_roofline": {"bound": "tensor" if compute_bound else "hbm", "roofline_ms": layer_roof_s * 1e3,
                               "frac": layer_roof_s / per_step_s, "algorithmic_bytes": alg, "flops": fl},
            "roofline": roof,
            "stages_ms": {k: v / max(calls, 1) for k, v in stage_ms.items()},
            "ms_per_step_with_stage_events": ms_profiled / args.steps,
            "gemm2": {"ms": g2_ms, "GB/s": gemm2_bytes(shape, active) / (g2_ms / 1e3) / 1e9},
            "clocks": clocks, "gpu_launches": kernels_per_step(A) * args.steps, "status": status,
            "graph": dict(graph_info, e2e=e2e_graphs is not None),
            "e2e": {"value": world * shape.num_tokens * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": x_h.numel() * 2 + (0 if args.gate else l_h.numel() * 4),
                    "d2h_bytes_per_step": y_h[0].numel() * 2,
                    "copies": "own streams, two buffer slots: they overlap the neighbouring steps",
                    "result_matches_device_loop": e2e_same},
        }
        if args.gate:
            T, H, E, k = shape.num_tokens, shape.hidden, shape.num_experts, shape.top_k
            # x, the three bf16 parts of the folded router weights, the logits, ids and weights
            gbytes = 2 * T * H + 6 * E * H + 4 * T * E + 8 * T * k
            gflops = 2.0 * T * E * H
            line["gate"] = {"kernel": "k_gate_mma + k_route", "ms_per_launch": gate_ms, "algorithmic_bytes": gbytes,
                            "GB/s": gbytes / (gate_ms / 1e3) / 1e9, "TFLOP/s": gflops / (gate_ms / 1e3) / 1e12,
                            "note": "stages_ms covers the forward after the gate (its route stage is "
                                    "empty: the routing comes from the gate)"}
        if cpu_prob is not None:
            n = cpu_prob.shape.num_tokens
            v, tot, reps, cores = time_cpu_oracle(cpu_prob.shape, cpu_prob, n, 10.0)
            line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                    "sample": f"{n} of {shape.num_tokens} tokens (seeded sample, every "
                                              f"weight) x {reps} runs, {tot:.1f} s"}
            if shape.name in ("tiny", "decode"):
                v1, tot1, reps1, _ = time_cpu_oracle(cpu_prob.shape, cpu_prob, n, 5.0, threads=1)
                line["cpu_baseline_1thread"] = {"value": v1, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                                "sample": f"{n} of {shape.num_tokens} tokens x {reps1} runs, "
                                                          f"{tot1:.1f} s"}
        elif world == 1:
            line["cpu_baseline"] = None
        print(json.dumps(line), flush=True)

    if dist:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
