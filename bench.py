"""Benchmark of the MoE layer hot path (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload NAME]

One step = one forward and one backward of the layer (routing, dispatch,
grouped SwiGLU experts, combine, and the backward of all of it, weight
gradients accumulated in fp32) over one microbatch of synthetic tokens that
is already resident in HBM. Default workload: one packed 32k-token sequence,
d_model 2048, 64 experts, top-8, SwiGLU width 1408, Zipf-skewed routing with
four starved experts, EP=4 send layout.

Timing: W untimed warm-up steps, then exactly K steps between a barrier +
synchronize on both sides, measured with CUDA events on the launching stream;
the slowest rank's time counts. With N GPUs (torchrun) every rank runs its own
microbatch against replicated weights (data parallel, no collective on the
data path): weak scaling, `value` counts the tokens of all ranks.
Per-call CUDA events inside the timed steps give each C call's duration; the
roofline entry is the grouped wgrad kernel (one launch per step).
The e2e leg repeats the step through the same C calls with the inputs copied
from pinned host memory and Y, dX copied back, inside the timed region.
`--impl reference` times the CPU oracle instead (rank 0 only).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer fwd+bwd tokens/s"
UNIT = "tokens/s"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------ algorithmic work

def algorithmic_work(w, T: int):
    """Flops (GEMM-like calls) or bytes (HBM-bound calls) per call, per step."""
    d, E, k, f = w.d, w.E, w.k, w.f
    P = T * k
    b = 2 if w.dtype == "bf16" else 4
    flops = {
        "router_logits": 2.0 * T * d * E,
        "grouped_ffn_fwd": 6.0 * d * f * P,
        "grouped_ffn_dgrad": 6.0 * d * f * P,
        "grouped_ffn_wgrad": 6.0 * d * f * P,
        "router_bwd": 2.0 * T * d * E,
    }
    # the fused-dispatch forms do the same arithmetic
    for n in ("grouped_ffn_fwd", "grouped_ffn_wgrad", "router_bwd"):
        flops[n + "_gather"] = flops[n]
    bytes_ = {
        "permute": (T * d + P * d) * b + 4 * P,
        "unpermute_combine": (P * d + T * d) * b + 8 * P,
        "unpermute_combine_bwd": (T * d + 2 * P * d) * b + 12 * P,
        "permute_bwd": (P * d + T * d) * b + 12 * P,
        "route": 4 * T * E + 16 * P,
        "route_bwd": 12 * P + 4 * T * E,
    }
    return flops, bytes_


def source_hash() -> str:
    h = hashlib.sha256()
    with open(os.path.join(ROOT, "grouped_expert_ffn_top_b200", "csrc", "grouped_gemm_sm100.cu"), "rb") as fh:
        h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key: str):
    """Per-launch DRAM bytes of the roofline kernel from the committed ncu
    summary, or None if absent or taken on another version of the kernel."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as fh:
            t = json.load(fh)
        ent = t[kernel_key]
        if ent.get("source_hash") != source_hash():
            return None
        return float(ent["bytes_per_launch"])
    except Exception:
        return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.dev), "-lms", "200"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------- CPU oracle

def oracle_step_fn(w, params_np, x_np, dY_np):
    """One oracle forward+backward over the given tokens (a bounded sample)."""
    import oracle

    def step(n: int):
        x = x_np[:n]
        dY = dY_np[:n]
        P = params_np
        fw = oracle.layer_forward(x, P["Wr"], P["b"], P["Wg"], P["Wu"], P["Wd"], w.k, w.ep_groups)
        oracle.layer_backward(fw, x, dY, P["Wr"], P["Wg"], P["Wu"], P["Wd"], w.k)
    return step


def oracle_inputs(w, seed: int = 0):
    """Workload params and the first microbatch on the host, in double."""
    import numpy as np
    import torch

    from grouped_expert_ffn_top_b200 import workloads
    p = workloads.make_params(w, device="cpu", seed=seed)
    bt = workloads.make_batch(w, device="cpu", seed=seed)
    P = {n: v.to(torch.float64).numpy() for n, v in p.items()}
    return P, bt["x"].to(torch.float64).numpy(), bt["dY"].to(torch.float64).numpy()


def calibrate_sample(step, budget_s: float, T: int) -> int:
    """Token count whose oracle step takes about budget_s seconds: a linear
    fit (fixed cost + cost per token) through two probe sizes."""
    def timed(n):
        t0 = time.perf_counter()
        step(n)
        return max(time.perf_counter() - t0, 1e-4)

    step(2)  # first call: thread start-up and first touches of the weights
    n0 = 8
    t0 = timed(n0)
    n1 = int(max(2 * n0, min(T, n0 * 0.25 * budget_s / t0)))
    t1 = timed(n1)
    per_token = max((t1 - t0) / (n1 - n0), 1e-9)
    fixed = max(t0 - per_token * n0, 0.0)
    return int(max(1, min(T, (budget_s - fixed) / per_token)))


def cpu_baseline(w, budget_s: float = 15.0):
    import oracle
    P, x, dY = oracle_inputs(w)
    step = oracle_step_fn(w, P, x, dY)
    n = calibrate_sample(step, budget_s, w.T[0])
    t0 = time.perf_counter()
    step(n)
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"oracle fwd+bwd of the first {n} of the {w.T[0]} tokens "
                      f"({dt:.1f} s of CPU work)"}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    P, x, dY = oracle_inputs(w)
    step = oracle_step_fn(w, P, x, dY)
    per_step_budget = max(0.5, 150.0 / max(1, args.steps + args.warmup))
    n = calibrate_sample(step, per_step_budget, w.T[0])
    for _ in range(args.warmup):
        step(n)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step(n)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * dt / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": dict(workload_config(w), parallelism=f"dp{args.gpus}"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"each step: oracle fwd+bwd of the first {n} tokens"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w):
    return {"workload": w.name, "tokens_per_gpu": w.T[0], "d_model": w.d, "experts": w.E,
            "top_k": w.k, "ffn": w.f, "ep_groups": w.ep_groups, "routing": str(w.bias),
            "l2": "inputs larger than L2 (x alone is %.0f MB; a step moves several GB); no flush"
                  % (w.T[0] * w.d * 2 / 1e6),
            "grads": "each step writes its own fp32 parameter gradients (one microbatch per "
                     "optimizer step)"}


# ------------------------------------------------------------ end to end

def run_e2e(layer, x_h, dY_h, steps: int, dev, stream) -> float:
    """Milliseconds for `steps` layer steps fed from pinned host memory.

    Every step copies its inputs x, dY host->device and its outputs Y, dX
    device->host inside the timed region. Copies run on their own streams
    with two buffers per tensor, so step i+1's inputs arrive while step i
    computes and step i's outputs leave while step i+1 computes (the way a
    training loop feeds the layer)."""
    import torch
    cin, cout = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    like = lambda t: torch.empty(t.shape, dtype=t.dtype, device=dev)
    x_d, dY_d = [like(x_h), like(x_h)], [like(dY_h), like(dY_h)]
    Y_d, dX_d = [like(x_h), like(x_h)], [like(dY_h), like(dY_h)]
    Y_h = [torch.empty_like(x_h).pin_memory() for _ in range(2)]
    dX_h = [torch.empty_like(dY_h).pin_memory() for _ in range(2)]
    in_ready, used, out_done = [None, None], [None, None], [None, None]

    def h2d(i):
        b = i % 2
        with torch.cuda.stream(cin):
            if used[b] is not None:
                cin.wait_event(used[b])  # step i-2 has finished reading this buffer
            x_d[b].copy_(x_h, non_blocking=True)
            dY_d[b].copy_(dY_h, non_blocking=True)
            in_ready[b] = torch.cuda.Event()
            in_ready[b].record(cin)

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    cin.wait_event(start)
    cout.wait_event(start)
    h2d(0)
    for i in range(steps):
        b = i % 2
        stream.wait_event(in_ready[b])
        if out_done[b] is not None:
            stream.wait_event(out_done[b])  # step i-2's outputs have left this buffer
        if i + 1 < steps:
            h2d(i + 1)
        layer.forward(x_d[b], stream=stream, out=Y_d[b])
        layer.backward(dY_d[b], stream=stream, out=dX_d[b], accumulate=False)
        used[b] = torch.cuda.Event()
        used[b].record(stream)
        with torch.cuda.stream(cout):
            cout.wait_event(used[b])
            Y_h[b].copy_(Y_d[b], non_blocking=True)
            dX_h[b].copy_(dX_d[b], non_blocking=True)
            out_done[b] = torch.cuda.Event()
            out_done[b].record(cout)
    for ev in out_done:
        if ev is not None:
            stream.wait_event(ev)
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end)


# ------------------------------------------------------------ ranks

class Ranks:
    """Data-parallel ranks of the benchmark (one process per GPU).

    Every rank draws its own microbatch (seed = rank) against the same
    weights; the only collectives are the barrier around the timed region and
    the max of the ranks' times, so nothing is exchanged on the data path."""

    def __init__(self, backend: str = "nccl", device=None):
        import datetime

        import torch
        import torch.distributed as dist
        self.dist = dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device if device is not None else torch.device("cuda", self.local)
        self.cuda = self.device.type == "cuda"
        if self.world > 1:
            kw = {"timeout": datetime.timedelta(seconds=120)}
            if self.cuda:
                torch.cuda.set_device(self.device)
                kw["device_id"] = self.device
            dist.init_process_group(backend, **kw)

    @property
    def batch_seed(self) -> int:
        return self.rank

    @property
    def prints(self) -> bool:
        return self.rank == 0

    def barrier(self):
        import torch
        if self.world > 1:
            self.dist.barrier()
        if self.cuda:
            torch.cuda.synchronize(self.device)

    def max_over_ranks(self, v: float) -> float:
        import torch
        if self.world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            self.dist.barrier()
            self.dist.destroy_process_group()


# ------------------------------------------------------------ native arm

def run_native(args, w):
    import numpy as np
    import torch

    from grouped_expert_ffn_top_b200 import native as N
    from grouped_expert_ffn_top_b200 import workloads
    from grouped_expert_ffn_top_b200.layer import MoELayer

    R = Ranks("nccl")
    world, rank, local, dev = R.world, R.rank, R.local, R.device
    N.lib()
    T = w.T[0]
    params = workloads.make_params(w, device=dev, seed=0)
    batch = workloads.make_batch(w, device=dev, seed=R.batch_seed)
    fused = args.dispatch == "fused"
    sfx = "_gather" if fused else ""
    layer = MoELayer(params, w.k, w.ep_groups, max_tokens=T, checkpoint=args.checkpoint,
                     fused_dispatch=fused)
    stream = torch.cuda.current_stream(dev)
    barrier = R.barrier
    max_over_ranks = R.max_over_ranks

    # one microbatch per optimizer step: each step writes its own parameter
    # gradients (no accumulation across steps)
    for _ in range(args.warmup):
        layer.forward(batch["x"])
        layer.backward(batch["dY"], accumulate=False)
    barrier()
    errs = layer.device_errors()
    if errs:
        raise RuntimeError(f"device error word {errs} during warm-up")

    # ---- device-timed region
    names = []
    events = []

    def mark(name):
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(stream)
        names.append(name)
        events.append(ev)

    sampler = ClockSampler(local) if rank == 0 else None
    launches0 = N.moe_launch_count()
    barrier()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    step_marks = []
    for _ in range(args.steps):
        first = len(events)
        mark("step_start")
        layer.forward(batch["x"], mark=mark)
        layer.backward(batch["dY"], mark=mark, accumulate=False)
        step_marks.append(first)
    end.record(stream)
    barrier()
    clocks = sampler.stop() if sampler else None
    launches = N.moe_launch_count() - launches0
    total_ms = max_over_ranks(start.elapsed_time(end))

    per_call = {}
    for i in range(1, len(events)):
        if names[i] == "step_start":
            continue
        per_call.setdefault(names[i], []).append(events[i - 1].elapsed_time(events[i]))
    call_ms = {n: statistics.mean(v) for n, v in per_call.items()}

    # ---- end-to-end region: host inputs in, host outputs out, every step
    x_h = batch["x"].cpu().pin_memory()
    dY_h = batch["dY"].cpu().pin_memory()
    run_e2e(layer, x_h, dY_h, 2, dev, stream)
    barrier()
    e2e_ms = max_over_ranks(run_e2e(layer, x_h, dY_h, args.steps, dev, stream))
    errs = layer.device_errors()
    if errs:
        raise RuntimeError(f"device error word {errs} in the timed region")

    # routing load of the batch and the device memory the step held (read
    # after the timed regions)
    counts = layer.r["counts"].cpu().numpy().astype(np.int64)
    nonzero = counts[counts > 0]
    routing = {"experts": int(counts.size), "empty_experts": int((counts == 0).sum()),
               "rows_max": int(counts.max()), "rows_min_nonzero": int(nonzero.min()) if nonzero.size else 0,
               "max_over_mean": round(float(counts.max() / max(counts.mean(), 1e-9)), 3)}
    free_b, total_b = torch.cuda.mem_get_info(dev)
    memory = {"peak_allocated_gb": round(torch.cuda.max_memory_allocated(dev) / 1e9, 2),
              "device_used_gb": round((total_b - free_b) / 1e9, 2),
              "device_total_gb": round(total_b / 1e9, 1)}

    hbm, bf16_burst, bf16_sust, peak_src = _peaks()
    flops, bytes_ = algorithmic_work(w, T)
    kernels = {}
    for n, ms in call_ms.items():
        ent = {"ms": round(ms, 4), "launches": 1}
        from grouped_expert_ffn_top_b200.layer import LAUNCHES_PER_CALL
        ent["launches"] = LAUNCHES_PER_CALL.get(n, 1)
        if n in flops:
            tf = flops[n] / (ms * 1e-3) / 1e12
            ent.update({"tflops": round(tf, 1), "frac_bf16_sustained": round(tf / bf16_sust, 3)})
        elif n in bytes_:
            gbs = bytes_[n] / (ms * 1e-3) / 1e9
            ent.update({"gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                        "frac_8tbs": round(gbs / 8000.0, 3)})
        kernels[n] = ent

    wg_ms = call_ms["grouped_ffn_wgrad" + sfx]
    wg_tf = flops["grouped_ffn_wgrad"] / (wg_ms * 1e-3) / 1e12
    traffic = ncu_traffic("grouped_ffn_wgrad" + sfx)
    roofline = {"kernel": f"grouped_ffn_wgrad{sfx} (tcgen05 grouped GEMM, ragged K)", "bound": "tensor",
                "achieved": round(wg_tf, 1), "peak": bf16_sust, "unit": "TFLOP/s",
                "frac": round(wg_tf / bf16_sust, 3), "traffic": traffic,
                "peak_source": f"{peak_src} bf16 sustained (timed inside a long step)",
                "algorithmic_flops_per_launch": flops["grouped_ffn_wgrad"]}
    gemm_ms = sum(call_ms[n] for n in ("grouped_ffn_fwd" + sfx, "grouped_ffn_dgrad", "grouped_ffn_wgrad" + sfx))
    gemm_tf = 18.0 * w.d * w.f * T * w.k / (gemm_ms * 1e-3) / 1e12
    mem_calls = tuple(n for n in ("permute", "unpermute_combine", "unpermute_combine_bwd", "permute_bwd")
                      if n in call_ms)
    mem_ms = sum(call_ms[n] for n in mem_calls)
    mem_gbs = sum(bytes_[n] for n in mem_calls) / (mem_ms * 1e-3) / 1e9

    ms_per_step = total_ms / args.steps
    value = world * T * args.steps / (total_ms * 1e-3)
    e2e_value = world * T * args.steps / (e2e_ms * 1e-3)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Gaussian activations and weights, Zipf-skewed router bias)",
        "impl": "native",
        "config": dict(workload_config(w), parallelism=f"dp{world}"),
        # how this arm runs the layer (the workload is the same either way)
        "options": {"dispatch": ("fused: expert rows gathered from x inside the GEMM operand loads, "
                                 "no permuted copy" if fused else "permute: rows copied to xp first"),
                    "activations": ("checkpointed: h1, h2 rebuilt in the backward" if args.checkpoint
                                    else "stored")},
        "grouped_gemm": {"tflops": round(gemm_tf, 1), "frac_bf16_sustained": round(gemm_tf / bf16_sust, 3),
                         "frac_bf16_burst": round(gemm_tf / bf16_burst, 3)},
        "permute_combine": {"gbs": round(mem_gbs, 1), "frac_hbm": round(mem_gbs / hbm, 3),
                            "frac_8tbs": round(mem_gbs / 8000.0, 3)},
        "roofline": roofline,
        "kernels": kernels,
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT,
                "h2d_bytes_per_step": int(x_h.numel() * x_h.element_size() * 2),
                "d2h_bytes_per_step": int(x_h.numel() * x_h.element_size() * 2),
                "how": "x, dY copied from pinned host memory and Y, dX copied back every step; "
                       "copies run on two copy streams, double-buffered so step i+1's inputs "
                       "arrive while step i computes"},
        "gpu_launches": int(launches),
        "routing": routing,
        "memory": memory,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget)
        except Exception as ex:  # report, do not hide
            line["cpu_baseline"] = {"error": repr(ex)}
    if R.prints:
        print(json.dumps(line), flush=True)
    R.close()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="fine_fwdbwd_32k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--checkpoint", action="store_true",
                    help="activation checkpointing: h1, h2 rebuilt in the backward")
    ap.add_argument("--dispatch", choices=["permute", "fused"], default="permute",
                    help="permute: copy the dispatch rows to xp before the GEMMs; fused: gather them "
                         "from x inside the GEMMs' operand loads")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    from grouped_expert_ffn_top_b200 import workloads
    w = workloads.WORKLOADS[args.workload]
    if len(w.T) != 1 or not w.backward:
        ap.error("the benchmark runs single-microbatch forward+backward workloads")
    if args.impl == "reference":
        return run_reference(args, w)
    return run_native(args, w)


if __name__ == "__main__":
    sys.exit(main())
