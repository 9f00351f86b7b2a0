"""Benchmark of the MoE layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload NAME] [--parallel dp|ep] [--dispatch permute|fused]
                    [--checkpoint]

One step = one pass of the layer over the workload's microbatches, with the
inputs already resident in HBM. For the default workload, `uneven_sweep`
(d_model 4096, 16 experts, top-2, SwiGLU width 14336), a step is the uneven
microbatch sweep T = 32768, 9000, 1, 0: each microbatch runs the forward
(routing, dispatch, grouped SwiGLU experts, combine) and the backward of all of
it; the first microbatch writes the fp32 parameter gradients and the others
add to them (gradient accumulation, the empty microbatch included).
`value` = tokens of all microbatches (and all ranks) per second.
Forward-only workloads (`dense_fwd`, `fine_fwd_32k`) time the forward alone
and are also reported beside the headline line under `forward_only`.

Timing: W untimed warm-up steps, then exactly K steps between a barrier +
synchronize on both sides, measured with CUDA events on the launching stream;
the slowest rank's time counts. Per-call CUDA events inside the timed steps
give each C call's duration. The roofline entry is the grouped weight-gradient
kernel's launch on the largest microbatch, against the measured bf16
sustained peak when the timed region lasts a second or more (the power-capped
condition that peak was measured in), else the burst peak; both fractions are
printed beside it.
The e2e leg repeats the steps through the same C calls with every
microbatch's x and dY copied from pinned host memory and Y, dX copied back,
inside the timed region.

Several GPUs: `--gpus N` without a launcher re-executes this script under
torch.distributed.run with N ranks (one per GPU); under a launcher WORLD_SIZE
must equal N. `--parallel dp` (default): every rank runs its own microbatches
against replicated weights, no collective on the data path (weak scaling).
`--parallel ep`: the experts are split over the ranks (expert parallelism);
rank r routes T >> r tokens of the largest microbatch (the last of three or
more ranks none), rows cross ranks in NCCL all-to-alls, whose time is
reported apart from the local kernels'.
`--impl reference` times the CPU oracle instead (rank 0 only; the other ranks
exit without work).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import socket
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

UNIT = "tokens/s"
HEADLINE = "uneven_sweep"
FORWARD_EXTRAS = ("dense_fwd", "fine_fwd_32k")


def metric_of(w) -> str:
    return "MoE layer fwd+bwd tokens/s" if w.backward else "MoE layer fwd tokens/s"


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
    """Flops (GEMM-like calls) or bytes (HBM-bound calls) of one call on a
    microbatch of T tokens."""
    d, E, k, f = w.d, w.E, w.k, w.f
    P = T * k
    b = 2 if w.dtype == "bf16" else 4
    flops = {
        "router_logits": 2.0 * T * d * E,
        "grouped_ffn_fwd": 6.0 * d * f * P,
        "grouped_ffn_recompute": 4.0 * d * f * P,
        "grouped_ffn_dgrad": 6.0 * d * f * P,
        "grouped_ffn_wgrad": 6.0 * d * f * P,
        "router_bwd": 2.0 * T * d * E,
    }
    # the fused-dispatch forms do the same arithmetic
    for n in ("grouped_ffn_fwd", "grouped_ffn_recompute", "grouped_ffn_wgrad", "router_bwd"):
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


GEMM_CALLS = ("grouped_ffn_fwd", "grouped_ffn_recompute", "grouped_ffn_dgrad", "grouped_ffn_wgrad")
MEM_CALLS = ("permute", "unpermute_combine", "unpermute_combine_bwd", "permute_bwd")


def _code_only(src: str) -> str:
    """C++ source without its comments and blank lines (string literals kept)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c == '"':  # string literal, copied as is
            j = i + 1
            while j < n and src[j] != '"':
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            while i < n and src[i] != "\n":
                i += 1
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = [ln.rstrip() for ln in "".join(out).splitlines()]
    return "\n".join(ln for ln in lines if ln.strip())


def source_hash() -> str:
    """Hash of the grouped GEMM's code (the kernel file and the headers it
    builds on, comments and blank lines left out): the committed DRAM
    counters of the kernel are used only while it matches."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "grouped_expert_ffn_top_b200", "csrc")
    for name in ("grouped_gemm_sm100.cu", "sm100.cuh", "common.cuh"):
        with open(os.path.join(csrc, name), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key: str, workload: str):
    """Per-launch DRAM bytes of the roofline kernel from the committed ncu
    summary for this workload, or None if absent or taken on another version
    of the kernel."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as fh:
            t = json.load(fh)
        ent = t[workload][kernel_key]
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
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows),
                "power_w_median": statistics.median(pw) if pw else None}


# ------------------------------------------------------------- CPU oracle

def oracle_step_fn(w, params_np, x_np, dY_np, aux_coef: float = 0.0):
    """One oracle pass over the first n tokens of a microbatch (a bounded
    sample): forward, and backward with every parameter gradient for a
    forward+backward workload; with a balance-loss coefficient, the loss and
    its metrics in the forward and its gradient in the backward."""
    import oracle

    def step(n: int):
        x = x_np[:n]
        P = params_np
        fw = oracle.layer_forward(x, P["Wr"], P["b"], P["Wg"], P["Wu"], P["Wd"], w.k, w.ep_groups)
        if aux_coef:
            oracle.aux_loss(fw["z"], fw["counts"], w.k, aux_coef)
        if w.backward:
            oracle.layer_backward(fw, x, dY_np[:n], P["Wr"], P["Wg"], P["Wu"], P["Wd"], w.k,
                                  aux=(aux_coef, 1.0) if aux_coef else None)
    return step


def oracle_inputs(w, seed: int = 0):
    """Workload params and the first microbatch on the host, in double."""
    import torch

    from grouped_expert_ffn_top_b200 import workloads
    p = workloads.make_params(w, device="cpu", seed=seed)
    bt = workloads.make_batch(w, device="cpu", seed=seed)
    P = {}
    for n in list(p):
        P[n] = p.pop(n).to(torch.float64).numpy()  # one tensor converted at a time
    return P, bt["x"].to(torch.float64).numpy(), bt["dY"].to(torch.float64).numpy()


def calibrate_sample(step, budget_s: float, T: int) -> int:
    """Token count whose oracle step takes about budget_s seconds: a linear
    fit (fixed cost + cost per token) through two probe sizes."""
    def timed(n):
        t0 = time.perf_counter()
        step(n)
        return max(time.perf_counter() - t0, 1e-4)

    step(min(2, T))  # first call: thread start-up and first touches of the weights
    n0 = min(8, T)
    t0 = timed(n0)
    n1 = int(max(min(2 * n0, T), min(T, n0 * 0.25 * budget_s / t0)))
    if n1 <= n0:
        return n0
    t1 = timed(n1)
    per_token = max((t1 - t0) / (n1 - n0), 1e-9)
    fixed = max(t0 - per_token * n0, 0.0)
    return int(max(1, min(T, (budget_s - fixed) / per_token)))


def _what(w, aux_coef: float = 0.0) -> str:
    what = "fwd+bwd (all parameter gradients)" if w.backward else "fwd"
    return what + (f" with the balance loss (coefficient {aux_coef})" if aux_coef else "")


def cpu_baseline(w, budget_s: float = 15.0, aux_coef: float = 0.0):
    import oracle
    P, x, dY = oracle_inputs(w)
    step = oracle_step_fn(w, P, x, dY, aux_coef)
    n = calibrate_sample(step, budget_s, w.T[0])
    t0 = time.perf_counter()
    step(n)
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"oracle {_what(w, aux_coef)} of the first {n} of the {w.T[0]} tokens of the first "
                      f"microbatch ({dt:.1f} s of CPU work)"}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    P, x, dY = oracle_inputs(w)
    step = oracle_step_fn(w, P, x, dY, args.aux_loss)
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
        "metric": metric_of(w), "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * dt / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        # the oracle runs on rank 0's host cores only: no GPU does any work
        "gpus_used": 0, "ranks_working": 1,
        "config": dict(workload_config(w), parallelism=f"{args.parallel}{args.gpus}"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"each step: oracle {_what(w, args.aux_loss)} of the first {n} tokens of the first "
                                   f"microbatch"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w):
    mbs = len(w.T)
    c = {"workload": w.name, "tokens_per_gpu": w.total_tokens, "microbatches": list(w.T),
         "d_model": w.d, "experts": w.E, "top_k": w.k, "ffn": w.f, "ep_groups": w.ep_groups,
         "routing": str(w.bias), "passes": "fwd+bwd" if w.backward else "fwd",
         "l2": "inputs larger than L2 (x alone is %.0f MB; a step moves several GB); no flush"
               % (max(w.T) * w.d * 2 / 1e6)}
    if w.backward:
        c["grads"] = ("the first microbatch writes the fp32 parameter gradients, the other %d add to "
                      "them (one optimizer step per sweep)" % (mbs - 1) if mbs > 1 else
                      "each step writes its own fp32 parameter gradients (one microbatch per "
                      "optimizer step)")
    return c


# ------------------------------------------------------------ ranks

def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def relaunch(argv, n: int) -> int:
    """Run this script again under torch.distributed.run with n ranks on this
    node (rendezvous on 127.0.0.1), bounded by an outer time limit; rank 0's
    JSON line reaches our stdout."""
    cmd = ["timeout", "-k", "60", "3600", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1", f"--master-port={_free_port()}",
           os.path.abspath(__file__)] + list(argv)
    return subprocess.run(cmd).returncode


class Ranks:
    """The benchmark's ranks (one process per GPU).

    In the data-parallel mode every rank draws its own microbatches (seed =
    rank) against the same weights; the only collectives are the barrier
    around the timed region and the max of the ranks' times, so nothing is
    exchanged on the data path."""

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


# ------------------------------------------------------------ end to end

def run_e2e(step_io, host, steps: int, dev, stream) -> float:
    """Milliseconds for `steps` steps fed from pinned host memory.

    host: pinned tensors of every microbatch's inputs, concatenated
    (x_all, and dY_all for a backward workload). Every step copies them
    host -> device and the outputs (Y_all, dX_all) device -> host inside the
    timed region. Copies run on their own streams with two device buffers per
    tensor, so step i+1's inputs arrive while step i computes and step i's
    outputs leave while step i+1 computes (the way a training loop feeds the
    layer). step_io(inputs, outputs) runs one step on device views."""
    import torch
    cin, cout = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    like = lambda t: torch.empty(t.shape, dtype=t.dtype, device=dev)
    ins = [[like(h) for h in host], [like(h) for h in host]]
    outs = [[like(h) for h in host], [like(h) for h in host]]
    back = [[torch.empty_like(h).pin_memory() for h in host] for _ in range(2)]
    in_ready, used, out_done = [None, None], [None, None], [None, None]

    def h2d(i):
        b = i % 2
        with torch.cuda.stream(cin):
            if used[b] is not None:
                cin.wait_event(used[b])  # step i-2 has finished reading this buffer
            for dst, src in zip(ins[b], host):
                dst.copy_(src, non_blocking=True)
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
        step_io(ins[b], outs[b])
        used[b] = torch.cuda.Event()
        used[b].record(stream)
        with torch.cuda.stream(cout):
            cout.wait_event(used[b])
            for dst, src in zip(back[b], outs[b]):
                dst.copy_(src, non_blocking=True)
            out_done[b] = torch.cuda.Event()
            out_done[b].record(cout)
    for ev in out_done:
        if ev is not None:
            stream.wait_event(ev)
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end)


# ------------------------------------------------------------ native arm

class Recorder:
    """CUDA events after each C call of the timed steps; durations per
    (microbatch, call) and per call summed over a step's microbatches."""

    def __init__(self, stream):
        self.stream = stream
        self.events = []  # (step, mb, name, event)
        self.step = 0
        self.mb = 0

    def mark(self, name):
        import torch
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(self.stream)
        self.events.append((self.step, self.mb, name, ev))

    def durations(self):
        per_step = {}   # name -> [ms per step]
        per_mb = {}     # (mb, name) -> [ms]
        for i in range(1, len(self.events)):
            s, mb, name, ev = self.events[i]
            if name == "step_start":
                continue
            ms = self.events[i - 1][3].elapsed_time(ev)
            per_mb.setdefault((mb, name), []).append(ms)
            d = per_step.setdefault(name, {})
            d[s] = d.get(s, 0.0) + ms
        call_ms = {n: statistics.mean(v.values()) for n, v in per_step.items()}
        mb_ms = {k: statistics.mean(v) for k, v in per_mb.items()}
        return call_ms, mb_ms


def _kernels_table(w, call_ms, hbm, bf16_burst, bf16_sust):
    from grouped_expert_ffn_top_b200.layer import LAUNCHES_PER_CALL
    kernels = {}
    for n, ms in call_ms.items():
        flops = sum(algorithmic_work(w, T)[0].get(n, 0.0) for T in w.T)
        bytes_ = sum(algorithmic_work(w, T)[1].get(n, 0.0) for T in w.T)
        ent = {"ms": round(ms, 4), "launches": LAUNCHES_PER_CALL.get(n, 1) * sum(1 for T in w.T if T > 0)}
        if flops and ms > 0:
            tf = flops / (ms * 1e-3) / 1e12
            ent.update({"tflops": round(tf, 1), "frac_bf16_burst": round(tf / bf16_burst, 3),
                        "frac_bf16_sustained": round(tf / bf16_sust, 3)})
        elif bytes_ and ms > 0:
            gbs = bytes_ / (ms * 1e-3) / 1e9
            ent.update({"gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                        "frac_8tbs": round(gbs / 8000.0, 3)})
        kernels[n] = ent
    return kernels


def time_layer(w, args, R, with_e2e: bool = True):
    """Times the workload's step through MoELayer on this rank; returns the
    measurements (rank-local except `total_ms` and `e2e_ms`, the max over
    ranks)."""
    import numpy as np
    import torch

    from grouped_expert_ffn_top_b200 import native as N
    from grouped_expert_ffn_top_b200 import workloads
    from grouped_expert_ffn_top_b200.layer import MoELayer

    dev = R.device
    params = workloads.make_params(w, device=dev, seed=0)
    batches = [workloads.make_batch(w, mb=mb, device=dev, seed=R.batch_seed) for mb in range(len(w.T))]
    fused = args.dispatch == "fused"
    layer = MoELayer(params, w.k, w.ep_groups, max_tokens=max(w.T), checkpoint=args.checkpoint,
                     fused_dispatch=fused, aux_coef=args.aux_loss)
    stream = torch.cuda.current_stream(dev)
    rec = Recorder(stream)

    def step(mark=None, xs=None, outs=None):
        for mb, bt in enumerate(batches):
            rec.mb = mb
            x = bt["x"] if xs is None else xs[0][mb]
            layer.forward(x, mark=mark, out=None if outs is None else outs[0][mb])
            if w.backward:
                dY = bt["dY"] if xs is None else xs[1][mb]
                # the first microbatch writes the parameter gradients, the rest add
                layer.backward(dY, mark=mark, accumulate=mb > 0, out=None if outs is None else outs[1][mb])

    for _ in range(args.warmup):
        step()
    R.barrier()
    errs = layer.device_errors()
    if errs:
        raise RuntimeError(f"device error word {errs} during warm-up")

    sampler = ClockSampler(R.local) if R.rank == 0 else None
    launches0 = N.moe_launch_count()
    R.barrier()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for s in range(args.steps):
        rec.step, rec.mb = s, 0
        rec.mark("step_start")
        step(mark=rec.mark)
    end.record(stream)
    R.barrier()
    clocks = sampler.stop() if sampler else None
    launches = N.moe_launch_count() - launches0
    total_ms = R.max_over_ranks(start.elapsed_time(end))
    call_ms, mb_ms = rec.durations()
    errs = layer.device_errors()
    if errs:
        raise RuntimeError(f"device error word {errs} in the timed region")

    out = {"total_ms": total_ms, "call_ms": call_ms, "mb_ms": mb_ms, "launches": launches, "clocks": clocks}
    if with_e2e:
        # every microbatch's x (and dY) in one pinned host tensor each; the
        # device step works on views of the copied buffers
        host = [torch.cat([bt["x"] for bt in batches]).cpu().pin_memory()]
        if w.backward:
            host.append(torch.cat([bt["dY"] for bt in batches]).cpu().pin_memory())
        bounds = np.concatenate([[0], np.cumsum(w.T)])

        def views(ts):
            return [[t[bounds[i]:bounds[i + 1]] for i in range(len(w.T))] for t in ts]

        def step_io(ins, outs):
            step(xs=views(ins), outs=views(outs))

        run_e2e(step_io, host, 2, dev, stream)
        R.barrier()
        out["e2e_ms"] = R.max_over_ranks(run_e2e(step_io, host, args.steps, dev, stream))
        out["h2d_bytes"] = int(sum(h.numel() * h.element_size() for h in host))
        out["d2h_bytes"] = out["h2d_bytes"]
        errs = layer.device_errors()
        if errs:
            raise RuntimeError(f"device error word {errs} in the e2e region")

    # routing load of the largest microbatch and the device memory the step
    # held (read after the timed regions): rerun its forward to read its counts
    big = int(np.argmax(w.T))
    layer.forward(batches[big]["x"])
    counts = layer.r["counts"].cpu().numpy().astype(np.int64)
    nonzero = counts[counts > 0]
    out["routing"] = {"microbatch_tokens": int(w.T[big]), "experts": int(counts.size),
                      "empty_experts": int((counts == 0).sum()), "rows_max": int(counts.max()),
                      "rows_min_nonzero": int(nonzero.min()) if nonzero.size else 0,
                      "max_over_mean": round(float(counts.max() / max(counts.mean(), 1e-9)), 3)}
    free_b, total_b = torch.cuda.mem_get_info(dev)
    out["memory"] = {"peak_allocated_gb": round(torch.cuda.max_memory_allocated(dev) / 1e9, 2),
                     "device_used_gb": round((total_b - free_b) / 1e9, 2),
                     "device_total_gb": round(total_b / 1e9, 1)}
    out["big_mb"] = big
    del layer, params, batches
    torch.cuda.empty_cache()
    return out


def forward_line(w, args, R):
    """Forward tokens/s of a forward-only workload (a sub-line of the
    headline: kernel durations and the grouped-GEMM fraction)."""
    hbm, bf16_burst, bf16_sust, _ = _peaks()
    m = time_layer(w, args, R, with_e2e=False)
    ms = m["total_ms"] / args.steps
    call_ms = m["call_ms"]
    gemm = "grouped_ffn_fwd" + ("_gather" if args.dispatch == "fused" else "")
    tf = sum(algorithmic_work(w, T)[0][gemm] for T in w.T) / (call_ms[gemm] * 1e-3) / 1e12
    return {"metric": metric_of(w), "value": round(R.world * w.total_tokens * args.steps / (m["total_ms"] * 1e-3), 1),
            "unit": UNIT, "ms_per_step": round(ms, 4),
            "config": workload_config(w),
            "grouped_gemm": {"tflops": round(tf, 1), "frac_bf16_burst": round(tf / bf16_burst, 3)},
            "kernels": _kernels_table(w, call_ms, hbm, bf16_burst, bf16_sust),
            "gpu_launches": int(m["launches"])}


def run_native(args, w):
    import torch

    from grouped_expert_ffn_top_b200 import native as N

    R = Ranks("nccl")
    N.lib()
    hbm, bf16_burst, bf16_sust, peak_src = _peaks()
    sfx = "_gather" if args.dispatch == "fused" else ""
    m = time_layer(w, args, R)
    call_ms, mb_ms = m["call_ms"], m["mb_ms"]
    kernels = _kernels_table(w, call_ms, hbm, bf16_burst, bf16_sust)

    ms_per_step = m["total_ms"] / args.steps
    value = R.world * w.total_tokens * args.steps / (m["total_ms"] * 1e-3)
    e2e_value = R.world * w.total_tokens * args.steps / (m["e2e_ms"] * 1e-3)
    line = {
        "metric": metric_of(w), "value": round(value, 1), "unit": UNIT, "n_gpus": R.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Gaussian activations and weights, router bias per workload)",
        "impl": "native",
        "config": dict(workload_config(w), parallelism=f"dp{R.world}"),
        # how this arm runs the layer (the workload is the same either way)
        "options": {"dispatch": ("fused: expert rows gathered from x inside the GEMM operand loads, "
                                 "no permuted copy" if sfx else "permute: rows copied to xp first"),
                    "activations": ("checkpointed: h1, h2 rebuilt in the backward" if args.checkpoint
                                    else "stored"),
                    "balance_loss": (f"coefficient {args.aux_loss}: loss, importance and entropy in the "
                                     "forward, its gradient in the backward" if args.aux_loss else "off")},
    }
    gemm_names = [n + s for n in GEMM_CALLS for s in ("", "_gather") if n + s in call_ms]
    if gemm_names:
        gemm_ms = sum(call_ms[n] for n in gemm_names)
        gemm_flops = sum(algorithmic_work(w, T)[0][n] for T in w.T for n in gemm_names)
        gemm_tf = gemm_flops / (gemm_ms * 1e-3) / 1e12
        line["grouped_gemm"] = {"tflops": round(gemm_tf, 1), "frac_bf16_burst": round(gemm_tf / bf16_burst, 3),
                                "frac_bf16_sustained": round(gemm_tf / bf16_sust, 3),
                                "share_of_step": round(gemm_ms / ms_per_step, 3)}
    mem = [n for n in MEM_CALLS if n in call_ms]
    if mem:
        mem_ms = sum(call_ms[n] for n in mem)
        mem_gbs = sum(algorithmic_work(w, T)[1][n] for T in w.T for n in mem) / (mem_ms * 1e-3) / 1e9
        line["permute_combine"] = {"gbs": round(mem_gbs, 1), "frac_hbm": round(mem_gbs / hbm, 3),
                                   "frac_8tbs": round(mem_gbs / 8000.0, 3)}
    # roofline: the dominant kernel's launch on the largest microbatch
    big = m["big_mb"]
    Tb = w.T[big]
    rk = ("grouped_ffn_wgrad" + sfx) if w.backward else ("grouped_ffn_fwd" + sfx)
    rk_ms = mb_ms[(big, rk)]
    rk_flops = algorithmic_work(w, Tb)[0][rk]
    rk_tf = rk_flops / (rk_ms * 1e-3) / 1e12
    # the peak for the way the kernel was timed: inside a timed region of a
    # second or more of back-to-back steps the GPU runs under its power cap,
    # which is where the sustained GEMM peak was measured; a shorter region
    # runs near the maximum clock (the burst peak)
    long_region = m["total_ms"] >= 1000.0
    peak = bf16_sust if long_region else bf16_burst
    line["roofline"] = {
        "kernel": f"{rk} (tcgen05 grouped GEMM{', ragged K' if 'wgrad' in rk else ''}), the launch on "
                  f"the {Tb}-token microbatch",
        "bound": "tensor", "achieved": round(rk_tf, 1), "peak": peak, "unit": "TFLOP/s",
        "frac": round(rk_tf / peak, 3),
        "frac_burst": round(rk_tf / bf16_burst, 3), "frac_sustained": round(rk_tf / bf16_sust, 3),
        "traffic": ncu_traffic(rk, w.name),
        "peak_source": (f"{peak_src} bf16 {'sustained' if long_region else 'burst'} "
                        f"({'timed inside %.1f s of back-to-back steps' % (m['total_ms'] / 1000.0) if long_region else 'timed region under 1 s'}); "
                        f"burst {bf16_burst}, sustained {bf16_sust}"),
        "algorithmic_flops_per_launch": rk_flops, "ms_per_launch": round(rk_ms, 4)}
    line["kernels"] = kernels
    line["kernels_by_microbatch"] = {
        str(w.T[mb]): {n: round(v, 4) for (b, n), v in sorted(mb_ms.items()) if b == mb}
        for mb in range(len(w.T)) if w.T[mb] > 0}
    line["e2e"] = {"value": round(e2e_value, 1), "unit": UNIT,
                   "h2d_bytes_per_step": m["h2d_bytes"], "d2h_bytes_per_step": m["d2h_bytes"],
                   "how": "every microbatch's x (and dY) copied from pinned host memory and Y (and dX) "
                          "copied back every step; copies on two copy streams, double-buffered so step "
                          "i+1's inputs arrive while step i computes"}
    line["gpu_launches"] = int(m["launches"])
    line["routing"] = m["routing"]
    line["memory"] = m["memory"]
    line["clocks"] = m["clocks"]
    if w.name == HEADLINE and not args.no_extras:
        from grouped_expert_ffn_top_b200 import workloads
        line["forward_only"] = {n: forward_line(workloads.WORKLOADS[n], args, R) for n in FORWARD_EXTRAS}
    if R.rank == 0 and R.world == 1 and not args.no_cpu_baseline:
        try:
            line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget, aux_coef=args.aux_loss)
        except Exception as ex:  # report, do not hide
            line["cpu_baseline"] = {"error": repr(ex)}
    if R.prints:
        print(json.dumps(line), flush=True)
    R.close()
    return 0


# ------------------------------------------------------- expert parallel arm

def ep_tokens(T: int, world: int):
    """Tokens of each rank in the expert-parallel mode: T >> r, and none on the
    last rank of three or more (uneven and empty per-rank work)."""
    n = [max(T >> r, 1) for r in range(world)]
    if world >= 3:
        n[-1] = 0
    return n


def run_ep(args, w):
    """Expert parallelism over NCCL: rank g owns experts [g E/N, (g+1) E/N),
    every rank routes its own tokens and the rows cross ranks in all-to-alls.
    The exchanges (with the small device-to-host copies of their split sizes)
    are timed apart from the local kernels."""
    import torch

    from grouped_expert_ffn_top_b200 import native as N
    from grouped_expert_ffn_top_b200 import workloads
    from grouped_expert_ffn_top_b200.ep import EPMoELayer

    R = Ranks("nccl")
    N.lib()
    if w.E % R.world:
        raise SystemExit(f"{w.E} experts do not split over {R.world} ranks")
    El = w.E // R.world
    dev = R.device
    full = workloads.make_params(w, device=dev, seed=0)
    lo = R.rank * El
    params = {"Wr": full["Wr"], "b": full["b"]}
    for n in ("Wg", "Wu", "Wd"):
        params[n] = full[n][lo:lo + El].contiguous()
    del full
    tok = ep_tokens(max(w.T), R.world)
    big = workloads.custom(w.name, [tok[R.rank]], w.d, w.E, w.k, w.f, dtype=w.dtype, bias=w.bias)
    bt = workloads.make_batch(big, device=dev, seed=R.batch_seed)
    layer = EPMoELayer(params, w.E, w.k)
    stream = torch.cuda.current_stream(dev)
    rec = Recorder(stream)

    def step(mark=None):
        layer.forward(bt["x"], mark=mark)
        layer.backward(bt["dY"], accumulate=False, mark=mark)

    for _ in range(args.warmup):
        step()
    R.barrier()
    R.barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    launches0 = N.moe_launch_count()
    start.record(stream)
    for s in range(args.steps):
        rec.step = s
        rec.mark("step_start")
        step(mark=rec.mark)
    end.record(stream)
    R.barrier()
    launches = N.moe_launch_count() - launches0
    total_ms = R.max_over_ranks(start.elapsed_time(end))
    call_ms, _ = rec.durations()
    exch = {n: v for n, v in call_ms.items() if n.startswith("a2a")}
    local_ms = sum(v for n, v in call_ms.items() if not n.startswith("a2a"))
    exch_ms = R.max_over_ranks(sum(exch.values()))
    local_ms = R.max_over_ranks(local_ms)
    value = sum(tok) * args.steps / (total_ms * 1e-3)
    line = {
        "metric": metric_of(w), "value": round(value, 1), "unit": UNIT, "n_gpus": R.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "impl": "native",
        "config": dict(workload_config(w), parallelism=f"ep{R.world}", tokens_per_rank=tok),
        "exchange_ms_per_step": round(exch_ms, 4), "local_ms_per_step": round(local_ms, 4),
        "exchanges": {n: round(v, 4) for n, v in exch.items()},
        "kernels": {n: round(v, 4) for n, v in call_ms.items() if not n.startswith("a2a")},
        "gpu_launches": int(launches),
    }
    if R.prints:
        print(json.dumps(line), flush=True)
    R.close()
    return 0


def main(argv=None):
    argv = sys.argv[1:] if argv is None else list(argv)
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--parallel", choices=["dp", "ep"], default="dp",
                    help="dp: data-parallel replicas (default); ep: experts split over the ranks")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the forward-only lines reported beside the headline workload")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--aux-loss", type=float, default=0.0,
                    help="Switch-style balance-loss coefficient: the forward also computes the loss "
                         "and the routing metrics, the backward adds its gradient (0: off)")
    ap.add_argument("--checkpoint", action="store_true",
                    help="activation checkpointing: h1, h2 rebuilt in the backward")
    ap.add_argument("--dispatch", choices=["permute", "fused"], default="permute",
                    help="permute: copy the dispatch rows to xp before the GEMMs; fused: gather them "
                         "from x inside the GEMMs' operand loads")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.aux_loss < 0:
        ap.error("--aux-loss must be non-negative")
    if args.aux_loss and args.parallel == "ep":
        ap.error("--aux-loss runs with the data-parallel layer (--parallel dp)")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1:
        return relaunch(argv, args.gpus)
    if env_world is not None and int(env_world) != args.gpus:
        ap.error(f"--gpus {args.gpus} but the launcher started WORLD_SIZE={env_world} ranks")
    from grouped_expert_ffn_top_b200 import workloads
    if args.workload not in workloads.WORKLOADS:
        ap.error(f"unknown workload {args.workload!r}; one of {sorted(workloads.WORKLOADS)}")
    w = workloads.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.parallel == "ep":
        if not w.backward:
            ap.error("--parallel ep runs forward+backward workloads")
        return run_ep(args, w)
    return run_native(args, w)


if __name__ == "__main__":
    sys.exit(main())
