"""bench.py's host-side logic on the CPU: the sizing of the oracle sample, the
algorithmic work the roofline divides by, and the workload description."""
import bench
from grouped_expert_ffn_top_b200 import workloads


def _fake_clock(monkeypatch, fixed, per_token):
    clock = [0.0]
    monkeypatch.setattr(bench.time, "perf_counter", lambda: clock[0])

    def step(n):
        clock[0] += fixed + per_token * n

    return step


def test_oracle_sample_fits_fixed_and_per_token_cost(monkeypatch):
    # a step of n tokens costs 0.5 s + 0.1 s per token: 145 tokens fill 15 s
    step = _fake_clock(monkeypatch, 0.5, 0.1)
    assert abs(bench.calibrate_sample(step, 15.0, 32768) - 145) <= 1


def test_oracle_sample_is_clamped_to_the_batch(monkeypatch):
    step = _fake_clock(monkeypatch, 0.0, 1e-6)
    assert bench.calibrate_sample(step, 15.0, 1000) == 1000
    step = _fake_clock(monkeypatch, 100.0, 1.0)  # even one token is over budget
    assert bench.calibrate_sample(step, 15.0, 1000) == 1


def test_algorithmic_work_of_the_bench_workload():
    w = workloads.WORKLOADS["fine_fwdbwd_32k"]
    T = w.T[0]
    P = T * w.k
    flops, bytes_ = bench.algorithmic_work(w, T)
    # each grouped GEMM call: three d x f products per dispatched row
    for n in ("grouped_ffn_fwd", "grouped_ffn_dgrad", "grouped_ffn_wgrad"):
        assert flops[n] == 6.0 * w.d * w.f * P
    # the fused-dispatch forms do the same arithmetic
    for n in ("grouped_ffn_fwd", "grouped_ffn_wgrad", "router_bwd"):
        assert flops[n + "_gather"] == flops[n]
    assert flops["router_logits"] == 2.0 * T * w.d * w.E
    # permute: x read once, k copies written, the row map read
    assert bytes_["permute"] == (T * w.d + P * w.d) * 2 + 4 * P


def test_workload_config_names_the_shape():
    w = workloads.WORKLOADS["fine_fwdbwd_32k"]
    c = bench.workload_config(w)
    assert c["workload"] == "fine_fwdbwd_32k"
    assert (c["tokens_per_gpu"], c["d_model"], c["experts"], c["top_k"], c["ffn"]) == (32768, 2048, 64, 8, 1408)
    assert "l2" in c


def test_workload_config_of_the_sweep_names_its_microbatches():
    w = workloads.WORKLOADS["uneven_sweep"]
    c = bench.workload_config(w)
    assert c["microbatches"] == [32768, 9000, 1, 0] and c["tokens_per_gpu"] == 41769
    assert "add to them" in c["grads"]
    assert bench.metric_of(w) == "MoE layer fwd+bwd tokens/s"
    assert bench.metric_of(workloads.WORKLOADS["dense_fwd"]) == "MoE layer fwd tokens/s"


def test_expert_parallel_ranks_get_uneven_work_and_one_empty_rank():
    assert bench.ep_tokens(32768, 1) == [32768]
    assert bench.ep_tokens(32768, 2) == [32768, 16384]
    assert bench.ep_tokens(32768, 4) == [32768, 16384, 8192, 0]


def _run_bench(args, env_extra=None, timeout=600):
    import os
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    env.update(env_extra or {})
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    return subprocess.run([sys.executable, os.path.join(root, "bench.py")] + args, capture_output=True,
                          text=True, timeout=timeout, env=env, cwd=root)


def test_gpus_two_without_a_launcher_starts_two_ranks():
    """`--gpus 2` re-executes bench.py under torch.distributed.run with two
    ranks; on the reference arm rank 0 times the oracle and reports n_gpus 2,
    the other rank exits without work."""
    import json
    r = _run_bench(["--impl", "reference", "--gpus", "2", "--workload", "tiny_fp32", "--steps", "3",
                    "--warmup", "3"])
    assert r.returncode == 0, r.stdout + r.stderr
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = lines[0]
    assert line["n_gpus"] == 2 and line["impl"] == "reference" and line["ranks_working"] == 1
    assert line["config"]["workload"] == "tiny_fp32" and line["value"] > 0


def test_gpus_must_match_the_launchers_world_size():
    r = _run_bench(["--impl", "reference", "--gpus", "2", "--workload", "tiny_fp32"],
                   env_extra={"WORLD_SIZE": "1", "RANK": "0", "LOCAL_RANK": "0"})
    assert r.returncode != 0
    assert "WORLD_SIZE=1" in r.stderr


def test_reference_arm_with_the_balance_loss():
    """`--aux-loss` reaches the reference arm: its oracle step computes the
    loss and adds its gradient, and the line says so."""
    import json
    r = _run_bench(["--impl", "reference", "--workload", "tiny_fp32", "--aux-loss", "0.01", "--steps", "3",
                    "--warmup", "3"])
    assert r.returncode == 0, r.stdout + r.stderr
    line = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")][0]
    assert "balance loss (coefficient 0.01)" in line["cpu_baseline"]["sample"]
    assert line["value"] > 0


def test_balance_loss_needs_the_data_parallel_layer():
    r = _run_bench(["--aux-loss", "0.01", "--parallel", "ep", "--workload", "tiny_fp32"])
    assert r.returncode != 0
    assert "--parallel dp" in r.stderr


def test_roofline_traffic_is_reported_only_for_the_kernel_it_was_taken_on(monkeypatch):
    """The committed DRAM bytes of the weight-gradient kernel are used while
    the grouped GEMM source hashes as it did at capture time, and dropped
    (None) once it changes."""
    import json
    import os
    with open(os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")) as fh:
        t = json.load(fh)
    for name, ent in t.items():
        e = ent["grouped_ffn_wgrad"]
        assert e["bytes_per_launch"] == int(round((e["dram_bytes_read_captured"] +
                                                   e["dram_bytes_write_captured"]) * e["scale"]))
        monkeypatch.setattr(bench, "source_hash", lambda h=e["source_hash"]: h)
        assert bench.ncu_traffic("grouped_ffn_wgrad", name) == float(e["bytes_per_launch"])
        monkeypatch.setattr(bench, "source_hash", lambda: "another kernel")
        assert bench.ncu_traffic("grouped_ffn_wgrad", name) is None
    assert bench.ncu_traffic("grouped_ffn_wgrad", "no such workload") is None


def test_kernel_hash_ignores_comments_but_not_code():
    code = 'asm volatile("tcgen05.commit // kept");  // the comment\n/* block */ int x = 1;\n\n'
    assert bench._code_only(code) == 'asm volatile("tcgen05.commit // kept");\n int x = 1;'
    assert bench._code_only(code.replace("the comment", "another one")) == bench._code_only(code)
    assert bench._code_only(code.replace("x = 1", "x = 2")) != bench._code_only(code)
