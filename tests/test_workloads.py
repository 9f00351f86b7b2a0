"""The seeded input generators: shapes, determinism and the load skew each
workload is meant to have (checked with the oracle's routing on the CPU)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from grouped_expert_ffn_top_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_shapes_and_dtypes():
    w = workloads.WORKLOADS["dense_fwd"]
    small = workloads.custom("s", 64, w.d, w.E, w.k, 256, bias=w.bias)
    p = workloads.make_params(small)
    assert p["Wr"].shape == (8, 1024) and p["Wr"].dtype == torch.bfloat16
    assert p["Wg"].shape == (8, 256, 1024) and p["Wd"].shape == (8, 1024, 256)
    assert p["b"].dtype == torch.float32
    bt = workloads.make_batch(small)
    assert bt["x"].shape == (64, 1024) and bt["dY"].shape == (64, 1024)


def test_deterministic():
    w = workloads.WORKLOADS["tiny_fp32"]
    a = workloads.make_params(w)
    b = workloads.make_params(w)
    for n in a:
        assert torch.equal(a[n], b[n])
    assert torch.equal(workloads.make_batch(w)["x"], workloads.make_batch(w)["x"])
    assert not torch.equal(workloads.make_batch(w, seed=1)["x"], workloads.make_batch(w)["x"])


def test_zipf_bias_starves_exactly_four_experts():
    w = workloads.WORKLOADS["fine_fwd_32k"]
    b = workloads.router_bias(w)
    assert int((b <= -1e4).sum()) == 4
    finite = b[b > -1e4]
    assert float(finite.max()) == 0.0  # rank 1 has bias -1.2 ln 1 = 0


def test_zipf_routing_is_skewed_on_a_token_sample():
    w = workloads.WORKLOADS["fine_fwd_32k"]
    p = workloads.make_params(workloads.custom("z", 2048, w.d, w.E, w.k, 64, bias="zipf"))
    x = workloads.make_batch(workloads.custom("z", 2048, w.d, w.E, w.k, 64, bias="zipf"))["x"]
    z = oracle.router_logits_f32(x.float().numpy(), p["Wr"].float().numpy(), p["b"].numpy())
    idx, _, _ = oracle.route(z.astype(np.float64), w.k)
    counts = np.bincount(idx.ravel(), minlength=w.E)
    assert (counts == 0).sum() >= 4
    assert counts.max() / counts.mean() > 4


def test_tiny_fp32_starves_last_expert_and_matches_golden():
    with open(os.path.join(GOLDEN, "tiny_fp32_routing.json")) as fh:
        g = json.load(fh)
    w = workloads.WORKLOADS["tiny_fp32"]
    p = workloads.make_params(w)
    bt = workloads.make_batch(w)
    z = oracle.router_logits_f32(bt["x"].numpy(), p["Wr"].numpy(), p["b"].numpy())
    idx, _, flags = oracle.route(z.astype(np.float64), w.k)
    lay = oracle.dispatch_layout(idx, w.E, w.ep_groups)
    assert lay["counts"].tolist() == g["counts"]
    assert lay["counts"][3] == 0
    assert lay["offsets"].tolist() == g["offsets"]
    assert lay["group_offsets"].tolist() == g["group_offsets"]
    assert idx[:16].tolist() == g["topk_idx_first16"]
    assert lay["pair_of_row"][:32].tolist() == g["pair_of_row_first32"]


def test_logits_generator_has_ties():
    z = workloads.make_logits(100, 16)
    row_has_tie = [(len(set(r.tolist())) < 16) for r in z]
    assert sum(row_has_tie) > 50


def test_sample_tokens_includes_required():
    s = workloads.sample_tokens(1000, 10, must_include=torch.tensor([3, 999]))
    assert 3 in s.tolist() and 999 in s.tolist()
    assert s.tolist() == sorted(set(s.tolist()))
