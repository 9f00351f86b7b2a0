"""Parity at the full sizes of the four benchmark workloads, in the launch
configuration bench.py uses (MoELayer over preallocated buffers).

Checked in full: router logits, top-k indices, counts, offsets, group layout
and the permutation (bit for bit). Checked on samples the oracle computes one
by one: Y, dX, dg and the router logit gradient on 1024 tokens per
microbatch, which include every token of the microbatch's smallest non-empty
expert (the rest drawn at random), Y and dX compared with a scale per token; dWg / dWu rows and dWd columns on 64 columns of three experts (the
smallest non-empty, the median and the largest), summed over microbatches,
compared per expert. Checked by invariants at any size: sum_e db[e] = 0 and
sum_e dWr[e, :] = 0 (the softmax gradient sums to zero per token), empty
experts' dW stays 0.
"""
import numpy as np
import pytest
import torch

from grouped_expert_ffn_top_b200 import native as N
from grouped_expert_ffn_top_b200 import workloads
from grouped_expert_ffn_top_b200.layer import MoELayer
from parity import (TOL, assert_close, assert_close_per, check_routing_bitexact, oracle_routing,
                    sampled_forward_backward, sampled_wgrad, to_np)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    N.lib()


N_TOKENS = 1024  # sampled tokens per microbatch
N_COLS = 64      # sampled f columns per checked expert


def _sample(T, ref, n=N_TOKENS, seed=0):
    """n tokens (all of them if T <= n): every token of the smallest
    non-empty expert, then a seeded random choice of the others."""
    if T <= n:
        return np.arange(T)
    counts = ref["counts"]
    nonempty = np.nonzero(counts)[0]
    small = nonempty[np.argmin(counts[nonempty])]
    rows = ref["pair_of_row"][ref["offsets"][small]:ref["offsets"][small + 1]]
    must = np.unique(rows // ref["idx"].shape[1])
    assert must.size <= n, "the smallest expert's tokens alone exceed the sample"
    order = np.random.default_rng(seed + 505).permutation(T)
    rest = order[~np.isin(order, must)][: n - must.size]
    out = np.sort(np.concatenate([must, rest]))
    assert out.size == n and np.unique(out).size == n
    return out


@pytest.mark.parametrize("name", ["dense_fwd", "fine_fwd_32k", "fine_fwdbwd_32k", "uneven_sweep"])
def test_workload_full_size(name):
    w = workloads.WORKLOADS[name]
    tol = TOL[w.torch_dtype()]
    params = workloads.make_params(w, device=DEV, seed=0)
    layer = MoELayer(params, w.k, w.ep_groups, max_tokens=max(w.T))
    batches, routes = [], []
    for mb, T in enumerate(w.T):
        bt = workloads.make_batch(w, mb=mb, device=DEV, seed=0)
        Y = layer.forward(bt["x"])
        dX = layer.backward(bt["dY"]) if w.backward else None
        torch.cuda.synchronize()
        assert layer.device_errors() == 0
        if T == 0:
            assert Y.shape == (0, w.d)
            batches.append(bt)
            routes.append(None)
            continue
        ref = oracle_routing(bt["x"], params["Wr"], params["b"], w.k, w.ep_groups)
        check_routing_bitexact(layer.r, layer.v["logits"], ref)
        if w.bias == "zipf":
            assert (ref["counts"] == 0).sum() >= 4
        tokens = _sample(T, ref)
        o = sampled_forward_backward(bt["x"], bt["dY"], params, ref, tokens, w.k, backward=w.backward)
        ti = torch.as_tensor(tokens, dtype=torch.long, device=DEV)
        assert_close_per(f"{name}[{mb}] Y", Y[ti], o["Y"], tol)
        if w.backward:
            assert_close_per(f"{name}[{mb}] dX", dX[ti], o["dX"], tol)
            # dg and the logit gradient hold k (of E) values per token that can
            # all be near zero by cancellation: one scale over the sample
            assert_close(f"{name}[{mb}] dg", layer.v["dg"][ti], o["dg"], tol)
            assert_close(f"{name}[{mb}] dlogits", layer.v["dlogits"][ti], o["dz"], tol)
        batches.append(bt)
        routes.append(ref)
    if not w.backward:
        return
    g = layer.grads
    # weight gradients on sampled columns of three experts, over all microbatches
    total = sum(r["counts"] for r in routes if r is not None)
    nonempty = np.nonzero(total)[0]
    order = nonempty[np.argsort(total[nonempty], kind="stable")]
    experts = sorted({int(order[0]), int(order[len(order) // 2]), int(order[-1])})
    cols = workloads.sample_tokens(w.f, N_COLS, seed=1).numpy()
    assert cols.size == N_COLS
    live = [(b, r) for b, r in zip(batches, routes) if r is not None]
    for e in experts:
        og, ou, od = sampled_wgrad([b for b, _ in live], params, [r for _, r in live], w.k, e, cols)
        ci = torch.as_tensor(cols, dtype=torch.long, device=DEV)
        # one scale per expert: these three are the three experts' own slices
        assert_close_per(f"dWg[{e}]", g["dWg"][e][ci][None], og[None], tol)
        assert_close_per(f"dWu[{e}]", g["dWu"][e][ci][None], ou[None], tol)
        assert_close_per(f"dWd[{e}]", g["dWd"][e][:, ci].T[None], od[None], tol)
    empty = np.nonzero(total == 0)[0]
    for e in empty:
        for n in ("dWg", "dWu", "dWd"):
            assert not g[n][int(e)].any()
    # invariants of the router gradient at any size
    db = to_np(g["db"]).astype(np.float64)
    assert abs(db.sum()) <= 1e-3 * np.abs(db).sum() + 1e-6
    dWr = to_np(g["dWr"]).astype(np.float64)
    assert np.abs(dWr.sum(0)).max() <= 1e-3 * np.abs(dWr).sum(0).max() + 1e-6
