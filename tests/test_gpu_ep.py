"""Expert parallelism on one GPU: with one rank the expert-parallel layer's
exchanges are identities, so through the library's kernels it must give the
plain layer's results bit for bit, with no process group and through a
one-rank NCCL group (which runs the real all-to-all calls); and its results
must match the oracle's layer directly."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from grouped_expert_ffn_top_b200 import native as N
from grouped_expert_ffn_top_b200 import workloads
from grouped_expert_ffn_top_b200.ep import EPMoELayer
from grouped_expert_ffn_top_b200.layer import MoELayer

import oracle
from parity import TOL, assert_close, assert_close_per, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    N.lib()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _compare(with_group: bool):
    T, d, E, k, f = 700, 256, 8, 2, 384
    w = workloads.custom("ep1", T, d, E, k, f, bias=("normal", 0.5))
    p = workloads.make_params(w, device=DEV, seed=8)
    p["b"][E - 1] = -1.0e4
    bt = workloads.make_batch(w, device=DEV, seed=8)
    ref = MoELayer(p, k, 1, max_tokens=T)
    Y0 = ref.forward(bt["x"]).clone()
    dX0 = ref.backward(bt["dY"], accumulate=False).clone()
    if with_group:
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                                world_size=1)
    try:
        ep = EPMoELayer(p, E, k)
        Y1 = ep.forward(bt["x"])
        dX1 = ep.backward(bt["dY"], accumulate=False)
        torch.cuda.synchronize()
    finally:
        if with_group:
            dist.destroy_process_group()
    assert torch.equal(Y0, Y1)
    assert torch.equal(dX0, dX1)
    for n in ref.grads:
        assert torch.equal(ref.grads[n], ep.grads[n]), n
    # the expert-parallel layer against the oracle's layer
    tol = TOL[torch.bfloat16]
    P = {n: to_np(v).astype(np.float64) for n, v in p.items()}
    x64 = to_np(bt["x"]).astype(np.float64)
    fw = oracle.layer_forward(x64, P["Wr"], P["b"], P["Wg"], P["Wu"], P["Wd"], k)
    bw = oracle.layer_backward(fw, x64, to_np(bt["dY"]).astype(np.float64), P["Wr"], P["Wg"], P["Wu"],
                               P["Wd"], k)
    assert_close_per("Y", Y1, fw["Y"], tol)
    assert_close_per("dX", dX1, bw["dX"], tol)
    for n in ("dWg", "dWu", "dWd"):
        assert_close_per(n, ep.grads[n], bw[n], tol)
    for n in ("dWr", "db"):
        assert_close(n, ep.grads[n], bw[n], tol)


def test_one_rank_expert_parallel_layer_is_the_plain_layer():
    _compare(with_group=False)


def test_one_rank_nccl_expert_parallel_layer_is_the_plain_layer():
    _compare(with_group=True)


@pytest.mark.parametrize("G,El,zero", [(1, 8, False), (2, 4, False), (4, 16, False), (8, 2, False),
                                       (3, 5, False), (16, 64, False), (4, 4, True)])
def test_device_regroup_map_is_the_stable_sort_by_expert_then_source(G, El, zero):
    """moe_ep_regroup against an independent definition: received row i
    (arrival order: source, then local expert, then position) goes to its rank
    in the order (local expert, source, position)."""
    rng = np.random.default_rng(G * 100 + El)
    counts = rng.integers(0, 50, size=(G, El)).astype(np.int32)
    counts[rng.random((G, El)) < 0.3] = 0
    if zero:
        counts[:] = 0
    rows = int(counts.sum())
    m, off = N.moe_ep_regroup(torch.as_tensor(counts, device=DEV), rows)
    torch.cuda.synchronize()
    flat = counts.reshape(-1)
    src = np.repeat(np.arange(G * El) // El, flat)
    exp = np.repeat(np.arange(G * El) % El, flat)
    pos = np.concatenate([np.arange(c) for c in flat]) if rows else np.zeros(0, np.int64)
    order = np.lexsort((pos, src, exp))  # primary key: expert, then source, then position
    dest = np.empty(rows, np.int64)
    dest[order] = np.arange(rows)
    assert np.array_equal(to_np(m).astype(np.int64), dest)
    assert np.array_equal(to_np(off), np.concatenate([[0], np.cumsum(counts.sum(axis=0))]))
