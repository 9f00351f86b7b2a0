"""A whole training step of the layer captured into one CUDA graph and
replayed. Every library call is asynchronous on its stream, allocates nothing
and reads the routing results (expert offsets, tile lists) on the device, so a
graph captured once stays valid while the routing changes from batch to batch:
each replay must equal an eager step on the same inputs bit for bit."""
import pytest
import torch

from grouped_expert_ffn_top_b200 import native as N
from grouped_expert_ffn_top_b200 import workloads
from grouped_expert_ffn_top_b200.layer import MoELayer

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    N.lib()


@pytest.mark.parametrize("dtype,fused,aux", [("bf16", False, 0.0), ("bf16", True, 0.0), ("bf16", False, 0.01),
                                             ("f32", False, 0.0)])
def test_captured_step_replays_like_eager_steps(dtype, fused, aux):
    T, d, E, k, f, G = (700, 256, 8, 2, 384, 2) if dtype == "bf16" else (200, 64, 4, 2, 128, 2)
    w = workloads.custom("graph", [T] * 3, d, E, k, f, dtype=dtype, bias=("normal", 0.5), ep_groups=G)
    p = workloads.make_params(w, device=DEV, seed=8)
    batches = [workloads.make_batch(w, mb=i, device=DEV, seed=8) for i in range(3)]
    eager = MoELayer(p, k, G, max_tokens=T, fused_dispatch=fused, aux_coef=aux)
    graphed = MoELayer(p, k, G, max_tokens=T, fused_dispatch=fused, aux_coef=aux)
    x = batches[0]["x"].clone()   # the graph's static inputs
    dY = batches[0]["dY"].clone()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # first calls (kernel attributes) outside the capture
        graphed.forward(x)
        graphed.backward(dY, accumulate=False)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        graphed.forward(x)
        graphed.backward(dY, accumulate=False)
    counts = []
    for b in batches:
        x.copy_(b["x"])
        dY.copy_(b["dY"])
        g.replay()
        eager.forward(b["x"])
        eager.backward(b["dY"], accumulate=False)
        torch.cuda.synchronize()
        assert graphed.device_errors() == 0 and eager.device_errors() == 0
        for n in ("logits", "h1", "h2", "a", "yp", "Y", "dyp", "dg", "dlogits", "dxp", "dX"):
            assert torch.equal(eager.v[n], graphed.v[n]), n
        for n in eager.grads:
            assert torch.equal(eager.grads[n], graphed.grads[n]), n
        counts.append(graphed.r["counts"].clone())
    # the replays really ran different routings through the one graph
    assert not all(torch.equal(counts[0], c) for c in counts[1:])
