"""Fused dispatch: the expert GEMMs and the router backward read the dispatch
rows in place from x through pair_of_row (cp.async row gathers on the bf16 path)
instead of from the permuted copy xp.

Dispatch row r is x[pair_of_row[r] / k], the row the permute copies to xp[r],
so the MMAs see the same bf16 values in the same order: every output and
gradient must equal the permuted path's bit for bit. The permuted path itself
is held to the oracle by the other parity tests; here the fused layer is also
checked against the oracle directly on one small case.
"""
import numpy as np
import pytest
import torch

import oracle
from grouped_expert_ffn_top_b200 import native as N
from grouped_expert_ffn_top_b200 import workloads
from grouped_expert_ffn_top_b200.layer import MoELayer
from parity import TOL, assert_close, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    N.lib()


SAVED = ("logits", "h1", "h2", "a", "yp", "Y", "dyp", "dg", "dlogits", "dxp", "dh1", "dh2", "dX")


def _assert_layers_equal(ref: MoELayer, fused: MoELayer, what: str):
    for n in SAVED:
        assert torch.equal(ref.v[n], fused.v[n]), f"{what}: {n}"
    for n in ref.grads:
        assert torch.equal(ref.grads[n], fused.grads[n]), f"{what}: {n}"


CASES = [
    # name, T, d, E, k, f, dtype, G, starve_last
    ("bf16_two_tiles", 700, 256, 8, 2, 384, "bf16", 2, True),
    ("bf16_ragged", 333, 192, 5, 3, 320, "bf16", 1, False),
    ("bf16_single_token", 1, 128, 4, 2, 128, "bf16", 2, False),
    ("bf16_long_k", 2048, 512, 4, 1, 256, "bf16", 1, True),
    ("bf16_f_not_256", 520, 320, 6, 2, 448, "bf16", 3, True),
    ("bf16_many_experts", 900, 128, 160, 4, 192, "bf16", 8, True),
    ("bf16_k8", 1500, 256, 64, 8, 192, "bf16", 4, True),
    # d and f multiples of 8 only: the last K block of the gathered rows is
    # zero-filled past d, the last column tiles are masked
    ("bf16_d1000_f1400", 300, 1000, 6, 2, 1400, "bf16", 2, True),
    ("bf16_d72_f40", 333, 72, 5, 2, 40, "bf16", 1, False),
    ("f32_tiny", 256, 64, 4, 2, 128, "f32", 2, True),
    ("f32_odd", 100, 48, 3, 2, 20, "f32", 1, False),
]


def _case(T, d, E, k, f, dtype, G, starve, seed=0):
    # four microbatches of T tokens (tests use one or several)
    w = workloads.custom("fused", [T] * 4, d, E, k, f, dtype=dtype, bias=("normal", 0.5), ep_groups=G)
    p = workloads.make_params(w, device=DEV, seed=seed)
    if starve:
        p["b"][E - 1] = -1.0e4
    return w, p


@pytest.mark.parametrize("checkpoint", [False, True], ids=["stored", "checkpointed"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_fused_layer_is_bitwise_the_permuted_layer(case, checkpoint):
    """Two microbatches (written, then accumulated): every activation, output
    and gradient of the fused layer equals the permuted layer's."""
    _, T, d, E, k, f, dtype, G, starve = case
    w, p = _case(T, d, E, k, f, dtype, G, starve)
    ref = MoELayer(p, k, G, max_tokens=T, checkpoint=checkpoint)
    fused = MoELayer(p, k, G, max_tokens=T, checkpoint=checkpoint, fused_dispatch=True)
    assert fused.buf["xp"].numel() == 0  # no permuted copy is kept
    for mb in range(2):
        bt = workloads.make_batch(w, mb=mb, device=DEV, seed=mb + 3)
        for layer in (ref, fused):
            layer.forward(bt["x"])
            layer.backward(bt["dY"], accumulate=mb > 0)
        torch.cuda.synchronize()
        assert ref.device_errors() == 0 and fused.device_errors() == 0
        _assert_layers_equal(ref, fused, f"microbatch {mb}")


def test_fused_layer_matches_oracle():
    T, d, E, k, f, G = 700, 256, 8, 2, 384, 2
    w, p = _case(T, d, E, k, f, "bf16", G, True)
    bt = workloads.make_batch(w, device=DEV, seed=11)
    layer = MoELayer(p, k, G, max_tokens=T, fused_dispatch=True)
    Y = layer.forward(bt["x"])
    dX = layer.backward(bt["dY"], accumulate=False)
    torch.cuda.synchronize()
    assert layer.device_errors() == 0
    P = {n: to_np(v).astype(np.float64) for n, v in p.items()}
    x64 = to_np(bt["x"]).astype(np.float64)
    fw = oracle.layer_forward(x64, P["Wr"], P["b"], P["Wg"], P["Wu"], P["Wd"], k, G)
    bw = oracle.layer_backward(fw, x64, to_np(bt["dY"]).astype(np.float64), P["Wr"], P["Wg"], P["Wu"],
                               P["Wd"], k)
    tol = TOL[torch.bfloat16]
    for n in ("h1", "h2", "a", "yp"):
        assert_close(n, layer.v[n], fw[n], tol)
    assert_close("Y", Y, fw["Y"], tol)
    assert_close("dX", dX, bw["dX"], tol)
    for n in ("dWg", "dWu", "dWd", "dWr", "db"):
        assert_close(n, layer.grads[n], bw[n], tol)
    assert not layer.grads["dWg"][E - 1].any()


def test_empty_and_single_token_microbatches():
    T, d, E, k, f = 64, 128, 4, 2, 128
    w, p = _case(T, d, E, k, f, "bf16", 1, False)
    ref = MoELayer(p, k, 1, max_tokens=T)
    fused = MoELayer(p, k, 1, max_tokens=T, fused_dispatch=True)
    for mb, n in enumerate([0, 1, 0, T]):
        x = workloads.make_batch(w, mb=mb, device=DEV, seed=mb)["x"][:n]
        dY = workloads.make_batch(w, mb=mb, device=DEV, seed=mb + 50)["dY"][:n]
        for layer in (ref, fused):
            layer.forward(x)
            layer.backward(dY, accumulate=mb > 0)
        torch.cuda.synchronize()
        for g in ref.grads:
            assert torch.equal(ref.grads[g], fused.grads[g]), (mb, g)
        if n:
            assert torch.equal(ref.v["Y"], fused.v["Y"]) and torch.equal(ref.v["dX"], fused.v["dX"])


def test_gathered_entries_called_directly():
    """The four gathered entry points against moe_permute plus the plain ones,
    including the write (accumulate = 0) form with an expert that has no rows."""
    T, d, E, k, f = 600, 256, 6, 2, 256
    w, p = _case(T, d, E, k, f, "bf16", 1, True)
    bt = workloads.make_batch(w, device=DEV, seed=5)
    x = bt["x"]
    z = N.moe_router_logits(x, p["Wr"], p["b"])
    r = N.moe_route(z, k, 1)
    xp = N.moe_permute(x, r["row_of_pair"], k)
    o_ref = N.moe_grouped_ffn_fwd(xp, p["Wg"], p["Wu"], p["Wd"], r["offsets"])
    o_g = N.moe_grouped_ffn_fwd_gather(x, r["pair_of_row"], k, p["Wg"], p["Wu"], p["Wd"], r["offsets"])
    # checkpointed form: h1, h2 not stored, then rebuilt
    ck = {n: torch.full_like(o_ref[n], float("nan")) for n in o_ref}
    ck["h1"] = ck["h2"] = None
    N.moe_grouped_ffn_fwd_gather(x, r["pair_of_row"], k, p["Wg"], p["Wu"], p["Wd"], r["offsets"], out=ck)
    h1 = torch.empty_like(o_ref["h1"])
    h2 = torch.empty_like(o_ref["h2"])
    N.moe_grouped_ffn_recompute_gather(x, r["pair_of_row"], k, p["Wg"], p["Wu"], r["offsets"], h1, h2)
    torch.cuda.synchronize()
    for n in ("h1", "h2", "a", "yp"):
        assert torch.equal(o_ref[n], o_g[n]), n
    assert torch.equal(ck["a"], o_ref["a"]) and torch.equal(ck["yp"], o_ref["yp"])
    assert torch.equal(h1, o_ref["h1"]) and torch.equal(h2, o_ref["h2"])

    gen = torch.Generator(device=DEV).manual_seed(9)
    dyp = torch.randn(o_ref["yp"].shape, generator=gen, device=DEV).to(torch.bfloat16)
    rows = T * k
    ws = N._ws(N.moe_grouped_ffn_bwd_workspace_bytes(rows, E, d, f, N.MOE_BF16), DEV)
    dh1 = torch.empty_like(h1)
    dh2 = torch.empty_like(h2)
    dxp = torch.empty_like(xp)
    N.moe_grouped_ffn_dgrad(p["Wg"], p["Wu"], p["Wd"], h1, h2, dyp, r["offsets"], dh1, dh2, dxp, ws)
    for acc in (False, True):
        gr = [torch.full((E, f, d), 3.0, device=DEV), torch.full((E, f, d), 3.0, device=DEV),
              torch.full((E, d, f), 3.0, device=DEV)]
        gg = [t.clone() for t in gr]
        N.moe_grouped_ffn_wgrad(xp, o_ref["a"], dyp, dh1, dh2, r["offsets"], *gr, ws, accumulate=acc)
        N.moe_grouped_ffn_wgrad_gather(x, r["pair_of_row"], k, o_ref["a"], dyp, dh1, dh2, r["offsets"], *gg, ws,
                                       accumulate=acc)
        torch.cuda.synchronize()
        for a_, b_ in zip(gr, gg):
            assert torch.equal(a_, b_), acc
        if not acc:  # the starved expert's gradient is written as zeros
            assert not gg[0][E - 1].any()
        # and the one-call backward
        dxp2 = torch.empty_like(xp)
        g2 = [t.clone().fill_(3.0) for t in gr]
        N.moe_grouped_ffn_bwd_gather(x, r["pair_of_row"], k, p["Wg"], p["Wu"], p["Wd"], h1, h2, o_ref["a"], dyp,
                                     r["offsets"], *g2, dxp=dxp2, accumulate=acc)
        torch.cuda.synchronize()
        assert torch.equal(dxp2, dxp)
        for a_, b_ in zip(gr, g2):
            assert torch.equal(a_, b_), acc

    dz = N.moe_route_bwd(torch.randn((T, k), generator=gen, device=DEV), r["topk_w"], r["topk_idx"], E)
    for acc in (False, True):
        wr = [torch.full((E, d), 2.0, device=DEV), torch.full((E,), 2.0, device=DEV)]
        wg = [t.clone() for t in wr]
        N.moe_router_bwd(xp, dz, r["pair_of_row"], r["offsets"], k, *wr, accumulate=acc)
        N.moe_router_bwd_gather(x, dz, r["pair_of_row"], r["offsets"], k, *wg, accumulate=acc)
        torch.cuda.synchronize()
        assert torch.equal(wr[0], wg[0]) and torch.equal(wr[1], wg[1])


@pytest.mark.parametrize("name", ["fine_fwdbwd_32k", "uneven_sweep"])
def test_fused_layer_full_size_is_bitwise_the_permuted_layer(name):
    """At the benchmark workloads' full sizes (the permuted layer is checked
    against the oracle there by the workload tests)."""
    w = workloads.WORKLOADS[name]
    params = workloads.make_params(w, device=DEV, seed=0)
    ref = MoELayer(params, w.k, w.ep_groups, max_tokens=max(w.T))
    fused = MoELayer(params, w.k, w.ep_groups, max_tokens=max(w.T), fused_dispatch=True)
    for mb, T in enumerate(w.T):
        bt = workloads.make_batch(w, mb=mb, device=DEV, seed=0)
        for layer in (ref, fused):
            layer.forward(bt["x"])
            layer.backward(bt["dY"], accumulate=mb > 0)
        torch.cuda.synchronize()
        assert ref.device_errors() == 0 and fused.device_errors() == 0
        if T:
            for n in SAVED:
                assert torch.equal(ref.v[n], fused.v[n]), f"{name}[{mb}] {n}"
    for n in ref.grads:
        assert torch.equal(ref.grads[n], fused.grads[n]), f"{name} {n}"
