"""GPU parity: every step of the layer, through the C ABI, against the oracle.

Integer results (top-k indices, counts, offsets, groups, permutation) and the
fp32 router logits must match bit for bit; float results must be within the
normwise tolerance of tests/parity.py. Sizes span several 128-row tiles and
ragged tails; edge cases cover T = 0 and T = 1, starved experts, ties and
non-finite logits.
"""
import numpy as np
import pytest
import torch

import oracle
from grouped_expert_ffn_top_b200 import native as N
from grouped_expert_ffn_top_b200 import workloads
from grouped_expert_ffn_top_b200.layer import MoELayer
from parity import TOL, assert_close, assert_close_per, check_routing_bitexact, oracle_routing, rel_err, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    N.lib()


# ------------------------------------------------------------------ routing

@pytest.mark.parametrize("T,E,k,G", [(1, 4, 2, 2), (255, 8, 2, 1), (256, 8, 2, 2), (257, 64, 8, 4),
                                     (5000, 64, 8, 4), (3000, 16, 2, 1), (1000, 128, 4, 8),
                                     (600, 1024, 8, 16), (100, 33, 32, 1), (70, 40, 1, 5)])
def test_route_bitexact_on_tied_logits(T, E, k, G):
    z = workloads.make_logits(T, E, seed=T * 7 + E)
    out = N.moe_route(z.to(DEV), k, G)
    idx, w, flags = oracle.route(z.double().numpy(), k)
    lay = oracle.dispatch_layout(idx, E, G)
    check_routing_bitexact(out, None, dict(idx=idx, w=w, **lay), check_logits=False)


def test_route_nonfinite_logits_raise_the_device_flag():
    inf, nan = float("inf"), float("nan")
    z = workloads.make_logits(300, 16, seed=5, specials=True)
    z[7, :] = -inf                       # all selected -inf: undefined, 1/k
    z[9, 3] = nan                        # NaN outside the selection: ignored
    z[11, :] = -inf
    z[11, 2], z[11, 5] = 1.0, 2.0        # two finite then -inf: defined, zeros
    z[13, 4] = inf                       # +inf selected: undefined
    z[15, :] = nan
    z[15, 0] = 0.5                       # NaN selected: undefined
    ws = N._ws(N.moe_route_workspace_bytes(300, 16), DEV)
    out = N.moe_route(z.to(DEV), 4, 1, ws=ws)
    assert N.moe_get_error(ws) & N.MOE_DEVERR_NONFINITE_LOGIT
    assert N.moe_get_error(ws) == 0  # cleared by the read
    idx, w, flags = oracle.route(z.double().numpy(), 4)
    assert flags & oracle.FLAG_NONFINITE
    assert np.array_equal(to_np(out["topk_idx"]), idx)
    gw = to_np(out["topk_w"])
    assert np.abs(gw - w).max() <= 1e-6
    for t in (7, 13, 15):
        assert np.array_equal(gw[t], np.full(4, 0.25, np.float32)), t
    assert gw[11, 2] == 0.0 and gw[11, 3] == 0.0 and abs(gw[11, 0] - 0.7310586) < 1e-6


def test_route_with_selected_minus_inf_is_a_defined_softmax():
    """-inf logits inside the selection next to finite ones: exact softmax
    (zero weight on the -inf slots), no device flag."""
    z = workloads.make_logits(500, 8, seed=6)
    z[::3, 2:] = -float("inf")           # only experts 0 and 1 finite, k = 4
    ws = N._ws(N.moe_route_workspace_bytes(500, 8), DEV)
    out = N.moe_route(z.to(DEV), 4, 2, ws=ws)
    assert N.moe_get_error(ws) == 0
    idx, w, flags = oracle.route(z.double().numpy(), 4)
    assert flags == 0
    lay = oracle.dispatch_layout(idx, 8, 2)
    check_routing_bitexact(out, None, dict(idx=idx, w=w, **lay), check_logits=False)
    assert not to_np(out["topk_w"])[::3, 2:].any()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d,E", [(1, 64, 4), (300, 264, 8), (129, 1024, 16), (1000, 512, 64),
                                   (77, 128, 100), (3, 4096, 16), (5000, 256, 16), (700, 136, 12),
                                   (4096, 64, 1), (600, 200, 24), (2000, 128, 32), (500, 96, 40)])
def test_router_logits_bitexact(dtype, T, d, E):
    """Bit-exact with the oracle's fixed-order fp32 logits on both kernels: one
    thread per logit for T E <= 4096, the 64-token tiles above it."""
    w = workloads.custom("l", T, d, E, 1, 64, dtype="bf16" if dtype == torch.bfloat16 else "f32")
    p = workloads.make_params(w, device=DEV, seed=T + d)
    x = workloads.make_batch(w, device=DEV, seed=E)["x"]
    z = N.moe_router_logits(x, p["Wr"], p["b"])
    ref = oracle.router_logits_f32(to_np(x), to_np(p["Wr"]), to_np(p["b"]))
    assert np.array_equal(to_np(z), ref)


# --------------------------------------------------------- whole layer

LAYER_CASES = [
    # name, T, d, E, k, f, dtype, G, starve_last
    ("bf16_two_tiles", 700, 256, 8, 2, 384, "bf16", 2, True),
    ("bf16_ragged", 333, 192, 5, 3, 320, "bf16", 1, False),
    ("bf16_single_token", 1, 128, 4, 2, 128, "bf16", 2, False),
    ("bf16_long_k", 2048, 512, 4, 1, 256, "bf16", 1, True),
    ("bf16_f_not_256", 520, 320, 6, 2, 448, "bf16", 3, True),
    # more experts than the deepest GEMM pipeline leaves schedule room for
    ("bf16_many_experts", 900, 128, 160, 4, 192, "bf16", 8, True),
    # d and f multiples of 8 but not of 64: ragged last K blocks (zero-filled by
    # TMA, weight rows past an expert's matrix included) and masked last column
    # tiles, at 8-column granularity (1000 = 15 * 64 + 40, 1400 = 21 * 64 + 56;
    # f = 40 is less than one K block and one 16-column store group)
    ("bf16_d1000_f1400", 300, 1000, 6, 2, 1400, "bf16", 2, True),
    ("bf16_d72_f40", 333, 72, 5, 2, 40, "bf16", 1, False),
    ("bf16_d136_f1032", 1100, 136, 3, 2, 1032, "bf16", 1, True),
    # the largest sizes the boundary accepts: MOE_MAX_EXPERTS experts (most of
    # them with no row or a handful, every GEMM's tile schedule at its
    # largest), and top-32 (the largest k of the routing and combine kernels)
    ("bf16_max_experts", 600, 128, 1024, 8, 64, "bf16", 16, True),
    ("bf16_top32", 200, 128, 64, 32, 128, "bf16", 4, False),
    # the GEMMs' tile orders for operands that do not fit in L2 beside each
    # other: K ranges of the down projection (f) and of the input gradient
    # (2f) too long for 16 row tiles of 256 rows (groups of 8, with 9 row
    # tiles per expert), and an expert whose d-side operand (2 d rows bytes,
    # 52 MB here) is too large to stay resident in the weight gradient
    ("bf16_long_k_row_groups", 2200, 64, 2, 2, 6400, "bf16", 1, False),
    ("bf16_wgrad_large_expert", 6300, 4096, 2, 1, 264, "bf16", 1, True),
    ("f32_tiny", 256, 64, 4, 2, 128, "f32", 2, True),
    ("f32_odd", 100, 48, 3, 2, 20, "f32", 1, False),
]


def _layer_case(T, d, E, k, f, dtype, G, starve, seed=0):
    w = workloads.custom("case", T, d, E, k, f, dtype=dtype, bias=("normal", 0.5), ep_groups=G)
    p = workloads.make_params(w, device=DEV, seed=seed)
    if starve:
        p["b"][E - 1] = -1.0e4
    bt = workloads.make_batch(w, device=DEV, seed=seed)
    return w, p, bt


def _np_params(p):
    return {n: to_np(v).astype(np.float64) for n, v in p.items()}


@pytest.mark.parametrize("case", LAYER_CASES, ids=[c[0] for c in LAYER_CASES])
def test_layer_forward_backward_matches_oracle(case):
    _, T, d, E, k, f, dtype, G, starve = case
    w, p, bt = _layer_case(T, d, E, k, f, dtype, G, starve)
    tol = TOL[w.torch_dtype()]
    layer = MoELayer(p, k, G, max_tokens=T)
    Y = layer.forward(bt["x"])
    dX = layer.backward(bt["dY"])
    torch.cuda.synchronize()
    assert layer.device_errors() == 0

    ref_route = oracle_routing(bt["x"], p["Wr"], p["b"], k, G)
    check_routing_bitexact(layer.r, layer.v["logits"], ref_route)
    if starve:
        assert ref_route["counts"][E - 1] == 0

    P = _np_params(p)
    x64 = to_np(bt["x"]).astype(np.float64)
    dY64 = to_np(bt["dY"]).astype(np.float64)
    fw = oracle.layer_forward(x64, P["Wr"], P["b"], P["Wg"], P["Wu"], P["Wd"], k, G)
    assert np.array_equal(fw["idx"], ref_route["idx"])
    bw = oracle.layer_backward(fw, x64, dY64, P["Wr"], P["Wg"], P["Wu"], P["Wd"], k)

    # scales: per dispatch row (h1, h2, a, yp, dyp, dxp), per token (Y, dX),
    # per expert (dWg, dWu, dWd); dg, dlogits, dWr and db, built from the logit
    # gradient g (dg - sum g dg), whose few values per token can all be near
    # zero by cancellation (an expert with one token has dWr = dz x), with one
    # scale
    v = layer.v
    assert np.array_equal(to_np(v["xp"]), fw["xp"]), "permute must copy rows exactly"
    for n in ("h1", "h2", "a", "yp"):
        assert_close_per(n, v[n], fw[n], tol)
    assert_close_per("Y", Y, fw["Y"], tol)
    assert_close_per("dyp", v["dyp"], bw["dyp"], tol)
    assert_close("dg", v["dg"], bw["dg"], tol)
    assert_close("dlogits", v["dlogits"], bw["dz"], tol)
    assert_close_per("dxp", v["dxp"], bw["dxp"], tol)
    assert_close_per("dX", dX, bw["dX"], tol)
    g = layer.grads
    for n in ("dWg", "dWu", "dWd"):
        assert_close_per(n, g[n], bw[n], tol)
    for n in ("dWr", "db"):
        assert_close(n, g[n], bw[n], tol)
    if starve:
        for n in ("dWg", "dWu", "dWd"):
            assert not g[n][E - 1].any(), f"{n} of the starved expert must stay exactly zero"


def test_microbatches_accumulate_like_one_batch():
    """Uneven microbatches (including T=0 and T=1) accumulate dW in fp32."""
    d, E, k, f = 128, 4, 2, 192
    w = workloads.custom("mb", [200, 0, 1, 77], d, E, k, f, bias=("normal", 0.5))
    p = workloads.make_params(w, device=DEV, seed=3)
    layer = MoELayer(p, k, 1, max_tokens=200)
    P = _np_params(p)
    acc = None
    for mb in range(4):
        bt = workloads.make_batch(w, mb=mb, device=DEV, seed=3)
        Y = layer.forward(bt["x"])
        dX = layer.backward(bt["dY"])
        x64 = to_np(bt["x"]).astype(np.float64)
        fw = oracle.layer_forward(x64, P["Wr"], P["b"], P["Wg"], P["Wu"], P["Wd"], k)
        bw = oracle.layer_backward(fw, x64, to_np(bt["dY"]).astype(np.float64), P["Wr"], P["Wg"],
                                   P["Wu"], P["Wd"], k, acc=acc)
        acc = {n: bw[n] for n in ("dWg", "dWu", "dWd", "dWr", "db")}
        assert Y.shape == (w.T[mb], d) and dX.shape == (w.T[mb], d)
        if w.T[mb]:
            assert_close_per("Y", Y, fw["Y"], TOL[torch.bfloat16])
            assert_close_per("dX", dX, bw["dX"], TOL[torch.bfloat16])
    torch.cuda.synchronize()
    for n, ref in acc.items():
        (assert_close if n in ("dWr", "db") else assert_close_per)(n, layer.grads[n], ref, TOL[torch.bfloat16])


def test_empty_microbatch_changes_nothing():
    d, E, k, f = 128, 4, 2, 128
    w = workloads.custom("e", [64], d, E, k, f)
    p = workloads.make_params(w, device=DEV)
    layer = MoELayer(p, k, 2, max_tokens=64)
    bt = workloads.make_batch(w, device=DEV)
    layer.forward(bt["x"])
    layer.backward(bt["dY"])
    torch.cuda.synchronize()
    before = {n: t.clone() for n, t in layer.grads.items()}
    x0 = torch.empty((0, d), dtype=torch.bfloat16, device=DEV)
    Y = layer.forward(x0)
    dX = layer.backward(x0)
    torch.cuda.synchronize()
    assert Y.shape == (0, d) and dX.shape == (0, d)
    for n in before:
        assert torch.equal(before[n], layer.grads[n])


def test_all_tokens_on_one_expert():
    """Extreme skew: one expert takes every token, the others none."""
    T, d, E, k, f = 1000, 128, 8, 1, 128
    w = workloads.custom("skew", T, d, E, k, f, bias="zero")
    p = workloads.make_params(w, device=DEV, seed=11)
    p["b"][:] = -1.0e4
    p["b"][5] = 0.0
    bt = workloads.make_batch(w, device=DEV, seed=11)
    layer = MoELayer(p, k, 1, max_tokens=T)
    Y = layer.forward(bt["x"])
    layer.backward(bt["dY"])
    torch.cuda.synchronize()
    counts = to_np(layer.r["counts"])
    assert counts[5] == T and counts.sum() == T
    P = _np_params(p)
    x64 = to_np(bt["x"]).astype(np.float64)
    fw = oracle.layer_forward(x64, P["Wr"], P["b"], P["Wg"], P["Wu"], P["Wd"], k)
    bw = oracle.layer_backward(fw, x64, to_np(bt["dY"]).astype(np.float64), P["Wr"], P["Wg"], P["Wu"],
                               P["Wd"], k)
    assert_close_per("Y", Y, fw["Y"], 2e-2)
    for n in ("dWg", "dWu", "dWd"):
        assert_close_per(n, layer.grads[n], bw[n], 2e-2)


@pytest.mark.parametrize("accumulate", [True, False])
def test_weight_gradient_of_long_and_short_experts(accumulate):
    """Seven experts with more than 1024 rows and seven with a few dozen, 12
    weight-gradient tiles each: more than a wave (74 CTA pairs) of long tiles
    and of short ones, so their waves alternate before the rest follows in
    list order. Full dW per expert against the oracle, added to a non-zero
    buffer or written over one."""
    T, d, E, k, f = 4608, 512, 14, 2, 512
    w = workloads.custom("long_short", T, d, E, k, f, dtype="bf16", bias="zero")
    p = workloads.make_params(w, device=DEV, seed=0)
    p["b"][:] = 0.0
    p["b"][7:] = -1.0
    bt = workloads.make_batch(w, device=DEV, seed=0)
    layer = MoELayer(p, k, 1, max_tokens=T)
    g0 = {n: torch.randn(layer.grads[n].shape, generator=torch.Generator().manual_seed(3)).to(DEV)
          for n in ("dWg", "dWu", "dWd")}
    for n in g0:
        layer.grads[n].copy_(g0[n])
    layer.forward(bt["x"])
    layer.backward(bt["dY"], accumulate=accumulate)
    torch.cuda.synchronize()
    assert layer.device_errors() == 0
    counts = to_np(layer.r["counts"])
    assert (counts[:7] > 1024).all() and ((counts[7:] > 0) & (counts[7:] < 1024)).all(), counts
    P = _np_params(p)
    x64 = to_np(bt["x"]).astype(np.float64)
    fw = oracle.layer_forward(x64, P["Wr"], P["b"], P["Wg"], P["Wu"], P["Wd"], k)
    acc = {n: to_np(g0[n]).astype(np.float64) for n in g0} if accumulate else None
    bw = oracle.layer_backward(fw, x64, to_np(bt["dY"]).astype(np.float64), P["Wr"], P["Wg"], P["Wu"],
                               P["Wd"], k, acc=acc)
    for n in ("dWg", "dWu", "dWd"):
        assert_close_per(n, layer.grads[n], bw[n], TOL[torch.bfloat16])


def test_long_ragged_weight_gradient_is_exact_and_reproducible():
    """Two experts of 4500 rows each: every weight-gradient tile runs 70 full
    64-row K blocks and a tail of 20 rows, ragged inside a 16-row MMA step.
    Full dW against the oracle, then the same backward again from zero must
    give bitwise the same dW."""
    T, d, E, k, f = 4500, 192, 3, 2, 256
    w = workloads.custom("chunks", T, d, E, k, f, bias="zero")
    p = workloads.make_params(w, device=DEV, seed=5)
    p["b"][:] = 0.0
    p["b"][2] = -1.0e4
    bt = workloads.make_batch(w, device=DEV, seed=5)
    layer = MoELayer(p, k, 1, max_tokens=T)
    layer.forward(bt["x"])
    layer.backward(bt["dY"])
    torch.cuda.synchronize()
    assert layer.device_errors() == 0
    counts = to_np(layer.r["counts"])
    assert counts.tolist() == [T, T, 0]
    P = _np_params(p)
    x64 = to_np(bt["x"]).astype(np.float64)
    fw = oracle.layer_forward(x64, P["Wr"], P["b"], P["Wg"], P["Wu"], P["Wd"], k)
    bw = oracle.layer_backward(fw, x64, to_np(bt["dY"]).astype(np.float64), P["Wr"], P["Wg"], P["Wu"],
                               P["Wd"], k)
    first = {n: layer.grads[n].clone() for n in ("dWg", "dWu", "dWd")}
    for n in first:
        assert_close_per(n, first[n], bw[n], 2e-2)
        assert not first[n][2].any()
    layer.zero_grad()
    layer.backward(bt["dY"])
    torch.cuda.synchronize()
    assert layer.device_errors() == 0
    for n in first:
        assert torch.equal(layer.grads[n], first[n]), n


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_backward_without_accumulate_writes_the_gradients(dtype):
    """accumulate=False: parameter gradients are written, whatever the
    buffers held (an expert no token selected gets zeros), and an empty
    microbatch writes zeros."""
    T, d, E, k, f = (700, 256, 8, 2, 384) if dtype == "bf16" else (200, 64, 4, 2, 128)
    w, p, bt = _layer_case(T, d, E, k, f, dtype, 2, True, seed=9)
    tol = TOL[w.torch_dtype()]
    layer = MoELayer(p, k, 2, max_tokens=T)
    for n, g in layer.grads.items():
        g.fill_(1.0e3)
    layer.forward(bt["x"])
    layer.backward(bt["dY"], accumulate=False)
    torch.cuda.synchronize()
    assert layer.device_errors() == 0
    P = _np_params(p)
    x64 = to_np(bt["x"]).astype(np.float64)
    fw = oracle.layer_forward(x64, P["Wr"], P["b"], P["Wg"], P["Wu"], P["Wd"], k, 2)
    bw = oracle.layer_backward(fw, x64, to_np(bt["dY"]).astype(np.float64), P["Wr"], P["Wg"], P["Wu"],
                               P["Wd"], k)
    for n in ("dWg", "dWu", "dWd"):
        assert_close_per(n, layer.grads[n], bw[n], tol)
    for n in ("dWr", "db"):
        assert_close(n, layer.grads[n], bw[n], tol)
    for n in ("dWg", "dWu", "dWd", "dWr"):
        assert not layer.grads[n][E - 1].any(), f"{n} of the starved expert must be written as zero"
    # an empty microbatch without accumulation: the gradient of nothing is zero
    x0 = torch.empty((0, d), dtype=w.torch_dtype(), device=DEV)
    layer.forward(x0)
    layer.backward(x0, accumulate=False)
    torch.cuda.synchronize()
    for n, g in layer.grads.items():
        assert not g.any(), n


# ----------------------------------------------------- failure detection

def test_bounded_wait_times_out_and_leaves_the_context_usable():
    """A wait on a barrier nothing arrives at gives up, raises the time-out
    bit in the error word, and the next calls still work."""
    ws = N._ws(256, DEV)
    rc = N.lib().moe_selftest_wait_timeout(N._ptr(ws), 2_000_000, N._stream(None))
    assert rc == N.MOE_OK
    assert N.moe_get_error(ws) == N.MOE_DEVERR_TIMEOUT
    assert N.moe_get_error(ws) == 0
    z = workloads.make_logits(100, 8, device=DEV, seed=1)
    out = N.moe_route(z, 2)
    idx, _, _ = oracle.route(z.double().cpu().numpy(), 2)
    assert np.array_equal(to_np(out["topk_idx"]), idx)


# ------------------------------------------------------- argument errors

def test_rejected_calls_report_errors_and_launch_nothing():
    z = torch.zeros((4, 8), device=DEV)
    with pytest.raises(N.MoeError) as ei:
        N.moe_route(z, 9)  # k > E
    assert ei.value.code == N.MOE_ERR_INVALID_ARG
    with pytest.raises(N.MoeError) as ei:
        N.moe_route(z, 2, ep_groups=3)  # E % groups != 0
    assert ei.value.code == N.MOE_ERR_UNSUPPORTED
    with pytest.raises(N.MoeError) as ei:
        N.moe_route(z, 2, ws=torch.zeros(16, dtype=torch.uint8, device=DEV))
    assert ei.value.code == N.MOE_ERR_WORKSPACE
    xp = torch.zeros((8, 100), dtype=torch.bfloat16, device=DEV)  # d not a multiple of 64
    Wg = torch.zeros((2, 128, 100), dtype=torch.bfloat16, device=DEV)
    Wd = torch.zeros((2, 100, 128), dtype=torch.bfloat16, device=DEV)
    off = torch.tensor([0, 4, 8], dtype=torch.int64, device=DEV)
    with pytest.raises(N.MoeError) as ei:
        N.moe_grouped_ffn_fwd(xp, Wg, Wg, Wd, off)
    assert ei.value.code == N.MOE_ERR_UNSUPPORTED
