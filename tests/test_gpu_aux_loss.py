"""GPU parity of the auxiliary load-balancing loss, its logit gradient, and the
dense router backward, through the C ABI, against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from grouped_expert_ffn_top_b200 import native as N
from grouped_expert_ffn_top_b200 import workloads
from grouped_expert_ffn_top_b200.layer import MoELayer
from parity import TOL, assert_close, assert_close_per, oracle_routing, rel_err, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL_F32 = 1e-5  # fp32 sums of at most a few thousand terms against double


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    N.lib()


@pytest.mark.parametrize("T,E,k", [(1000, 16, 2), (257, 64, 8), (300, 1024, 8), (5, 3, 1), (70, 40, 4)])
def test_aux_loss_and_gradient_match_oracle(T, E, k):
    z = workloads.make_logits(T, E, seed=T + E, tie_fraction=0.0).to(DEV)
    z[:, E - 1] -= 30.0  # a starved expert
    r = N.moe_route(z, k, 1)
    out = N.moe_aux_loss(z, r["counts"], k, 0.01)
    dz = N.moe_aux_loss_bwd(z, r["counts"], k, 0.01, dloss=1.3)
    torch.cuda.synchronize()
    counts = to_np(r["counts"])
    ref = oracle.aux_loss(to_np(z).astype(np.float64), counts, k, 0.01)
    assert_close("importance", out["importance"], ref["importance"], TOL_F32)
    assert abs(float(out["loss"]) - ref["loss"]) <= TOL_F32 * abs(ref["loss"])
    assert abs(float(out["entropy"]) - ref["entropy"]) <= TOL_F32 * abs(ref["entropy"])
    dz_ref = oracle.aux_loss_bwd(to_np(z).astype(np.float64), counts, k, 0.01, 1.3)
    assert_close("dlogits_aux", dz, dz_ref, TOL_F32)


def test_aux_loss_of_an_empty_batch_is_zero():
    z = torch.empty((0, 8), dtype=torch.float32, device=DEV)
    counts = torch.zeros(8, dtype=torch.int32, device=DEV)
    o = {n: torch.full(s, 5.0, device=DEV) for n, s in (("importance", (8,)), ("loss", (1,)), ("entropy", (1,)))}
    N.moe_aux_loss(z, counts, 2, 0.1, out=o)
    torch.cuda.synchronize()
    for n, t in o.items():
        assert not t.any(), n


def _offset_copy(t, offset):
    """A copy of t whose data starts `offset` elements into a fresh buffer
    (offset 2: 4 or 8 bytes past an aligned start, so the kernels take their
    element-by-element path)."""
    if not offset:
        return t.contiguous()
    buf = torch.empty(t.numel() + offset, dtype=t.dtype, device=t.device)
    v = buf[offset:].view(t.shape)
    v.copy_(t)
    return v


# E <= 16 (experts staged 16 at a time) and above (32 at a time, a partial
# last chunk at E = 70); d with a partial 128-column tile; T off the 64-token
# steps and 256-token chunks; aligned and misaligned operands
@pytest.mark.parametrize("dtype,T,d,E,offset", [("bf16", 700, 192, 70, 0), ("f32", 333, 200, 9, 0),
                                                ("bf16", 64, 64, 64, 0), ("bf16", 1000, 256, 16, 0),
                                                ("bf16", 300, 136, 40, 2), ("f32", 130, 68, 5, 2)])
def test_dense_router_backward_matches_oracle(dtype, T, d, E, offset):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    g = torch.Generator(device="cpu").manual_seed(T * 31 + E)
    x = _offset_copy(torch.randn((T, d), generator=g).to(tdt).to(DEV), offset)
    Wr = _offset_copy((torch.randn((E, d), generator=g) * 0.05).to(tdt).to(DEV), offset)
    dz = (torch.randn((T, E), generator=g) * 0.1).to(DEV)
    dX = _offset_copy(torch.randn((T, d), generator=g).to(tdt).to(DEV), offset)
    dWr = torch.randn((E, d), generator=g).to(DEV)
    db = torch.randn(E, generator=g).to(DEV)
    dX0, dWr0, db0 = (to_np(t).astype(np.float64) for t in (dX, dWr, db))
    N.moe_router_bwd_dense(x, Wr, dz, dX, dWr, db, accumulate=True)
    torch.cuda.synchronize()
    rX, rWr, rb = oracle.router_bwd(to_np(x).astype(np.float64), to_np(Wr).astype(np.float64),
                                    to_np(dz).astype(np.float64), dX0, dWr0, db0)
    tol = TOL[tdt]
    assert_close("dX", dX, rX, tol)
    assert_close("dWr", dWr, rWr, TOL_F32)
    assert_close("db", db, rb, TOL_F32)
    # written, not added
    N.moe_router_bwd_dense(x, Wr, dz, None, dWr, db, accumulate=False)
    torch.cuda.synchronize()
    _, wWr, wb = oracle.router_bwd(to_np(x).astype(np.float64), to_np(Wr).astype(np.float64),
                                   to_np(dz).astype(np.float64), dX0)
    assert_close("dWr written", dWr, wWr, TOL_F32)
    assert_close("db written", db, wb, TOL_F32)


def test_layer_with_balance_loss_matches_oracle():
    T, d, E, k, f, G, alpha = 700, 256, 8, 2, 384, 2, 0.01
    w = workloads.custom("aux", T, d, E, k, f, bias=("normal", 0.5), ep_groups=G)
    p = workloads.make_params(w, device=DEV, seed=4)
    p["b"][E - 1] = -1.0e4
    bt = workloads.make_batch(w, device=DEV, seed=4)
    layer = MoELayer(p, k, G, max_tokens=T, aux_coef=alpha)
    layer.forward(bt["x"])
    dX = layer.backward(bt["dY"], accumulate=False, aux_dloss=2.0)
    torch.cuda.synchronize()
    assert layer.device_errors() == 0
    P = {n: to_np(v).astype(np.float64) for n, v in p.items()}
    x64 = to_np(bt["x"]).astype(np.float64)
    fw = oracle.layer_forward(x64, P["Wr"], P["b"], P["Wg"], P["Wu"], P["Wd"], k, G)
    ref_aux = oracle.aux_loss(fw["z"], fw["counts"], k, alpha)
    assert abs(float(layer.aux["loss"]) - ref_aux["loss"]) <= TOL_F32 * ref_aux["loss"]
    assert_close("importance", layer.aux["importance"], ref_aux["importance"], TOL_F32)
    bw = oracle.layer_backward(fw, x64, to_np(bt["dY"]).astype(np.float64), P["Wr"], P["Wg"], P["Wu"],
                               P["Wd"], k, aux=(alpha, 2.0))
    tol = TOL[torch.bfloat16]
    assert_close("dX", dX, bw["dX"], tol)
    for n in ("dWr", "db", "dWg", "dWu", "dWd"):
        assert_close(n, layer.grads[n], bw[n], tol)
    # the balance loss's gradient is dense over the experts: it changes dWr
    plain = MoELayer(p, k, G, max_tokens=T)
    plain.forward(bt["x"])
    plain.backward(bt["dY"], accumulate=False)
    torch.cuda.synchronize()
    assert not torch.equal(plain.grads["dWr"], layer.grads["dWr"])


# ------------------------------------------------ activation checkpointing

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_checkpointed_backward_is_bitwise_the_stored_one(dtype):
    """checkpoint=True: the forward leaves h1 and h2 unwritten, the backward
    rebuilds them with the same kernel, and every output and gradient equals
    the stored-activation path bit for bit."""
    T, d, E, k, f = (700, 256, 8, 2, 384) if dtype == "bf16" else (200, 64, 4, 2, 128)
    w = workloads.custom("ckpt", T, d, E, k, f, dtype=dtype, bias=("normal", 0.5), ep_groups=2)
    p = workloads.make_params(w, device=DEV, seed=6)
    bt = workloads.make_batch(w, device=DEV, seed=6)
    ref = MoELayer(p, k, 2, max_tokens=T)
    ck = MoELayer(p, k, 2, max_tokens=T, checkpoint=True)
    ck.buf["h1"].fill_(float("nan"))
    ck.buf["h2"].fill_(float("nan"))
    Y0 = ref.forward(bt["x"]).clone()
    Y1 = ck.forward(bt["x"]).clone()
    torch.cuda.synchronize()
    assert torch.isnan(ck.buf["h1"]).all() and torch.isnan(ck.buf["h2"]).all()
    assert torch.equal(Y0, Y1)
    dX0 = ref.backward(bt["dY"], accumulate=False).clone()
    dX1 = ck.backward(bt["dY"], accumulate=False).clone()
    torch.cuda.synchronize()
    assert ck.device_errors() == 0
    assert torch.equal(dX0, dX1)
    for n in ("h1", "h2", "dh1", "dh2"):
        assert torch.equal(ref.v[n], ck.v[n]), n
    for n in ref.grads:
        assert torch.equal(ref.grads[n], ck.grads[n]), n
    # and the checkpointed layer itself against the oracle
    tol = TOL[w.torch_dtype()]
    P = {n: to_np(v).astype(np.float64) for n, v in p.items()}
    x64 = to_np(bt["x"]).astype(np.float64)
    fw = oracle.layer_forward(x64, P["Wr"], P["b"], P["Wg"], P["Wu"], P["Wd"], k, 2)
    bw = oracle.layer_backward(fw, x64, to_np(bt["dY"]).astype(np.float64), P["Wr"], P["Wg"], P["Wu"],
                               P["Wd"], k)
    assert_close_per("Y", Y1, fw["Y"], tol)
    assert_close_per("dX", dX1, bw["dX"], tol)
    for n in ("h1", "h2"):
        assert_close_per(n, ck.v[n], fw[n], tol)
    for n in ("dWg", "dWu", "dWd"):
        assert_close_per(n, ck.grads[n], bw[n], tol)
    for n in ("dWr", "db"):
        assert_close(n, ck.grads[n], bw[n], tol)
