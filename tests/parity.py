"""Helpers shared by the parity tests, the smoke check and the benchmark's
CPU leg: the error metric, and oracle evaluations of a workload (whole, or on
sampled tokens and columns for sizes the oracle cannot run in full).

Only the seeded generators and `oracle/` are used to produce expected values;
GPU results are only ever compared against them.
"""
from __future__ import annotations

from typing import Dict, List, Optional

import numpy as np
import torch

import oracle

# Float tolerances (normwise max relative error, max|gpu-ref| / max|ref|):
# bf16 storage rounds h1, h2, a, yp, dyp, dh1, dh2, dxp once each (2^-9
# relative), which 2e-2 covers with margin; the fp32 path sums in fp32
# (about sqrt(K) * 2^-24 relative), far inside 1e-4.
TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


def rel_err(gpu, ref) -> float:
    g = to_np(gpu).astype(np.float64) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    if r.size == 0:
        return 0.0
    scale = np.abs(r).max()
    if scale == 0.0:
        return float(np.abs(g - r).max())
    return float(np.abs(g - r).max() / scale)


def assert_close(name: str, gpu, ref, tol: float):
    e = rel_err(gpu, ref)
    assert e <= tol, f"{name}: normwise relative error {e:.3e} > {tol:.1e}"
    return e


def rel_err_per(gpu, ref) -> float:
    """Worst over the leading index (a token, a dispatch row, an expert) of
    max|gpu - ref| / max|ref| taken within that slice, so a wrong result in a
    small slice cannot hide under the largest slice's magnitude. A slice whose
    reference is all zero is measured against the whole tensor's scale."""
    g = to_np(gpu).astype(np.float64) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    if r.size == 0:
        return 0.0
    n = r.shape[0]
    g = g.reshape(n, -1)
    r = r.reshape(n, -1)
    glob = np.abs(r).max()
    scale = np.abs(r).max(axis=1)
    scale = np.where(scale > 0.0, scale, glob if glob > 0.0 else 1.0)
    return float((np.abs(g - r).max(axis=1) / scale).max())


def assert_close_per(name: str, gpu, ref, tol: float):
    """assert_close with the scale taken per leading index (rel_err_per)."""
    e = rel_err_per(gpu, ref)
    assert e <= tol, f"{name}: max relative error per slice {e:.3e} > {tol:.1e}"
    return e


def oracle_routing(x: torch.Tensor, Wr: torch.Tensor, b: torch.Tensor, k: int, G: int):
    """Oracle logits (fp32 fixed order), top-k and layout for all tokens."""
    z = oracle.router_logits_f32(to_np(x).astype(np.float32), to_np(Wr).astype(np.float32),
                                 to_np(b).astype(np.float32))
    idx, w, flags = oracle.route(z.astype(np.float64), k)
    lay = oracle.dispatch_layout(idx, Wr.shape[0], G)
    return dict(z=z, idx=idx, w=w, flags=flags, **lay)


def check_routing_bitexact(layer_route: Dict[str, torch.Tensor], logits_gpu: torch.Tensor, ref: dict,
                           check_logits: bool = True):
    if check_logits:
        assert np.array_equal(to_np(logits_gpu), ref["z"]), "router logits differ"
    assert np.array_equal(to_np(layer_route["topk_idx"]), ref["idx"]), "top-k indices differ"
    for n in ("counts", "offsets", "group_counts", "group_offsets", "row_of_pair", "pair_of_row"):
        assert np.array_equal(to_np(layer_route[n]), ref[n]), f"{n} differs"
    assert np.abs(to_np(layer_route["topk_w"]) - ref["w"]).max() <= 1e-6


def sampled_forward_backward(x, dY, params, ref_route: dict, tokens: np.ndarray, k: int,
                             backward: bool = True):
    """Oracle Y (and dX, dg, dlogits) for the given tokens, one expert at a time.

    Each pair's expert output y_{t,j} = FFN_{S_{t,j}}(x_t) comes from the
    per-token oracle (one expert's weights at a time); the sample's pairs are
    then laid out as dispatch rows in (token, slot) order, and Y and dg come
    from oracle.combine / oracle.combine_bwd over them. The expert part of dX
    of each pair is the per-token oracle's backward of that pair alone, the
    router part oracle.route_bwd / oracle.router_bwd over the token's k slots."""
    E = params["Wg"].shape[0]
    d = x.shape[1]
    xs = to_np(x[torch.as_tensor(tokens, dtype=torch.long, device=x.device)]).astype(np.float64)
    dYs = to_np(dY[torch.as_tensor(tokens, dtype=torch.long, device=dY.device)]).astype(np.float64) \
        if backward else None
    idx = ref_route["idx"][tokens]
    w = ref_route["w"][tokens]
    n = len(tokens)
    ys_all = np.zeros((n, k, d))
    dX = np.zeros((n, d))
    for e in np.unique(idx):
        sel_t, sel_j = np.nonzero(idx == e)
        Wg = to_np(params["Wg"][e:e + 1]).astype(np.float64)
        Wu = to_np(params["Wu"][e:e + 1]).astype(np.float64)
        Wd = to_np(params["Wd"][e:e + 1]).astype(np.float64)
        one = np.zeros((len(sel_t), 1), np.int32)
        g = w[sel_t, sel_j][:, None]
        _, ys = oracle.tokens_fwd(xs[sel_t], one, np.ones_like(g), Wg, Wu, Wd)
        ys_all[sel_t, sel_j] = ys[:, 0, :]
        if backward:
            _, dXe = oracle.tokens_bwd(xs[sel_t], dYs[sel_t], one, g, ys, np.zeros((1, d)), Wg, Wu, Wd)
            np.add.at(dX, sel_t, dXe)
    # the sample's pairs as dispatch rows in (token, slot) order
    yp = ys_all.reshape(n * k, d)
    rop = np.arange(n * k, dtype=np.int32)
    out = {"Y": oracle.combine(yp, w, rop)}
    if backward:
        _, dg = oracle.combine_bwd(dYs, yp, w, rop)
        dz = oracle.route_bwd(dg, w, idx, E)
        Wr = to_np(params["Wr"]).astype(np.float64)
        dX, _, _ = oracle.router_bwd(xs, Wr, dz, dX)
        out.update(dX=dX, dz=dz, dg=dg)
    return out


def sampled_wgrad(batches: List[dict], params, routes: List[dict], k: int, e: int, cols: np.ndarray):
    """Oracle columns `cols` of dWg[e], dWu[e] (rows) and dWd[e] (columns),
    summed over every microbatch."""
    Wg = to_np(params["Wg"][e]).astype(np.float64)
    Wu = to_np(params["Wu"][e]).astype(np.float64)
    Wd = to_np(params["Wd"][e]).astype(np.float64)
    d = Wg.shape[1]
    acc = [np.zeros((len(cols), d)) for _ in range(3)]
    for bt, rt in zip(batches, routes):
        lo, hi = rt["offsets"][e], rt["offsets"][e + 1]
        if hi == lo:
            continue
        pairs = rt["pair_of_row"][lo:hi]
        toks = pairs // k
        gs = rt["w"].reshape(-1)[pairs]
        tt = torch.as_tensor(toks, dtype=torch.long, device=bt["x"].device)
        xs = to_np(bt["x"][tt]).astype(np.float64)
        dYs = to_np(bt["dY"][tt]).astype(np.float64)
        og, ou, od = oracle.wgrad_columns(xs, dYs, gs, Wg, Wu, Wd, cols.astype(np.int32))
        acc[0] += og
        acc[1] += ou
        acc[2] += od
    return acc
