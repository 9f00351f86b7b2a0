"""One MoE layer driven through the C ABI: the call sequence of a training step.

Forward:  moe_router_logits -> moe_route -> moe_permute -> moe_grouped_ffn_fwd
          -> moe_unpermute_combine
Backward: moe_unpermute_combine_bwd -> moe_route_bwd -> moe_grouped_ffn_dgrad
          -> moe_grouped_ffn_wgrad -> moe_permute_bwd (with the router's input
          gradient) -> moe_router_bwd_gather (dispatch rows read from x)
With checkpoint=True the forward does not store h1 and h2 and the backward
first rebuilds them with moe_grouped_ffn_recompute (activation checkpointing:
2 T k f activation elements less to keep between forward and backward, for
one more gate/up GEMM).
With fused_dispatch=True there is no permuted copy xp: the gate/up GEMM and
the weight gradient's dWg / dWu operand read dispatch row r in place as
x[pair_of_row[r] / k] (moe_grouped_ffn_fwd_gather,
moe_grouped_ffn_wgrad_gather), with results bitwise those of the permuted
path. It saves the T k d copy but is slower on this shape: the GEMMs re-read
each row many times, and row-sized gathers move those re-reads at a fraction
of the tiled loads' rate. Either way x must stay unchanged until the backward.
With a balance-loss coefficient (aux_coef > 0) the forward also calls
moe_aux_loss after routing, and the backward ends with moe_aux_loss_bwd ->
moe_router_bwd_dense (the loss's dense logit gradient into dX, dWr, db).

The object owns device buffers sized for `max_tokens`, so a step allocates
nothing; microbatches of any size up to that (0 included) reuse them. No call
synchronises with the host, so forward + backward on fixed input buffers can be
captured once into a CUDA graph and replayed for every new batch of that size
(the routing, expert offsets and GEMM tile lists all live on the device). Weight
gradients accumulate in fp32 across microbatches until zero_grad(); a
backward with accumulate=False writes them instead (the first microbatch of a
step: the old values are neither read nor needed).
"""
from __future__ import annotations

from typing import Dict, Optional

import torch

from . import native as N


def _no_mark(name: str) -> None:
    pass


# Kernels each C call launches (bf16 and fp32 paths alike).
LAUNCHES_PER_CALL = {
    "router_logits": 1, "route": 3, "permute": 1, "grouped_ffn_fwd": 2, "unpermute_combine": 1,
    "unpermute_combine_bwd": 1, "route_bwd": 1, "grouped_ffn_dgrad": 2, "grouped_ffn_wgrad": 1,
    "permute_bwd": 1, "router_bwd": 2, "aux_loss": 2, "aux_loss_bwd": 1, "router_bwd_dense": 3,
    "grouped_ffn_recompute": 1, "grouped_ffn_fwd_gather": 2, "grouped_ffn_wgrad_gather": 1,
    "router_bwd_gather": 2, "grouped_ffn_recompute_gather": 1,
}


class MoELayer:
    def __init__(self, params: Dict[str, torch.Tensor], k: int, ep_groups: int = 1,
                 max_tokens: int = 0, aux_coef: float = 0.0, checkpoint: bool = False,
                 fused_dispatch: bool = False):
        self.Wr, self.b = params["Wr"], params["b"]
        self.Wg, self.Wu, self.Wd = params["Wg"], params["Wu"], params["Wd"]
        self.E, self.f, self.d = self.Wg.shape
        self.k, self.G = k, ep_groups
        self.dtype = self.Wg.dtype
        self.dt = N.MOE_BF16 if self.dtype == torch.bfloat16 else N.MOE_F32
        dev = self.Wg.device
        self.device = dev
        f32 = torch.float32
        self.grads = {
            "dWr": torch.zeros((self.E, self.d), dtype=f32, device=dev),
            "db": torch.zeros(self.E, dtype=f32, device=dev),
            "dWg": torch.zeros((self.E, self.f, self.d), dtype=f32, device=dev),
            "dWu": torch.zeros((self.E, self.f, self.d), dtype=f32, device=dev),
            "dWd": torch.zeros((self.E, self.d, self.f), dtype=f32, device=dev),
        }
        # Switch-style balance loss coefficient (0: no auxiliary loss); after a
        # forward, self.aux holds its loss [1], importance [E], entropy [1]
        self.aux_coef = float(aux_coef)
        self.checkpoint = bool(checkpoint)
        self.fused = bool(fused_dispatch)
        self.aux = {
            "loss": torch.zeros(1, dtype=f32, device=dev),
            "importance": torch.zeros(self.E, dtype=f32, device=dev),
            "entropy": torch.zeros(1, dtype=f32, device=dev),
        }
        self.max_tokens = 0
        self.T = 0
        self.reserve(max(1, max_tokens))

    def reserve(self, T: int) -> None:
        """Make the buffers hold microbatches of up to T tokens."""
        if T <= self.max_tokens:
            return
        dev, dt, E, k, d, f = self.device, self.dtype, self.E, self.k, self.d, self.f
        P = T * k
        f32 = torch.float32
        self.buf = {
            "logits": torch.empty((T, E), dtype=f32, device=dev),
            "xp": torch.empty((0 if self.fused else P, d), dtype=dt, device=dev),
            "h1": torch.empty((P, f), dtype=dt, device=dev),
            "h2": torch.empty((P, f), dtype=dt, device=dev),
            "a": torch.empty((P, f), dtype=dt, device=dev),
            "yp": torch.empty((P, d), dtype=dt, device=dev),
            "Y": torch.empty((T, d), dtype=dt, device=dev),
            "dyp": torch.empty((P, d), dtype=dt, device=dev),
            "dg": torch.empty((T, k), dtype=f32, device=dev),
            "dlogits": torch.empty((T, E), dtype=f32, device=dev),
            "dxp": torch.empty((P, d), dtype=dt, device=dev),
            "dh1": torch.empty((P, f), dtype=dt, device=dev),
            "dh2": torch.empty((P, f), dtype=dt, device=dev),
            "dX": torch.empty((T, d), dtype=dt, device=dev),
        }
        self.route = N.route_outputs(T, E, k, self.G, dev)
        self.ws = {
            "route": N._ws(N.moe_route_workspace_bytes(T, E), dev),
            "ffn_fwd": N._ws(N.moe_grouped_ffn_fwd_workspace_bytes(P, E, d, f, self.dt), dev),
            # dgrad, wgrad and recompute use its error word
            "ffn_bwd": N._ws(max(N.moe_grouped_ffn_fwd_workspace_bytes(P, E, d, f, self.dt),
                                 N.moe_grouped_ffn_wgrad_workspace_bytes(E, self.dt)), dev),
            "router_bwd": N._ws(N.moe_router_bwd_workspace_bytes(P, d, E), dev),
        }
        if self.aux_coef:
            self.buf["dz_aux"] = torch.empty((T, E), dtype=f32, device=dev)
            self.ws["aux"] = N._ws(N.moe_aux_loss_workspace_bytes(T, E), dev)
            self.ws["dense"] = N._ws(N.moe_router_bwd_dense_workspace_bytes(T, d, E), dev)
        self.max_tokens = T

    def zero_grad(self) -> None:
        for g in self.grads.values():
            g.zero_()

    def _views(self, T: int):
        P = T * self.k
        b = self.buf
        r = self.route
        v = {n: b[n][:T] for n in ("logits", "Y", "dg", "dlogits", "dX", "dz_aux") if n in b}
        v.update({n: b[n][:P] for n in ("xp", "h1", "h2", "a", "yp", "dyp", "dxp", "dh1", "dh2")})
        ro = dict(r)
        for n in ("topk_idx", "topk_w"):
            ro[n] = r[n][:T]
        for n in ("row_of_pair", "pair_of_row"):
            ro[n] = r[n][:P]
        return v, ro

    def forward(self, x: torch.Tensor, stream=None, mark=None, out=None) -> torch.Tensor:
        """Y = layer(x), written to `out` if given (else to a layer buffer).
        `mark(name)`, if given, is called after each C call (the benchmark
        records CUDA events there)."""
        mark = mark or _no_mark
        T = x.shape[0]
        self.reserve(T)
        self.T = T
        self.x = x
        v, r = self._views(T)
        self.v, self.r = v, r
        N.moe_router_logits(x, self.Wr, self.b, v["logits"], stream)
        mark("router_logits")
        N.moe_route(v["logits"], self.k, self.G, r, self.ws["route"], stream)
        mark("route")
        if self.aux_coef:
            N.moe_aux_loss(v["logits"], r["counts"], self.k, self.aux_coef, self.aux, self.ws["aux"],
                           stream)
            mark("aux_loss")
        saved = {n: v[n] for n in ("h1", "h2", "a", "yp")}
        if self.checkpoint:
            saved["h1"] = saved["h2"] = None  # rebuilt in the backward
        if self.fused:
            N.moe_grouped_ffn_fwd_gather(x, r["pair_of_row"], self.k, self.Wg, self.Wu, self.Wd, r["offsets"],
                                         saved, self.ws["ffn_fwd"], stream)
            mark("grouped_ffn_fwd_gather")
        else:
            N.moe_permute(x, r["row_of_pair"], self.k, v["xp"], stream)
            mark("permute")
            N.moe_grouped_ffn_fwd(v["xp"], self.Wg, self.Wu, self.Wd, r["offsets"], saved, self.ws["ffn_fwd"],
                                  stream)
            mark("grouped_ffn_fwd")
        Y = v["Y"] if out is None else out
        N.moe_unpermute_combine(v["yp"], r["topk_w"], r["row_of_pair"], Y, stream)
        mark("unpermute_combine")
        return Y

    def backward(self, dY: torch.Tensor, stream=None, mark=None, out=None,
                 accumulate: bool = True, aux_dloss: float = 1.0) -> torch.Tensor:
        """dX for upstream gradient dY of the last forward (written to `out`
        if given); dW += the batch's gradient (fp32), or dW = it if not
        `accumulate`. With a balance loss, its gradient (scaled by
        `aux_dloss`) is included."""
        mark = mark or _no_mark
        T = self.T
        v, r = self.v, self.r
        g = self.grads
        N.moe_unpermute_combine_bwd(dY, v["yp"], r["topk_w"], r["row_of_pair"], v["dyp"], v["dg"], stream)
        mark("unpermute_combine_bwd")
        N.moe_route_bwd(v["dg"], r["topk_w"], r["topk_idx"], self.E, v["dlogits"], stream)
        mark("route_bwd")
        if self.checkpoint and self.fused:
            N.moe_grouped_ffn_recompute_gather(self.x, r["pair_of_row"], self.k, self.Wg, self.Wu, r["offsets"],
                                               v["h1"], v["h2"], self.ws["ffn_bwd"], stream)
            mark("grouped_ffn_recompute_gather")
        elif self.checkpoint:
            N.moe_grouped_ffn_recompute(v["xp"], self.Wg, self.Wu, r["offsets"], v["h1"], v["h2"],
                                        self.ws["ffn_bwd"], stream)
            mark("grouped_ffn_recompute")
        N.moe_grouped_ffn_dgrad(self.Wg, self.Wu, self.Wd, v["h1"], v["h2"], v["dyp"], r["offsets"],
                                v["dh1"], v["dh2"], v["dxp"], self.ws["ffn_bwd"], stream)
        mark("grouped_ffn_dgrad")
        if self.fused:
            N.moe_grouped_ffn_wgrad_gather(self.x, r["pair_of_row"], self.k, v["a"], v["dyp"], v["dh1"], v["dh2"],
                                           r["offsets"], g["dWg"], g["dWu"], g["dWd"], self.ws["ffn_bwd"],
                                           stream, accumulate=accumulate)
            mark("grouped_ffn_wgrad_gather")
        else:
            N.moe_grouped_ffn_wgrad(v["xp"], v["a"], v["dyp"], v["dh1"], v["dh2"], r["offsets"], g["dWg"],
                                    g["dWu"], g["dWd"], self.ws["ffn_bwd"], stream, accumulate=accumulate)
            mark("grouped_ffn_wgrad")
        dX = v["dX"] if out is None else out
        N.moe_permute_bwd(v["dxp"], r["row_of_pair"], v["dlogits"], self.Wr, r["topk_idx"], T, self.k,
                          dX, stream)
        mark("permute_bwd")
        # the router's weight gradient reads the dispatch rows from x (T d
        # elements, k times fewer than xp) in both layouts: bitwise the same sums
        N.moe_router_bwd_gather(self.x, v["dlogits"], r["pair_of_row"], r["offsets"], self.k, g["dWr"],
                                g["db"], self.ws["router_bwd"], stream, accumulate=accumulate)
        mark("router_bwd_gather")
        if self.aux_coef:
            N.moe_aux_loss_bwd(v["logits"], r["counts"], self.k, self.aux_coef, aux_dloss, v["dz_aux"],
                               stream)
            mark("aux_loss_bwd")
            N.moe_router_bwd_dense(self.x, self.Wr, v["dz_aux"], dX, g["dWr"], g["db"], accumulate=True,
                                   ws=self.ws["dense"], stream=stream)
            mark("router_bwd_dense")
        return dX

    def device_errors(self) -> int:
        """Synchronises and returns (and clears) the device error words."""
        err = 0
        for n in ("route", "ffn_fwd", "ffn_bwd"):
            err |= N.moe_get_error(self.ws[n])
        return err
