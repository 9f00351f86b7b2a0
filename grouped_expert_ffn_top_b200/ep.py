"""Expert parallelism: the MoE layer with its experts sharded over the ranks of
a process group (expert communication groups, ART issue #917 "Support
combined expert and data parallelism in TrainerRank", Desired behavior; EP
token dispatch, leap-finetune PR #26 "Add MoE expert parallel training
runtime", Summary).

Rank g of a group of G owns experts [g E/G, (g+1) E/G). Every rank routes its
own tokens against the replicated router, and the dispatch layout's per-group
counts and offsets (moe_route with ep_groups = G) are the send splits:

  forward   route -> permute -> all-to-all of the per-expert counts -> ragged
            all-to-all of the rows -> regroup by local expert -> grouped FFN
            of the local experts -> inverse regroup -> ragged all-to-all back
            -> combine
  backward  combine backward -> route backward -> rows' gradients out the same
            way -> local dgrad and wgrad -> back -> permute backward (with the
            router's input gradient) -> router backward

Ranks with no tokens, and local experts that receive no rows, still join
every exchange (zero-length splits). The received rows arrive grouped by
source rank; the regroup puts them in (local expert, source rank, order)
order with the library's permute kernel used as a row scatter (k = 1), and
the inverse is its permute backward used as a row gather.

The exchanges are torch.distributed all-to-alls (NCCL on GPUs): the split
sizes have to be known on the host, so the forward makes one small
device-to-host copy of the counts (the received counts and this rank's send
splits together); the backward reuses those splits. The regroup map and the
local experts' offsets are built on the device from the received counts
(moe_ep_regroup). The local steps run in `ops`, the library's kernels through
the C ABI (`KernelOps`).
"""
from __future__ import annotations

from typing import Dict

import numpy as np
import torch
import torch.distributed as dist

from . import native as N


def _no_mark(name: str) -> None:
    pass


class KernelOps:
    """The layer's steps through the C ABI (one GPU's share of the work)."""

    def router_logits(self, x, Wr, b):
        return N.moe_router_logits(x, Wr, b)

    def route(self, z, k, G):
        T, E = z.shape
        r = N.route_outputs(T, E, k, G, z.device)  # counts and offsets start at zero
        return N.moe_route(z, k, G, out=r)

    def permute(self, x, row_of_pair, k):
        return N.moe_permute(x, row_of_pair, k)

    def regroup(self, recv_dev, recv_host):
        """Row map and local offsets of the received rows, built on the
        device from the counts there (moe_ep_regroup)."""
        return N.moe_ep_regroup(recv_dev, int(recv_host.sum()))

    def gather_rows(self, src, rows_of):
        """out[i] = src[rows_of[i]] (the permute backward with k = 1)."""
        return N.moe_permute_bwd(src, rows_of, None, None, None, rows_of.numel(), 1)

    def ffn_fwd(self, xp, Wg, Wu, Wd, offsets):
        return N.moe_grouped_ffn_fwd(xp, Wg, Wu, Wd, offsets)

    def combine(self, yp, topk_w, row_of_pair):
        return N.moe_unpermute_combine(yp, topk_w, row_of_pair)

    def combine_bwd(self, dY, yp, topk_w, row_of_pair):
        return N.moe_unpermute_combine_bwd(dY, yp, topk_w, row_of_pair)

    def route_bwd(self, dg, topk_w, topk_idx, E):
        return N.moe_route_bwd(dg, topk_w, topk_idx, E)

    def ffn_bwd(self, xp, Wg, Wu, Wd, h1, h2, a, dyp, offsets, dWg, dWu, dWd, accumulate):
        return N.moe_grouped_ffn_bwd(xp, Wg, Wu, Wd, h1, h2, a, dyp, offsets, dWg, dWu, dWd,
                                     accumulate=accumulate)

    def permute_bwd(self, dxp, row_of_pair, dlogits, Wr, topk_idx, T, k):
        return N.moe_permute_bwd(dxp, row_of_pair, dlogits, Wr, topk_idx, T, k)

    def router_bwd(self, xp, dlogits, pair_of_row, offsets, k, dWr, db, accumulate):
        N.moe_router_bwd(xp, dlogits, pair_of_row, offsets, k, dWr, db, accumulate=accumulate)


def regroup_map(recv_counts: np.ndarray) -> np.ndarray:
    """The host form of moe_ep_regroup's row map (for ops that keep their
    tensors on the host). Destination of every received row. recv_counts[s, e] rows for local
    expert e arrive from rank s, sources in rank order and, within a source,
    experts in order; row q of block (s, e) goes to
        sum_{e' < e} sum_s' recv_counts[s', e'] + sum_{s' < s} recv_counts[s', e] + q,
    i.e. the rows end up sorted by (local expert, source rank, arrival)."""
    G, El = recv_counts.shape
    per_expert = recv_counts.sum(axis=0)
    expert_base = np.concatenate([[0], np.cumsum(per_expert)[:-1]]) if El else np.zeros(0, np.int64)
    out = np.empty(int(recv_counts.sum()), np.int64)
    i = 0
    for s in range(G):
        for e in range(El):
            n = int(recv_counts[s, e])
            base = int(expert_base[e]) + int(recv_counts[:s, e].sum())
            out[i:i + n] = base + np.arange(n)
            i += n
    return out


class EPMoELayer:
    """One MoE layer whose experts are sharded over `group` (see the module
    docstring). params: the full router (Wr [E, d], b [E]) and this rank's
    experts (Wg, Wu [El, f, d], Wd [El, d, f], El = E / G)."""

    def __init__(self, params: Dict[str, torch.Tensor], E: int, k: int, group=None, ops=None):
        self.group = group
        self.dist = dist.is_initialized()  # without a process group: one rank, no exchange
        self.G = dist.get_world_size(group) if self.dist else 1
        self.g = dist.get_rank(group) if self.dist else 0
        self.E, self.k = E, k
        if E % self.G:
            raise ValueError(f"E={E} experts do not split over {self.G} ranks")
        self.El = E // self.G
        self.Wr, self.b = params["Wr"], params["b"]
        self.Wg, self.Wu, self.Wd = params["Wg"], params["Wu"], params["Wd"]
        if self.Wg.shape[0] != self.El:
            raise ValueError("this rank's expert weights must hold E / G experts")
        self.ops = ops or KernelOps()
        dev, f32 = self.Wg.device, torch.float32
        self.grads = {
            "dWr": torch.zeros_like(self.Wr, dtype=f32),
            "db": torch.zeros(E, dtype=f32, device=dev),
            "dWg": torch.zeros(self.Wg.shape, dtype=f32, device=dev),
            "dWu": torch.zeros(self.Wu.shape, dtype=f32, device=dev),
            "dWd": torch.zeros(self.Wd.shape, dtype=f32, device=dev),
        }

    # -- exchanges ----------------------------------------------------------

    def _a2a_rows(self, rows: torch.Tensor, send: list, recv: list) -> torch.Tensor:
        out = rows.new_empty((sum(recv),) + tuple(rows.shape[1:]))
        if not self.dist:
            out.copy_(rows)
        else:
            dist.all_to_all_single(out, rows, output_split_sizes=recv, input_split_sizes=send,
                                   group=self.group)
        return out

    def _exchange_counts(self, counts: torch.Tensor, group_counts: torch.Tensor):
        """All-to-all of the per-expert counts; returns the received counts on
        the device [G, El], and on the host (with this rank's own send splits)
        from one device-to-host copy: the split sizes of the row all-to-alls
        must be known on the host."""
        recv = torch.empty_like(counts)
        if not self.dist:
            recv.copy_(counts)
        else:
            dist.all_to_all_single(recv, counts, group=self.group)
        host = torch.cat([recv, group_counts.to(recv.dtype)]).cpu().numpy()
        n = self.G * self.El
        return recv.view(self.G, self.El), host[:n].reshape(self.G, self.El), [int(v) for v in host[n:]]

    # -- forward / backward -------------------------------------------------

    def forward(self, x: torch.Tensor, mark=None) -> torch.Tensor:
        """Y = layer(x). `mark(name)`, if given, is called after each step
        (names starting with "a2a" are the exchanges)."""
        mark = mark or _no_mark
        ops, k, dev = self.ops, self.k, x.device
        T = x.shape[0]
        z = ops.router_logits(x, self.Wr, self.b)
        r = ops.route(z, k, self.G)
        xp = ops.permute(x, r["row_of_pair"], k)
        mark("route_permute")
        recv_dev, recv_counts, send = self._exchange_counts(r["counts"], r["group_counts"])
        recv = [int(v) for v in recv_counts.sum(axis=1)]
        mark("a2a_counts")
        xr = self._a2a_rows(xp, send, recv)
        mark("a2a_rows_fwd")
        m, loc_off = ops.regroup(recv_dev, recv_counts)
        xl = ops.permute(xr, m, 1)
        ffn = ops.ffn_fwd(xl, self.Wg, self.Wu, self.Wd, loc_off)
        yl = ops.gather_rows(ffn["yp"], m)
        mark("local_ffn_fwd")
        yp = self._a2a_rows(yl, recv, send)
        mark("a2a_rows_back")
        Y = ops.combine(yp, r["topk_w"], r["row_of_pair"])
        mark("combine")
        self.saved = dict(T=T, x=x, z=z, r=r, xp=xp, yp=yp, send=send, recv=recv, m=m, loc_off=loc_off,
                          xl=xl, **{n: ffn[n] for n in ("h1", "h2", "a")})
        return Y

    def backward(self, dY: torch.Tensor, accumulate: bool = True, mark=None) -> torch.Tensor:
        mark = mark or _no_mark
        ops, k, s = self.ops, self.k, self.saved
        r, g = s["r"], self.grads
        dyp, dg = ops.combine_bwd(dY, s["yp"], r["topk_w"], r["row_of_pair"])
        dlogits = ops.route_bwd(dg, r["topk_w"], r["topk_idx"], self.E)
        mark("combine_route_bwd")
        dyr = self._a2a_rows(dyp, s["send"], s["recv"])
        mark("a2a_rows_bwd")
        dyl = ops.permute(dyr, s["m"], 1)
        dxl = ops.ffn_bwd(s["xl"], self.Wg, self.Wu, self.Wd, s["h1"], s["h2"], s["a"], dyl, s["loc_off"],
                          g["dWg"], g["dWu"], g["dWd"], accumulate)
        dxr = ops.gather_rows(dxl, s["m"])
        mark("local_ffn_bwd")
        dxp = self._a2a_rows(dxr, s["recv"], s["send"])
        mark("a2a_rows_bwd_back")
        dX = ops.permute_bwd(dxp, r["row_of_pair"], dlogits, self.Wr, r["topk_idx"], s["T"], k)
        ops.router_bwd(s["xp"], dlogits, r["pair_of_row"], r["offsets"], k, g["dWr"], g["db"], accumulate)
        mark("permute_router_bwd")
        return dX
