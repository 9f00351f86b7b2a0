"""Expert parallelism on the CPU: two and four gloo ranks (experts sharded
4 + 4, or 2 + 2 + 2 + 2), with uneven and empty microbatches and local experts
that receive no rows. The
layer's exchange logic (count all-to-all, ragged row all-to-alls, regroup by
local expert and back) runs as in production; the local steps run in the
oracle (test-only `OracleOps`), so every rank's Y and dX must equal the
single-process oracle layer to double precision, and its router gradients and
local expert gradients (summed over every rank's tokens) to their fp32
storage."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from grouped_expert_ffn_top_b200.ep import regroup_map  # noqa: E402


def test_regroup_map_orders_rows_by_expert_then_source():
    # 3 sources, 2 local experts; arrival order: s0(e0 x2, e1 x1), s1(e0 x0, e1 x2), s2(e0 x1, e1 x0)
    rc = np.array([[2, 1], [0, 2], [1, 0]])
    m = regroup_map(rc)
    # expert 0 rows: s0 q0, s0 q1, s2 q0 -> 0, 1, 2; expert 1 rows: s0 q0, s1 q0, s1 q1 -> 3, 4, 5
    assert m.tolist() == [0, 1, 3, 4, 5, 2]
    assert sorted(m.tolist()) == list(range(6))
    assert regroup_map(np.zeros((2, 3), np.int64)).size == 0


def _t(a, dtype=torch.float64):
    return torch.as_tensor(np.ascontiguousarray(a), dtype=dtype)


class OracleOps:
    """The layer's local steps in the oracle (float64, CPU tensors)."""

    def __init__(self, oracle):
        self.o = oracle

    def router_logits(self, x, Wr, b):
        return _t(self.o.router_logits_f64(x.numpy(), Wr.numpy(), b.numpy()))

    def route(self, z, k, G):
        idx, w, _ = self.o.route(z.numpy(), k)
        lay = self.o.dispatch_layout(idx, z.shape[1], G)
        r = {n: torch.as_tensor(v) for n, v in lay.items()}
        r.update(topk_idx=torch.as_tensor(idx), topk_w=_t(w))
        return r

    def permute(self, x, row_of_pair, k):
        rop = row_of_pair.numpy()
        por = np.empty_like(rop)
        por[rop] = np.arange(rop.size, dtype=rop.dtype)
        return _t(self.o.permute(x.numpy(), por, k)) if rop.size else x.new_empty((0, x.shape[1]))

    def regroup(self, recv_dev, recv_host):
        """The regroup map and local offsets on the host (regroup_map)."""
        m = torch.as_tensor(regroup_map(recv_host), dtype=torch.int64)
        off = torch.as_tensor(np.concatenate([[0], np.cumsum(recv_host.sum(axis=0))]), dtype=torch.int64)
        return m, off

    def gather_rows(self, src, rows_of):
        if rows_of.numel() == 0:
            return src.new_empty((0, src.shape[1]))
        return _t(self.o.permute_bwd(src.numpy(), rows_of.numpy(), rows_of.numel(), 1))

    def ffn_fwd(self, xp, Wg, Wu, Wd, offsets):
        h1, h2, a, yp = self.o.expert_ffn_fwd(xp.numpy(), Wg.numpy(), Wu.numpy(), Wd.numpy(), offsets.numpy())
        return dict(h1=_t(h1), h2=_t(h2), a=_t(a), yp=_t(yp))

    def combine(self, yp, topk_w, row_of_pair):
        return _t(self.o.combine(yp.numpy(), topk_w.numpy(), row_of_pair.numpy()))

    def combine_bwd(self, dY, yp, topk_w, row_of_pair):
        dyp, dg = self.o.combine_bwd(dY.numpy(), yp.numpy(), topk_w.numpy(), row_of_pair.numpy())
        return _t(dyp), _t(dg)

    def route_bwd(self, dg, topk_w, topk_idx, E):
        return _t(self.o.route_bwd(dg.numpy(), topk_w.numpy(), topk_idx.numpy(), E))

    def ffn_bwd(self, xp, Wg, Wu, Wd, h1, h2, a, dyp, offsets, dWg, dWu, dWd, accumulate):
        acc = [g.numpy().astype(np.float64) if accumulate else np.zeros(g.shape) for g in (dWg, dWu, dWd)]
        dxp, gg, gu, gd = self.o.expert_ffn_bwd(xp.numpy(), Wg.numpy(), Wu.numpy(), Wd.numpy(), h1.numpy(),
                                                h2.numpy(), a.numpy(), dyp.numpy(), offsets.numpy(), *acc)
        for dst, src in ((dWg, gg), (dWu, gu), (dWd, gd)):
            dst.copy_(_t(src))
        return _t(dxp)

    def permute_bwd(self, dxp, row_of_pair, dlogits, Wr, topk_idx, T, k):
        dX0 = self.o.permute_bwd(dxp.numpy(), row_of_pair.numpy(), T, k)
        dX, _, _ = self.o.router_bwd(np.zeros(dX0.shape), Wr.numpy(), dlogits.numpy(), dX0)
        return _t(dX)

    def router_bwd(self, xp, dlogits, pair_of_row, offsets, k, dWr, db, accumulate):
        T = dlogits.shape[0]
        x = np.zeros((T, xp.shape[1]))
        por = pair_of_row.numpy()
        x[por // k] = xp.numpy()
        _, gW, gb = self.o.router_bwd(x, dWr.numpy().astype(np.float64), dlogits.numpy(), np.zeros(x.shape),
                                      dWr.numpy().astype(np.float64) if accumulate else None,
                                      db.numpy().astype(np.float64) if accumulate else None)
        dWr.copy_(_t(gW)); db.copy_(_t(gb))


def _problem(Ts, d=12, E=8, f=16, seed=0):
    rng = np.random.default_rng(seed)
    Wr = rng.standard_normal((E, d)) * 0.5
    b = rng.standard_normal(E) * 0.3
    b[E - 1] = -1.0e4  # an expert no token selects: its rank receives nothing for it
    Wg = rng.standard_normal((E, f, d)) * 0.3
    Wu = rng.standard_normal((E, f, d)) * 0.3
    Wd = rng.standard_normal((E, d, f)) * 0.3
    xs = [rng.standard_normal((T, d)) for T in Ts]
    dYs = [rng.standard_normal((T, d)) for T in Ts]
    return Wr, b, Wg, Wu, Wd, xs, dYs


def _worker(rank, world, port, Ts, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    import oracle
    from grouped_expert_ffn_top_b200.ep import EPMoELayer
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        k, E = 2, 8
        Wr, b, Wg, Wu, Wd, xs, dYs = _problem(Ts)
        El = E // world
        sl = slice(rank * El, (rank + 1) * El)
        params = dict(Wr=_t(Wr), b=_t(b), Wg=_t(Wg[sl]), Wu=_t(Wu[sl]), Wd=_t(Wd[sl]))
        layer = EPMoELayer(params, E, k, ops=OracleOps(oracle))
        errs = {}
        for step, acc in ((0, False), (1, True)):
            Y = layer.forward(_t(xs[rank]))
            dX = layer.backward(_t(dYs[rank]), accumulate=acc)
            fw = oracle.layer_forward(xs[rank], Wr, b, Wg, Wu, Wd, k, world, logits="f64")
            bw = oracle.layer_backward(fw, xs[rank], dYs[rank], Wr, Wg, Wu, Wd, k)
            # local experts see every rank's tokens
            dWl = {n: np.zeros_like(bw[n][sl]) for n in ("dWg", "dWu", "dWd")}
            for r2 in range(world):
                f2 = oracle.layer_forward(xs[r2], Wr, b, Wg, Wu, Wd, k, world, logits="f64")
                b2 = oracle.layer_backward(f2, xs[r2], dYs[r2], Wr, Wg, Wu, Wd, k)
                for n in dWl:
                    dWl[n] += b2[n][sl]
            mult = 2.0 if acc else 1.0  # the second step adds the same gradients again
            ref = dict(Y=fw["Y"], dX=bw["dX"], dWr=mult * bw["dWr"], db=mult * bw["db"],
                       **{n: mult * v for n, v in dWl.items()})
            got = dict(Y=Y.numpy(), dX=dX.numpy(), **{n: layer.grads[n].numpy() for n in ("dWr", "db", "dWg",
                                                                                          "dWu", "dWd")})
            for n, v in ref.items():
                if v.size == 0:
                    errs[f"{n}@{step}"] = 0.0 if got[n].size == 0 else 1.0
                    continue
                scale = max(float(np.abs(v).max()), 1e-30)
                errs[f"{n}@{step}"] = float(np.abs(got[n] - v).max() / scale)
        out.put((rank, errs))
    except Exception:  # report instead of leaving the peer waiting in a collective
        import traceback
        out.put((rank, {"error": traceback.format_exc()}))
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("Ts", [(37, 0), (20, 13), (25, 0, 9, 1)],
                         ids=["2 ranks, one empty", "2 ranks", "4 ranks, uneven, one empty"])
def test_expert_parallel_layer_matches_oracle(Ts):
    """World size len(Ts): 2 ranks with experts sharded 4 + 4, and 4 ranks
    (expert groups of 2, the group count of the 32k workload's layout)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = len(Ts)
    procs = [ctx.Process(target=_worker, args=(r, world, port, Ts, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, errs in res.items():
        assert "error" not in errs, f"rank {rank} failed:\n{errs.get('error')}"
        for n, e in errs.items():
            # Y and dX stay in double; the parameter gradients live in fp32 buffers
            tol = 1e-12 if n.startswith(("Y@", "dX@")) else 1e-6
            assert e < tol, f"rank {rank} {n}: relative error {e:.2e}"
