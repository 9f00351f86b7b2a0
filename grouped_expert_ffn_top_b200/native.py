"""Python binding of the C ABI in include/moe.h (ctypes, argument marshalling only).

Every function here has the name of the C entry point it calls, takes torch
CUDA tensors, passes their device pointers and the current CUDA stream, and
raises MoeError on a non-zero return. All arithmetic happens in the CUDA
kernels of libmoe_b200.so; if that library is missing this module fails on
first use (there is no other implementation to fall back to).
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Dict, Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_F32 = 0
MOE_BF16 = 1
MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_WORKSPACE = -3
MOE_ERR_CUDA = -4
MOE_DEVERR_NONFINITE_LOGIT = 1
MOE_DEVERR_TIMEOUT = 2

_lock = threading.Lock()
_lib = None


class MoeError(RuntimeError):
    def __init__(self, code: int, fn: str, msg: str):
        super().__init__(f"{fn} returned {code}: {msg}")
        self.code = code


_p = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t
_f = ctypes.c_float

_SIGNATURES = {
    "moe_last_error": ([], ctypes.c_char_p),
    "moe_version": ([], _i),
    "moe_launch_count": ([], _i64),
    "moe_selftest_wait_timeout": ([_p, ctypes.c_longlong, _p], _i),
    "moe_get_error": ([_p, _p], _i),
    "moe_router_logits": ([_p, _p, _p, _i, _i64, _i, _i, _p, _p], _i),
    "moe_route_workspace_bytes": ([_i64, _i], _sz),
    "moe_route": ([_p, _i64, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p], _i),
    "moe_route_noalloc": ([_p, _i64, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p], _i),
    "moe_permute": ([_p, _i, _i64, _i, _i, _p, _p, _p], _i),
    "moe_grouped_ffn_fwd_workspace_bytes": ([_i64, _i, _i, _i, _i], _sz),
    "moe_grouped_ffn_fwd": ([_p, _p, _p, _p, _i, _p, _i64, _i, _i, _i, _p, _p, _p, _p, _p, _sz, _p], _i),
    "moe_unpermute_combine": ([_p, _p, _p, _i, _i64, _i, _i, _p, _p], _i),
    "moe_unpermute_combine_bwd": ([_p, _p, _p, _p, _i, _i64, _i, _i, _p, _p, _p], _i),
    "moe_route_bwd": ([_p, _p, _p, _i64, _i, _i, _p, _p], _i),
    "moe_grouped_ffn_bwd_workspace_bytes": ([_i64, _i, _i, _i, _i], _sz),
    "moe_grouped_ffn_wgrad_workspace_bytes": ([_i, _i], _sz),
    "moe_grouped_ffn_bwd": ([_p] * 8 + [_i, _p, _i64, _i, _i, _i, _p, _p, _p, _p, _i, _p, _sz, _p], _i),
    "moe_grouped_ffn_dgrad": ([_p] * 6 + [_i, _p, _i64, _i, _i, _i, _p, _p, _p, _p, _sz, _p], _i),
    "moe_grouped_ffn_wgrad": ([_p] * 5 + [_i, _p, _i64, _i, _i, _i, _p, _p, _p, _i, _p, _sz, _p], _i),
    "moe_permute_bwd": ([_p, _p, _p, _p, _p, _i, _i64, _i, _i, _i, _p, _p], _i),
    "moe_ep_regroup": ([_p, _i, _i, _p, _p, _p], _i),
    "moe_router_bwd_workspace_bytes": ([_i64, _i, _i], _sz),
    "moe_router_bwd": ([_p, _p, _p, _p, _i, _i64, _i, _i, _i, _p, _p, _i, _p, _sz, _p], _i),
    "moe_aux_loss_workspace_bytes": ([_i64, _i], _sz),
    "moe_grouped_ffn_recompute": ([_p, _p, _p, _i, _p, _i64, _i, _i, _i, _p, _p, _p, _sz, _p], _i),
    "moe_aux_loss": ([_p, _p, _i64, _i, _i, _f, _p, _p, _p, _p, _sz, _p], _i),
    "moe_aux_loss_bwd": ([_p, _p, _i64, _i, _i, _f, _f, _p, _p], _i),
    "moe_router_bwd_dense_workspace_bytes": ([_i64, _i, _i], _sz),
    "moe_router_bwd_dense": ([_p, _p, _p, _i, _i64, _i, _i, _p, _p, _p, _i, _p, _sz, _p], _i),
    "moe_grouped_ffn_fwd_gather": ([_p, _p, _i64, _i, _p, _p, _p, _i, _p, _i, _i, _i, _p, _p, _p, _p, _p, _sz,
                                    _p], _i),
    "moe_grouped_ffn_recompute_gather": ([_p, _p, _i64, _i, _p, _p, _i, _p, _i, _i, _i, _p, _p, _p, _sz, _p],
                                         _i),
    "moe_grouped_ffn_bwd_gather": ([_p, _p, _i64, _i] + [_p] * 7 + [_i, _p, _i, _i, _i, _p, _p, _p, _p, _i, _p,
                                                                   _sz, _p], _i),
    "moe_grouped_ffn_wgrad_gather": ([_p, _p, _i64, _i] + [_p] * 4 + [_i, _p, _i, _i, _i, _p, _p, _p, _i, _p,
                                                                     _sz, _p], _i),
    "moe_router_bwd_gather": ([_p, _p, _p, _p, _i, _i64, _i, _i, _i, _p, _p, _i, _p, _sz, _p], _i),
}


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m grouped_expert_ffn_top_b200.build`"
                    " (the MoE layer has no non-CUDA implementation)")
            L = ctypes.CDLL(LIB_PATH)
            for name, (args, res) in _SIGNATURES.items():
                fn = getattr(L, name)
                fn.argtypes = args
                fn.restype = res
            _lib = L
    return _lib


def exported_symbols():
    return list(_SIGNATURES)


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    if t.dtype == torch.float32:
        return MOE_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _check(rc: int, fn: str):
    if rc != MOE_OK:
        raise MoeError(rc, fn, lib().moe_last_error().decode())


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _ws(nbytes: int, device) -> torch.Tensor:
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ----------------------------------------------------------------- calls

def moe_get_error(ws: torch.Tensor, stream=None) -> int:
    rc = lib().moe_get_error(_ptr(ws), _stream(stream))
    if rc < 0:
        _check(rc, "moe_get_error")
    return rc


def moe_launch_count() -> int:
    return lib().moe_launch_count()


def moe_router_logits(x, Wr, b, logits=None, stream=None):
    _contig(x, Wr, b)
    T, d = x.shape
    E = Wr.shape[0]
    if logits is None:
        logits = torch.empty((T, E), dtype=torch.float32, device=x.device)
    _check(lib().moe_router_logits(_ptr(x), _ptr(Wr), _ptr(b), _dt(x), T, d, E, _ptr(logits),
                                   _stream(stream)), "moe_router_logits")
    return logits


def moe_route_workspace_bytes(T: int, E: int) -> int:
    return lib().moe_route_workspace_bytes(T, E)


def route_outputs(T: int, E: int, k: int, G: int, device) -> Dict[str, torch.Tensor]:
    i32, i64 = torch.int32, torch.int64
    return {
        "topk_idx": torch.empty((T, k), dtype=i32, device=device),
        "topk_w": torch.empty((T, k), dtype=torch.float32, device=device),
        "counts": torch.zeros(E, dtype=i32, device=device),
        "offsets": torch.zeros(E + 1, dtype=i64, device=device),
        "group_counts": torch.zeros(G, dtype=i32, device=device),
        "group_offsets": torch.zeros(G + 1, dtype=i64, device=device),
        "row_of_pair": torch.empty(T * k, dtype=i32, device=device),
        "pair_of_row": torch.empty(T * k, dtype=i32, device=device),
    }


def moe_route(logits, k: int, ep_groups: int = 1, out=None, ws=None, stream=None):
    _contig(logits)
    T, E = logits.shape
    o = out if out is not None else route_outputs(T, E, k, ep_groups, logits.device)
    if ws is None:
        ws = _ws(moe_route_workspace_bytes(T, E), logits.device)
    _check(lib().moe_route(_ptr(logits), T, E, k, ep_groups, _ptr(o["topk_idx"]), _ptr(o["topk_w"]),
                           _ptr(o["counts"]), _ptr(o["offsets"]), _ptr(o["group_counts"]),
                           _ptr(o["group_offsets"]), _ptr(o["row_of_pair"]), _ptr(o["pair_of_row"]),
                           _ptr(ws), ws.numel(), _stream(stream)), "moe_route")
    return o


def moe_permute(x, row_of_pair, k: int, xp=None, stream=None):
    _contig(x, row_of_pair)
    T, d = x.shape
    if xp is None:
        xp = torch.empty((T * k, d), dtype=x.dtype, device=x.device)
    _check(lib().moe_permute(_ptr(x), _dt(x), T, d, k, _ptr(row_of_pair), _ptr(xp), _stream(stream)),
           "moe_permute")
    return xp


def moe_grouped_ffn_fwd_workspace_bytes(rows, E, d, f, dtype) -> int:
    return lib().moe_grouped_ffn_fwd_workspace_bytes(rows, E, d, f, dtype)


def moe_grouped_ffn_fwd(xp, Wg, Wu, Wd, expert_offsets, out=None, ws=None, stream=None):
    _contig(xp, Wg, Wu, Wd, expert_offsets)
    rows, d = xp.shape
    E, f, _ = Wg.shape
    dt = _dt(xp)
    if out is None:
        out = {n: torch.empty((rows, f), dtype=xp.dtype, device=xp.device) for n in ("h1", "h2", "a")}
        out["yp"] = torch.empty((rows, d), dtype=xp.dtype, device=xp.device)
    if ws is None:
        ws = _ws(moe_grouped_ffn_fwd_workspace_bytes(rows, E, d, f, dt), xp.device)
    _check(lib().moe_grouped_ffn_fwd(_ptr(xp), _ptr(Wg), _ptr(Wu), _ptr(Wd), dt, _ptr(expert_offsets),
                                     rows, E, d, f, _ptr(out["h1"]), _ptr(out["h2"]), _ptr(out["a"]),
                                     _ptr(out["yp"]), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_grouped_ffn_fwd")
    return out


def moe_grouped_ffn_recompute(xp, Wg, Wu, expert_offsets, h1, h2, ws=None, stream=None):
    """h1 = xp Wg_e^T, h2 = xp Wu_e^T for a forward that did not store them."""
    _contig(xp, Wg, Wu, expert_offsets, h1, h2)
    rows, d = xp.shape
    E, f, _ = Wg.shape
    dt = _dt(xp)
    if ws is None:
        ws = _ws(moe_grouped_ffn_fwd_workspace_bytes(rows, E, d, f, dt), xp.device)
    _check(lib().moe_grouped_ffn_recompute(_ptr(xp), _ptr(Wg), _ptr(Wu), dt, _ptr(expert_offsets), rows, E,
                                           d, f, _ptr(h1), _ptr(h2), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_grouped_ffn_recompute")


def moe_grouped_ffn_fwd_gather(x, pair_of_row, k: int, Wg, Wu, Wd, expert_offsets, out=None, ws=None,
                               stream=None):
    """moe_grouped_ffn_fwd on the dispatch rows x[pair_of_row[r] // k], read
    in place (no permuted copy)."""
    _contig(x, pair_of_row, Wg, Wu, Wd, expert_offsets)
    T, d = x.shape
    E, f, _ = Wg.shape
    rows, dt = T * k, _dt(x)
    if out is None:
        out = {n: torch.empty((rows, f), dtype=x.dtype, device=x.device) for n in ("h1", "h2", "a")}
        out["yp"] = torch.empty((rows, d), dtype=x.dtype, device=x.device)
    if ws is None:
        ws = _ws(moe_grouped_ffn_fwd_workspace_bytes(rows, E, d, f, dt), x.device)
    _check(lib().moe_grouped_ffn_fwd_gather(_ptr(x), _ptr(pair_of_row), T, k, _ptr(Wg), _ptr(Wu), _ptr(Wd), dt,
                                            _ptr(expert_offsets), E, d, f, _ptr(out["h1"]), _ptr(out["h2"]),
                                            _ptr(out["a"]), _ptr(out["yp"]), _ptr(ws), ws.numel(),
                                            _stream(stream)), "moe_grouped_ffn_fwd_gather")
    return out


def moe_grouped_ffn_recompute_gather(x, pair_of_row, k: int, Wg, Wu, expert_offsets, h1, h2, ws=None,
                                     stream=None):
    _contig(x, pair_of_row, Wg, Wu, expert_offsets, h1, h2)
    T, d = x.shape
    E, f, _ = Wg.shape
    dt = _dt(x)
    if ws is None:
        ws = _ws(moe_grouped_ffn_fwd_workspace_bytes(T * k, E, d, f, dt), x.device)
    _check(lib().moe_grouped_ffn_recompute_gather(_ptr(x), _ptr(pair_of_row), T, k, _ptr(Wg), _ptr(Wu), dt,
                                                  _ptr(expert_offsets), E, d, f, _ptr(h1), _ptr(h2), _ptr(ws),
                                                  ws.numel(), _stream(stream)),
           "moe_grouped_ffn_recompute_gather")


def moe_unpermute_combine(yp, topk_w, row_of_pair, Y=None, stream=None):
    _contig(yp, topk_w, row_of_pair)
    T, k = topk_w.shape
    d = yp.shape[1]
    if Y is None:
        Y = torch.empty((T, d), dtype=yp.dtype, device=yp.device)
    _check(lib().moe_unpermute_combine(_ptr(yp), _ptr(topk_w), _ptr(row_of_pair), _dt(yp), T, d, k,
                                       _ptr(Y), _stream(stream)), "moe_unpermute_combine")
    return Y


def moe_unpermute_combine_bwd(dY, yp, topk_w, row_of_pair, dyp=None, dg=None, stream=None):
    _contig(dY, yp, topk_w, row_of_pair)
    T, k = topk_w.shape
    d = dY.shape[1]
    if dyp is None:
        dyp = torch.empty((T * k, d), dtype=dY.dtype, device=dY.device)
    if dg is None:
        dg = torch.empty((T, k), dtype=torch.float32, device=dY.device)
    _check(lib().moe_unpermute_combine_bwd(_ptr(dY), _ptr(yp), _ptr(topk_w), _ptr(row_of_pair),
                                           _dt(dY), T, d, k, _ptr(dyp), _ptr(dg), _stream(stream)),
           "moe_unpermute_combine_bwd")
    return dyp, dg


def moe_route_bwd(dg, topk_w, topk_idx, E: int, dlogits=None, stream=None):
    _contig(dg, topk_w, topk_idx)
    T, k = topk_w.shape
    if dlogits is None:
        dlogits = torch.empty((T, E), dtype=torch.float32, device=dg.device)
    _check(lib().moe_route_bwd(_ptr(dg), _ptr(topk_w), _ptr(topk_idx), T, E, k, _ptr(dlogits),
                               _stream(stream)), "moe_route_bwd")
    return dlogits


def moe_aux_loss_workspace_bytes(T, E) -> int:
    return lib().moe_aux_loss_workspace_bytes(T, E)


def moe_aux_loss(logits, expert_counts, k: int, alpha: float, out=None, ws=None, stream=None):
    """Balance loss and routing metrics; returns dict(importance [E], loss [1], entropy [1])."""
    _contig(logits, expert_counts)
    T, E = logits.shape
    dev = logits.device
    o = out if out is not None else {
        "importance": torch.empty(E, dtype=torch.float32, device=dev),
        "loss": torch.empty(1, dtype=torch.float32, device=dev),
        "entropy": torch.empty(1, dtype=torch.float32, device=dev)}
    if ws is None:
        ws = _ws(moe_aux_loss_workspace_bytes(T, E), dev)
    _check(lib().moe_aux_loss(_ptr(logits), _ptr(expert_counts), T, E, k, float(alpha),
                              _ptr(o["importance"]), _ptr(o["loss"]), _ptr(o["entropy"]), _ptr(ws),
                              ws.numel(), _stream(stream)), "moe_aux_loss")
    return o


def moe_aux_loss_bwd(logits, expert_counts, k: int, alpha: float, dloss: float = 1.0,
                     dlogits_aux=None, stream=None):
    _contig(logits, expert_counts)
    T, E = logits.shape
    if dlogits_aux is None:
        dlogits_aux = torch.empty((T, E), dtype=torch.float32, device=logits.device)
    _check(lib().moe_aux_loss_bwd(_ptr(logits), _ptr(expert_counts), T, E, k, float(alpha), float(dloss),
                                  _ptr(dlogits_aux), _stream(stream)), "moe_aux_loss_bwd")
    return dlogits_aux


def moe_router_bwd_dense_workspace_bytes(T, d, E) -> int:
    return lib().moe_router_bwd_dense_workspace_bytes(T, d, E)


def moe_router_bwd_dense(x, Wr, dz, dX, dWr, db, accumulate: bool = True, ws=None, stream=None):
    """dX += dz Wr (dX may be None); dWr (+)= dz^T x; db (+)= column sums of dz."""
    _contig(x, Wr, dz, dX, dWr, db)
    T, d = x.shape
    E = Wr.shape[0]
    if ws is None:
        ws = _ws(moe_router_bwd_dense_workspace_bytes(T, d, E), x.device)
    _check(lib().moe_router_bwd_dense(_ptr(x), _ptr(Wr), _ptr(dz), _dt(x), T, d, E, _ptr(dX), _ptr(dWr),
                                      _ptr(db), int(accumulate), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_router_bwd_dense")


def moe_grouped_ffn_bwd_workspace_bytes(rows, E, d, f, dtype) -> int:
    return lib().moe_grouped_ffn_bwd_workspace_bytes(rows, E, d, f, dtype)


def moe_grouped_ffn_wgrad_workspace_bytes(E, dtype) -> int:
    return lib().moe_grouped_ffn_wgrad_workspace_bytes(E, dtype)


def moe_grouped_ffn_bwd(xp, Wg, Wu, Wd, h1, h2, a, dyp, expert_offsets, dWg, dWu, dWd,
                        dxp=None, ws=None, stream=None, accumulate: bool = True):
    _contig(xp, Wg, Wu, Wd, h1, h2, a, dyp, expert_offsets, dWg, dWu, dWd)
    rows, d = xp.shape
    E, f, _ = Wg.shape
    dt = _dt(xp)
    if dxp is None:
        dxp = torch.empty((rows, d), dtype=xp.dtype, device=xp.device)
    if ws is None:
        ws = _ws(moe_grouped_ffn_bwd_workspace_bytes(rows, E, d, f, dt), xp.device)
    _check(lib().moe_grouped_ffn_bwd(_ptr(xp), _ptr(Wg), _ptr(Wu), _ptr(Wd), _ptr(h1), _ptr(h2),
                                     _ptr(a), _ptr(dyp), dt, _ptr(expert_offsets), rows, E, d, f,
                                     _ptr(dxp), _ptr(dWg), _ptr(dWu), _ptr(dWd), int(accumulate), _ptr(ws),
                                     ws.numel(), _stream(stream)), "moe_grouped_ffn_bwd")
    return dxp


def moe_grouped_ffn_bwd_gather(x, pair_of_row, k: int, Wg, Wu, Wd, h1, h2, a, dyp, expert_offsets, dWg, dWu,
                               dWd, dxp=None, ws=None, stream=None, accumulate: bool = True):
    _contig(x, pair_of_row, Wg, Wu, Wd, h1, h2, a, dyp, expert_offsets, dWg, dWu, dWd)
    T, d = x.shape
    E, f, _ = Wg.shape
    rows, dt = T * k, _dt(x)
    if dxp is None:
        dxp = torch.empty((rows, d), dtype=x.dtype, device=x.device)
    if ws is None:
        ws = _ws(moe_grouped_ffn_bwd_workspace_bytes(rows, E, d, f, dt), x.device)
    _check(lib().moe_grouped_ffn_bwd_gather(_ptr(x), _ptr(pair_of_row), T, k, _ptr(Wg), _ptr(Wu), _ptr(Wd),
                                            _ptr(h1), _ptr(h2), _ptr(a), _ptr(dyp), dt, _ptr(expert_offsets),
                                            E, d, f, _ptr(dxp), _ptr(dWg), _ptr(dWu), _ptr(dWd),
                                            int(accumulate), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_grouped_ffn_bwd_gather")
    return dxp


def moe_grouped_ffn_dgrad(Wg, Wu, Wd, h1, h2, dyp, expert_offsets, dh1, dh2, dxp, ws, stream=None):
    _contig(Wg, Wu, Wd, h1, h2, dyp, expert_offsets, dh1, dh2, dxp)
    rows, d = dyp.shape
    E, f, _ = Wg.shape
    _check(lib().moe_grouped_ffn_dgrad(_ptr(Wg), _ptr(Wu), _ptr(Wd), _ptr(h1), _ptr(h2), _ptr(dyp),
                                       _dt(dyp), _ptr(expert_offsets), rows, E, d, f, _ptr(dh1),
                                       _ptr(dh2), _ptr(dxp), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_grouped_ffn_dgrad")
    return dxp


def moe_grouped_ffn_wgrad(xp, a, dyp, dh1, dh2, expert_offsets, dWg, dWu, dWd, ws, stream=None,
                          accumulate: bool = True):
    _contig(xp, a, dyp, dh1, dh2, expert_offsets, dWg, dWu, dWd)
    rows, d = xp.shape
    E, f, _ = dWg.shape
    _check(lib().moe_grouped_ffn_wgrad(_ptr(xp), _ptr(a), _ptr(dyp), _ptr(dh1), _ptr(dh2), _dt(xp),
                                       _ptr(expert_offsets), rows, E, d, f, _ptr(dWg), _ptr(dWu),
                                       _ptr(dWd), int(accumulate), _ptr(ws), ws.numel(),
                                       _stream(stream)),
           "moe_grouped_ffn_wgrad")


def moe_grouped_ffn_wgrad_gather(x, pair_of_row, k: int, a, dyp, dh1, dh2, expert_offsets, dWg, dWu, dWd, ws,
                                 stream=None, accumulate: bool = True):
    _contig(x, pair_of_row, a, dyp, dh1, dh2, expert_offsets, dWg, dWu, dWd)
    T, d = x.shape
    E, f, _ = dWg.shape
    _check(lib().moe_grouped_ffn_wgrad_gather(_ptr(x), _ptr(pair_of_row), T, k, _ptr(a), _ptr(dyp), _ptr(dh1),
                                              _ptr(dh2), _dt(x), _ptr(expert_offsets), E, d, f, _ptr(dWg),
                                              _ptr(dWu), _ptr(dWd), int(accumulate), _ptr(ws), ws.numel(),
                                              _stream(stream)),
           "moe_grouped_ffn_wgrad_gather")


def moe_permute_bwd(dxp, row_of_pair, dlogits, Wr, topk_idx, T: int, k: int, dX=None, stream=None):
    _contig(dxp, row_of_pair, dlogits, Wr, topk_idx)
    d = dxp.shape[1]
    E = Wr.shape[0] if Wr is not None else (dlogits.shape[1] if dlogits is not None else k)
    if dX is None:
        dX = torch.empty((T, d), dtype=dxp.dtype, device=dxp.device)
    _check(lib().moe_permute_bwd(_ptr(dxp), _ptr(row_of_pair), _ptr(dlogits), _ptr(Wr), _ptr(topk_idx),
                                 _dt(dxp), T, d, E, k, _ptr(dX), _stream(stream)), "moe_permute_bwd")
    return dX


def moe_ep_regroup(recv_counts, rows: int, stream=None):
    """Row map [rows] int32 and local offsets [El+1] int64 of the received
    rows (recv_counts [G, El] int32 on the device; rows = its sum, which the
    caller knows from its host copy of the counts)."""
    _contig(recv_counts)
    G, El = recv_counts.shape
    dev = recv_counts.device
    row_map = torch.empty(max(rows, 1), dtype=torch.int32, device=dev)
    local_offsets = torch.empty(El + 1, dtype=torch.int64, device=dev)
    _check(lib().moe_ep_regroup(_ptr(recv_counts), G, El, _ptr(row_map), _ptr(local_offsets),
                                _stream(stream)), "moe_ep_regroup")
    return row_map[:rows], local_offsets


def moe_router_bwd_workspace_bytes(rows, d, E) -> int:
    return lib().moe_router_bwd_workspace_bytes(rows, d, E)


def moe_router_bwd(xp, dlogits, pair_of_row, expert_offsets, k: int, dWr, db, ws=None, stream=None,
                   accumulate: bool = True):
    _contig(xp, dlogits, pair_of_row, expert_offsets, dWr, db)
    rows, d = xp.shape
    T, E = dlogits.shape
    if ws is None:
        ws = _ws(moe_router_bwd_workspace_bytes(rows, d, E), xp.device)
    _check(lib().moe_router_bwd(_ptr(xp), _ptr(dlogits), _ptr(pair_of_row), _ptr(expert_offsets),
                                _dt(xp), T, d, E, k, _ptr(dWr), _ptr(db), int(accumulate), _ptr(ws),
                                ws.numel(), _stream(stream)), "moe_router_bwd")


def moe_router_bwd_gather(x, dlogits, pair_of_row, expert_offsets, k: int, dWr, db, ws=None, stream=None,
                          accumulate: bool = True):
    """moe_router_bwd reading dispatch row r as x[pair_of_row[r] // k]."""
    _contig(x, dlogits, pair_of_row, expert_offsets, dWr, db)
    T, d = x.shape
    E = dlogits.shape[1]
    if ws is None:
        ws = _ws(moe_router_bwd_workspace_bytes(T * k, d, E), x.device)
    _check(lib().moe_router_bwd_gather(_ptr(x), _ptr(dlogits), _ptr(pair_of_row), _ptr(expert_offsets),
                                       _dt(x), T, d, E, k, _ptr(dWr), _ptr(db), int(accumulate), _ptr(ws),
                                       ws.numel(), _stream(stream)), "moe_router_bwd_gather")
