"""CPU oracle of the MoE layer hot path (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg import
this package. The library never does: it shares no code with the CUDA path.

`moe_oracle.c` holds the arithmetic (plain loops, double precision, fp32 only
for the router logits that decide the top-k); this module builds it with gcc,
loads it with ctypes and moves numpy arrays in and out. Each wrapper names the
C function it calls; the C file documents the definition each one follows and
the page passage it comes from.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

FLAG_NONFINITE = 1


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so (plain gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = ctypes.CDLL(_LIB)
            _declare(_lib)
    return _lib


_i64 = ctypes.c_int64
_i32 = ctypes.c_int
_p = ctypes.c_void_p


def _declare(L):
    L.orc_router_logits_f32.argtypes = [_p, _p, _p, _i64, _i32, _i32, _p]
    L.orc_router_logits_f64.argtypes = [_p, _p, _p, _i64, _i32, _i32, _p]
    L.orc_route.argtypes = [_p, _i64, _i32, _i32, _p, _p]
    L.orc_route.restype = _i32
    L.orc_dispatch_layout.argtypes = [_p, _i64, _i32, _i32, _i32, _p, _p, _p, _p, _p, _p]
    L.orc_dispatch_layout.restype = _i32
    L.orc_permute.argtypes = [_p, _i64, _i32, _i32, _p, _p]
    L.orc_expert_ffn_fwd.argtypes = [_p, _p, _p, _p, _p, _i32, _i32, _i32, _p, _p, _p, _p]
    L.orc_combine.argtypes = [_p, _p, _p, _i64, _i32, _i32, _p]
    L.orc_combine_bwd.argtypes = [_p, _p, _p, _p, _i64, _i32, _i32, _p, _p]
    L.orc_route_bwd.argtypes = [_p, _p, _p, _i64, _i32, _i32, _p]
    L.orc_expert_ffn_bwd.argtypes = [_p] * 9 + [_i32, _i32, _i32] + [_p] * 4
    L.orc_permute_bwd.argtypes = [_p, _p, _i64, _i32, _i32, _p]
    L.orc_router_bwd.argtypes = [_p, _p, _p, _i64, _i32, _i32, _p, _p, _p]
    L.orc_tokens_fwd.argtypes = [_p, _p, _p, _i64, _i32, _p, _p, _p, _i32, _i32, _p, _p]
    L.orc_tokens_bwd.argtypes = [_p, _p, _p, _p, _p, _i64, _i32, _i32, _p, _p, _p, _p,
                                 _i32, _i32, _p, _p]
    L.orc_wgrad_columns.argtypes = [_p, _p, _p, _i64, _p, _p, _p, _i32, _i32, _p, _i32,
                                    _p, _p, _p]
    L.orc_num_threads.restype = _i32
    L.orc_aux_loss.argtypes = [_p, _p, _i64, _i32, _i32, ctypes.c_double, _p, _p, _p]
    L.orc_aux_loss_bwd.argtypes = [_p, _p, _i64, _i32, _i32, ctypes.c_double, ctypes.c_double, _p]


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return lib().orc_num_threads()


# --------------------------------------------------------------- routing

def router_logits_f32(x, Wr, b) -> np.ndarray:
    """fp32 logits with one fma per element in ascending order (orc_router_logits_f32)."""
    x = _c(x, np.float32); Wr = _c(Wr, np.float32); b = _c(b, np.float32)
    T, d = x.shape
    E = Wr.shape[0]
    z = np.empty((T, E), np.float32)
    lib().orc_router_logits_f32(_ptr(x), _ptr(Wr), _ptr(b), T, d, E, _ptr(z))
    return z


def router_logits_f64(x, Wr, b) -> np.ndarray:
    """The logits in double (orc_router_logits_f64)."""
    x = _c(x, np.float64); Wr = _c(Wr, np.float64); b = _c(b, np.float64)
    T, d = x.shape
    E = Wr.shape[0]
    z = np.empty((T, E), np.float64)
    lib().orc_router_logits_f64(_ptr(x), _ptr(Wr), _ptr(b), T, d, E, _ptr(z))
    return z


def route(z, k: int):
    """Top-k selection and gate weights (orc_route). Returns (idx int32 [T,k], w f64 [T,k], flags)."""
    z = _c(z, np.float64)
    T, E = z.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    flags = lib().orc_route(_ptr(z), T, E, k, _ptr(idx), _ptr(w))
    return idx, w, flags


def dispatch_layout(idx, E: int, G: int) -> Dict[str, np.ndarray]:
    """Counts, offsets, permutation and group layout (orc_dispatch_layout)."""
    idx = _c(idx, np.int32)
    T, k = idx.shape
    P = T * k
    out = {
        "counts": np.empty(E, np.int32),
        "offsets": np.empty(E + 1, np.int64),
        "group_counts": np.empty(G, np.int32),
        "group_offsets": np.empty(G + 1, np.int64),
        "row_of_pair": np.empty(max(P, 1), np.int32)[:P],
        "pair_of_row": np.empty(max(P, 1), np.int32)[:P],
    }
    rc = lib().orc_dispatch_layout(_ptr(idx), T, E, k, G, _ptr(out["counts"]), _ptr(out["offsets"]),
                                   _ptr(out["group_counts"]), _ptr(out["group_offsets"]),
                                   _ptr(out["row_of_pair"]), _ptr(out["pair_of_row"]))
    if rc != 0:
        raise ValueError("E % G != 0")
    return out


# ------------------------------------------------------ dispatch / combine

def permute(x, pair_of_row, k: int) -> np.ndarray:
    x = _c(x, np.float64); por = _c(pair_of_row, np.int32)
    T, d = x.shape
    xp = np.empty((T * k, d), np.float64)
    lib().orc_permute(_ptr(x), T, d, k, _ptr(por), _ptr(xp))
    return xp


def expert_ffn_fwd(xp, Wg, Wu, Wd, offsets):
    xp = _c(xp, np.float64); Wg = _c(Wg, np.float64); Wu = _c(Wu, np.float64); Wd = _c(Wd, np.float64)
    off = _c(offsets, np.int64)
    E, f, d = Wg.shape
    P = xp.shape[0]
    h1 = np.empty((P, f)); h2 = np.empty((P, f)); a = np.empty((P, f)); yp = np.empty((P, d))
    lib().orc_expert_ffn_fwd(_ptr(xp), _ptr(Wg), _ptr(Wu), _ptr(Wd), _ptr(off), E, d, f,
                             _ptr(h1), _ptr(h2), _ptr(a), _ptr(yp))
    return h1, h2, a, yp


def combine(yp, w, row_of_pair) -> np.ndarray:
    yp = _c(yp, np.float64); w = _c(w, np.float64); rop = _c(row_of_pair, np.int32)
    T, k = w.shape
    d = yp.shape[1]
    Y = np.empty((T, d))
    lib().orc_combine(_ptr(yp), _ptr(w), _ptr(rop), T, d, k, _ptr(Y))
    return Y


def combine_bwd(dY, yp, w, row_of_pair):
    dY = _c(dY, np.float64); yp = _c(yp, np.float64); w = _c(w, np.float64)
    rop = _c(row_of_pair, np.int32)
    T, k = w.shape
    d = dY.shape[1]
    dyp = np.zeros((T * k, d)); dg = np.empty((T, k))
    lib().orc_combine_bwd(_ptr(dY), _ptr(yp), _ptr(w), _ptr(rop), T, d, k, _ptr(dyp), _ptr(dg))
    return dyp, dg


def route_bwd(dg, w, idx, E: int) -> np.ndarray:
    dg = _c(dg, np.float64); w = _c(w, np.float64); idx = _c(idx, np.int32)
    T, k = w.shape
    dz = np.empty((T, E))
    lib().orc_route_bwd(_ptr(dg), _ptr(w), _ptr(idx), T, E, k, _ptr(dz))
    return dz


def expert_ffn_bwd(xp, Wg, Wu, Wd, h1, h2, a, dyp, offsets, dWg=None, dWu=None, dWd=None):
    xp = _c(xp, np.float64); Wg = _c(Wg, np.float64); Wu = _c(Wu, np.float64); Wd = _c(Wd, np.float64)
    h1 = _c(h1, np.float64); h2 = _c(h2, np.float64); a = _c(a, np.float64); dyp = _c(dyp, np.float64)
    off = _c(offsets, np.int64)
    E, f, d = Wg.shape
    P = xp.shape[0]
    dxp = np.empty((P, d))
    dWg = np.zeros((E, f, d)) if dWg is None else _c(dWg, np.float64).copy()
    dWu = np.zeros((E, f, d)) if dWu is None else _c(dWu, np.float64).copy()
    dWd = np.zeros((E, d, f)) if dWd is None else _c(dWd, np.float64).copy()
    lib().orc_expert_ffn_bwd(_ptr(xp), _ptr(Wg), _ptr(Wu), _ptr(Wd), _ptr(h1), _ptr(h2), _ptr(a),
                             _ptr(dyp), _ptr(off), E, d, f, _ptr(dxp), _ptr(dWg), _ptr(dWu), _ptr(dWd))
    return dxp, dWg, dWu, dWd


def permute_bwd(dxp, row_of_pair, T: int, k: int) -> np.ndarray:
    dxp = _c(dxp, np.float64); rop = _c(row_of_pair, np.int32)
    d = dxp.shape[1]
    dX = np.empty((T, d))
    lib().orc_permute_bwd(_ptr(dxp), _ptr(rop), T, d, k, _ptr(dX))
    return dX


def router_bwd(x, Wr, dz, dX, dWr=None, db=None):
    x = _c(x, np.float64); Wr = _c(Wr, np.float64); dz = _c(dz, np.float64)
    dX = _c(dX, np.float64).copy()
    T, d = x.shape
    E = Wr.shape[0]
    dWr = np.zeros((E, d)) if dWr is None else _c(dWr, np.float64).copy()
    db = np.zeros(E) if db is None else _c(db, np.float64).copy()
    lib().orc_router_bwd(_ptr(x), _ptr(Wr), _ptr(dz), T, d, E, _ptr(dX), _ptr(dWr), _ptr(db))
    return dX, dWr, db


# ------------------------------------------- auxiliary load-balancing loss

def aux_loss(z, counts, k: int, alpha: float):
    """Switch-style balance loss and routing metrics (orc_aux_loss).
    Returns dict(importance [E], loss, entropy)."""
    z = _c(z, np.float64); counts = _c(counts, np.int32)
    T, E = z.shape
    imp = np.zeros(E)
    loss = np.zeros(1); ent = np.zeros(1)
    lib().orc_aux_loss(_ptr(z), _ptr(counts), T, E, k, float(alpha), _ptr(imp), _ptr(loss), _ptr(ent))
    return dict(importance=imp, loss=float(loss[0]), entropy=float(ent[0]))


def aux_loss_bwd(z, counts, k: int, alpha: float, dL: float = 1.0) -> np.ndarray:
    """Gradient of the balance loss in the logits, counts held fixed (orc_aux_loss_bwd)."""
    z = _c(z, np.float64); counts = _c(counts, np.int32)
    T, E = z.shape
    dz = np.zeros((T, E))
    lib().orc_aux_loss_bwd(_ptr(z), _ptr(counts), T, E, k, float(alpha), float(dL), _ptr(dz))
    return dz


# ------------------------------------------------- per-token brute force

def tokens_fwd(xs, idx, w, Wg, Wu, Wd):
    """Per-token evaluation with no permutation (orc_tokens_fwd). Returns (Y, ys)."""
    xs = _c(xs, np.float64); idx = _c(idx, np.int32); w = _c(w, np.float64)
    Wg = _c(Wg, np.float64); Wu = _c(Wu, np.float64); Wd = _c(Wd, np.float64)
    n, k = idx.shape
    E, f, d = Wg.shape
    Y = np.empty((n, d)); ys = np.empty((n, k, d))
    lib().orc_tokens_fwd(_ptr(xs), _ptr(idx), _ptr(w), n, k, _ptr(Wg), _ptr(Wu), _ptr(Wd), d, f,
                         _ptr(Y), _ptr(ys))
    return Y, ys


def tokens_bwd(xs, dYs, idx, w, ys, Wr, Wg, Wu, Wd):
    """Per-token backward (orc_tokens_bwd). Returns (dz [n,E], dX [n,d])."""
    xs = _c(xs, np.float64); dYs = _c(dYs, np.float64); idx = _c(idx, np.int32)
    w = _c(w, np.float64); ys = _c(ys, np.float64); Wr = _c(Wr, np.float64)
    Wg = _c(Wg, np.float64); Wu = _c(Wu, np.float64); Wd = _c(Wd, np.float64)
    n, k = idx.shape
    E, f, d = Wg.shape
    dz = np.empty((n, E)); dX = np.empty((n, d))
    lib().orc_tokens_bwd(_ptr(xs), _ptr(dYs), _ptr(idx), _ptr(w), _ptr(ys), n, k, E, _ptr(Wr),
                         _ptr(Wg), _ptr(Wu), _ptr(Wd), d, f, _ptr(dz), _ptr(dX))
    return dz, dX


def wgrad_columns(xs, dYs, gs, Wg_e, Wu_e, Wd_e, cols):
    """Selected columns of one expert's dWg rows, dWu rows and dWd columns (orc_wgrad_columns)."""
    xs = _c(xs, np.float64); dYs = _c(dYs, np.float64); gs = _c(gs, np.float64)
    Wg_e = _c(Wg_e, np.float64); Wu_e = _c(Wu_e, np.float64); Wd_e = _c(Wd_e, np.float64)
    cols = _c(cols, np.int32)
    n, d = xs.shape
    f = Wg_e.shape[0]
    q = cols.shape[0]
    og = np.empty((q, d)); ou = np.empty((q, d)); od = np.empty((q, d))
    lib().orc_wgrad_columns(_ptr(xs), _ptr(dYs), _ptr(gs), n, _ptr(Wg_e), _ptr(Wu_e), _ptr(Wd_e),
                            d, f, _ptr(cols), q, _ptr(og), _ptr(ou), _ptr(od))
    return og, ou, od


# ------------------------------------------------------ composed layer

def layer_forward(x, Wr, b, Wg, Wu, Wd, k: int, G: int = 1, logits: str = "f32"):
    """Whole forward in the permuted form: route, layout, permute, experts, combine.

    logits="f32" decides the top-k from the fp32 fixed-order logits (the
    kernel's precision); logits="f64" uses the double definition (for the
    finite-difference checks). Inputs are numpy arrays (any float type)."""
    x = np.asarray(x)
    E = Wr.shape[0]
    if logits == "f32":
        z = router_logits_f32(x, Wr, b).astype(np.float64)
    else:
        z = router_logits_f64(x, Wr, b)
    idx, w, flags = route(z, k)
    lay = dispatch_layout(idx, E, G)
    xp = permute(x, lay["pair_of_row"], k)
    h1, h2, a, yp = expert_ffn_fwd(xp, Wg, Wu, Wd, lay["offsets"])
    Y = combine(yp, w, lay["row_of_pair"])
    return dict(z=z, idx=idx, w=w, flags=flags, xp=xp, h1=h1, h2=h2, a=a, yp=yp, Y=Y, **lay)


def layer_backward(fw, x, dY, Wr, Wg, Wu, Wd, k: int, acc: Optional[dict] = None,
                   aux: Optional[tuple] = None):
    """Whole backward given the forward record `fw` and dY; dW terms add to `acc`.
    aux = (alpha, dL) adds the balance loss's gradient (dL times dL_aux/dz) to
    the router's."""
    T = x.shape[0]
    E = Wr.shape[0]
    dyp, dg = combine_bwd(dY, fw["yp"], fw["w"], fw["row_of_pair"])
    dz = route_bwd(dg, fw["w"], fw["idx"], E)
    if aux is not None:
        dz = dz + aux_loss_bwd(fw["z"], fw["counts"], k, aux[0], aux[1])
    acc = acc or {}
    dxp, dWg, dWu, dWd = expert_ffn_bwd(fw["xp"], Wg, Wu, Wd, fw["h1"], fw["h2"], fw["a"], dyp,
                                        fw["offsets"], acc.get("dWg"), acc.get("dWu"), acc.get("dWd"))
    dX0 = permute_bwd(dxp, fw["row_of_pair"], T, k)
    dX, dWr, db = router_bwd(x, Wr, dz, dX0, acc.get("dWr"), acc.get("db"))
    return dict(dyp=dyp, dg=dg, dz=dz, dxp=dxp, dX=dX, dWg=dWg, dWu=dWu, dWd=dWd, dWr=dWr, db=db)
