"""The C ABI on a machine without a GPU: the library loads, exports every
symbol include/moe.h declares, and rejects invalid arguments with the
documented codes before touching CUDA (no kernel is launched here)."""
import ctypes
import os
import re

import pytest

from grouped_expert_ffn_top_b200 import native as N

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(N.LIB_PATH):
        from grouped_expert_ffn_top_b200 import build
        build.build()
    return N.lib()


def test_header_declares_the_path():
    syms = declared_symbols()
    for name in ("moe_router_logits", "moe_route", "moe_permute", "moe_grouped_ffn_fwd",
                 "moe_unpermute_combine", "moe_unpermute_combine_bwd", "moe_route_bwd",
                 "moe_grouped_ffn_bwd", "moe_grouped_ffn_dgrad", "moe_grouped_ffn_wgrad",
                 "moe_permute_bwd", "moe_router_bwd", "moe_get_error", "moe_last_error"):
        assert name in syms


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
    assert set(declared_symbols()) <= set(N.exported_symbols()) | {"moe_launch_count"}


def test_exports_nothing_else():
    out = os.popen(f"nm -D --defined-only {N.LIB_PATH}").read()
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert exported == set(declared_symbols())


def test_version_and_counter(L):
    assert L.moe_version() == 1
    assert L.moe_launch_count() >= 0


def test_workspace_sizes(L):
    assert L.moe_route_workspace_bytes(0, 8) >= 256
    big = L.moe_route_workspace_bytes(32768, 64)
    assert big >= 256 + 2 * 4 * (32768 // 256) * 64
    assert L.moe_route_workspace_bytes(-1, 8) == 0
    assert L.moe_grouped_ffn_bwd_workspace_bytes(1000, 8, 256, 384, N.MOE_BF16) >= 2 * 1000 * 384 * 2
    assert L.moe_router_bwd_workspace_bytes(8192, 1024, 8) >= 256 + 4 * (8192 // 256 + 8) * 1025


null = ctypes.c_void_p(0)


def test_route_argument_errors(L):
    code = L.moe_route(null, 4, 8, 9, 1, *([null] * 8), null, 0, null)
    assert code == N.MOE_ERR_INVALID_ARG
    assert b"k=9" in L.moe_last_error()
    assert L.moe_route(null, 4, 8, 0, 1, *([null] * 8), null, 0, null) == N.MOE_ERR_INVALID_ARG
    assert L.moe_route(null, 4, 6, 2, 4, *([null] * 8), null, 0, null) == N.MOE_ERR_UNSUPPORTED
    assert L.moe_route(null, 4, 2048, 2, 1, *([null] * 8), null, 0, null) == N.MOE_ERR_UNSUPPORTED
    assert L.moe_route(null, 4, 64, 33, 1, *([null] * 8), null, 0, null) == N.MOE_ERR_UNSUPPORTED
    # T = 0 is valid and launches nothing, even with null pointers
    assert L.moe_route(null, 0, 8, 2, 1, *([null] * 8), null, 0, null) == N.MOE_OK
    # null outputs with T > 0
    assert L.moe_route(null, 4, 8, 2, 1, *([null] * 8), null, 0, null) == N.MOE_ERR_INVALID_ARG


def test_ffn_argument_errors(L):
    args = [null] * 4 + [N.MOE_BF16, null, 100, 4, 100, 128] + [null] * 4 + [null, 0, null]
    assert L.moe_grouped_ffn_fwd(*args) == N.MOE_ERR_UNSUPPORTED  # d % 64 != 0 for bf16
    args = [null] * 4 + [7, null, 100, 4, 128, 128] + [null] * 4 + [null, 0, null]
    assert L.moe_grouped_ffn_fwd(*args) == N.MOE_ERR_UNSUPPORTED  # unknown dtype
    args = [null] * 4 + [N.MOE_BF16, null, 0, 4, 128, 128] + [null] * 4 + [null, 0, null]
    assert L.moe_grouped_ffn_fwd(*args) == N.MOE_OK  # no rows: nothing to do
    args = [null] * 4 + [N.MOE_BF16, null, 10, 4, 128, 128] + [null] * 4 + [null, 0, null]
    assert L.moe_grouped_ffn_fwd(*args) == N.MOE_ERR_INVALID_ARG  # null pointers
    args = [null] * 4 + [N.MOE_F32, null, 10, 4, 130, 128] + [null] * 4 + [null, 0, null]
    assert L.moe_grouped_ffn_fwd(*args) == N.MOE_ERR_UNSUPPORTED  # fp32 needs multiples of 4


def test_row_pass_argument_errors(L):
    assert L.moe_permute(null, N.MOE_BF16, 4, 100, 2, null, null, null) == N.MOE_ERR_UNSUPPORTED
    assert L.moe_permute(null, N.MOE_BF16, -1, 128, 2, null, null, null) == N.MOE_ERR_INVALID_ARG
    assert L.moe_permute(null, N.MOE_BF16, 0, 128, 2, null, null, null) == N.MOE_OK
    assert L.moe_unpermute_combine(null, null, null, N.MOE_BF16, 4, 128, 40, null, null) == \
        N.MOE_ERR_UNSUPPORTED
    assert L.moe_permute_bwd(null, null, null, null, null, N.MOE_BF16, 4, 128, 2, 3, null, null) == \
        N.MOE_ERR_INVALID_ARG  # k > E
    assert L.moe_route_bwd(null, null, null, 4, 8, 9, null, null) == N.MOE_ERR_INVALID_ARG
    assert L.moe_router_bwd(null, null, null, null, N.MOE_BF16, 0, 128, 8, 2, null, null, 1, null, 0,
                            null) == N.MOE_OK
    assert L.moe_router_bwd(null, null, null, null, N.MOE_BF16, 4, 128, 8, 9, null, null, 1, null, 0,
                            null) == N.MOE_ERR_INVALID_ARG
    # accumulate must be 0 or 1; writing the gradient of an empty batch needs the buffer
    assert L.moe_router_bwd(null, null, null, null, N.MOE_BF16, 0, 128, 8, 2, null, null, 2, null, 0,
                            null) == N.MOE_ERR_INVALID_ARG
    assert L.moe_router_bwd(null, null, null, null, N.MOE_BF16, 0, 128, 8, 2, null, null, 0, null, 0,
                            null) == N.MOE_ERR_INVALID_ARG


def test_wgrad_accumulate_flag_errors(L):
    args = [null] * 5 + [N.MOE_BF16, null, 0, 4, 128, 128, null, null, null]
    assert L.moe_grouped_ffn_wgrad(*args, 1, null, 0, null) == N.MOE_OK  # empty batch, adding
    assert L.moe_grouped_ffn_wgrad(*args, 2, null, 0, null) == N.MOE_ERR_INVALID_ARG
    assert L.moe_grouped_ffn_wgrad(*args, 0, null, 0, null) == N.MOE_ERR_INVALID_ARG  # null dW
    bargs = [null] * 8 + [N.MOE_BF16, null, 0, 4, 128, 128, null, null, null, null]
    assert L.moe_grouped_ffn_bwd(*bargs, 1, null, 0, null) == N.MOE_OK
    assert L.moe_grouped_ffn_bwd(*bargs, 0, null, 0, null) == N.MOE_ERR_INVALID_ARG


def test_balance_loss_argument_errors(L):
    f = ctypes.c_float
    assert L.moe_aux_loss(null, null, 4, 8, 9, f(0.01), null, null, null, null, 0, null) == \
        N.MOE_ERR_INVALID_ARG  # k > E
    assert L.moe_aux_loss(null, null, 4, 2048, 2, f(0.01), null, null, null, null, 0, null) == \
        N.MOE_ERR_UNSUPPORTED  # E > MOE_MAX_EXPERTS
    assert L.moe_aux_loss(null, null, 4, 8, 2, f(0.01), null, null, null, null, 0, null) == \
        N.MOE_ERR_INVALID_ARG  # null outputs
    assert L.moe_aux_loss_bwd(null, null, 0, 8, 2, f(0.01), f(1.0), null, null) == N.MOE_OK
    assert L.moe_aux_loss_workspace_bytes(1000, 64) >= 256 + 4 * 4 * 65
    args = [null, null, null, N.MOE_BF16, 10, 130, 8, null, null, null]
    assert L.moe_router_bwd_dense(*args, 1, null, 0, null) == N.MOE_ERR_UNSUPPORTED  # d % 4
    args = [null, null, null, N.MOE_BF16, 0, 128, 8, null, null, null]
    assert L.moe_router_bwd_dense(*args, 2, null, 0, null) == N.MOE_ERR_INVALID_ARG  # accumulate
    assert L.moe_router_bwd_dense(*args, 1, null, 0, null) == N.MOE_ERR_INVALID_ARG  # null dWr
    assert L.moe_router_bwd_dense_workspace_bytes(512, 128, 8) >= 256 + 4 * 2 * 8 * 129


def test_gathered_dispatch_argument_errors(L):
    """The fused-dispatch entries check k, T and the row map before anything
    else (a fake non-null address stands in for pair_of_row: it is never read
    because every call here is rejected or has nothing to do)."""
    fake = ctypes.c_void_p(256)
    tail = [null] * 4 + [null, 0, null]  # h1, h2, a, yp, ws, ws_bytes, stream
    fwd = lambda por, T, k, dt=N.MOE_BF16, d=128: L.moe_grouped_ffn_fwd_gather(  # noqa: E731
        null, por, T, k, null, null, null, dt, null, 4, d, 128, *tail)
    assert fwd(null, 10, 2) == N.MOE_ERR_INVALID_ARG  # no row map
    assert b"null pointer" in L.moe_last_error()
    assert fwd(fake, 10, 0) == N.MOE_ERR_INVALID_ARG  # k < 1
    assert fwd(fake, 10, 33) == N.MOE_ERR_UNSUPPORTED  # k > 32
    assert fwd(fake, 10, 2, d=100) == N.MOE_ERR_UNSUPPORTED  # bf16 d % 64
    assert fwd(fake, -1, 2) == N.MOE_ERR_INVALID_ARG
    assert fwd(fake, 0, 2) == N.MOE_OK  # no tokens: nothing to do
    assert fwd(fake, 10, 2) == N.MOE_ERR_INVALID_ARG  # null operands
    rec = L.moe_grouped_ffn_recompute_gather(null, fake, 10, 0, null, null, N.MOE_BF16, null, 4, 128, 128,
                                             null, null, null, 0, null)
    assert rec == N.MOE_ERR_INVALID_ARG
    wg = lambda acc, T=0: L.moe_grouped_ffn_wgrad_gather(  # noqa: E731
        null, fake, T, 2, null, null, null, null, N.MOE_BF16, null, 4, 128, 128, null, null, null, acc,
        null, 0, null)
    assert wg(1) == N.MOE_OK  # empty batch, adding: nothing to do
    assert wg(2) == N.MOE_ERR_INVALID_ARG
    assert wg(0) == N.MOE_ERR_INVALID_ARG  # writing needs dW
    bw = L.moe_grouped_ffn_bwd_gather(null, null, 5, 2, *([null] * 7), N.MOE_BF16, null, 4, 128, 128,
                                      *([null] * 4), 1, null, 0, null)
    assert bw == N.MOE_ERR_INVALID_ARG
    rb = lambda T, k, acc: L.moe_router_bwd_gather(null, null, fake, null, N.MOE_BF16, T, 128, 8, k,  # noqa: E731
                                                  null, null, acc, null, 0, null)
    assert rb(0, 2, 1) == N.MOE_OK
    assert rb(4, 9, 1) == N.MOE_ERR_INVALID_ARG  # k > E
    assert rb(4, 2, 1) == N.MOE_ERR_INVALID_ARG  # null operands
