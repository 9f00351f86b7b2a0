"""moe_route_noalloc: routing for callers that cannot allocate device memory.

Such callers (code inside a runtime that owns every device buffer, hosts that
forbid allocations after planning, paths where cudaMalloc's implicit device
synchronisation is not allowed) cannot hand moe_route a workspace; this entry
point uses a fixed array inside the library instead. The test calls it
through the C ABI twice in a row, on different logits, and checks every
output against moe_route on the same input. Run after the other GPU tests, the
array's address was looked up by an earlier call in this process; the last
test repeats the same check in a fresh Python process, where the first call
on the device makes that lookup.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from grouped_expert_ffn_top_b200 import native as N
from grouped_expert_ffn_top_b200 import workloads

pytestmark = pytest.mark.gpu


def _noalloc(logits, k, G, err):
    T, E = logits.shape
    o = N.route_outputs(T, E, k, G, logits.device)
    p = N._ptr
    rc = N.lib().moe_route_noalloc(p(logits), T, E, k, G, p(o["topk_idx"]), p(o["topk_w"]),
                                   p(o["counts"]), p(o["offsets"]), p(o["group_counts"]),
                                   p(o["group_offsets"]), p(o["row_of_pair"]), p(o["pair_of_row"]),
                                   p(err), N._stream(None))
    return rc, o


@pytest.mark.skipif(not torch.cuda.is_available(), reason="no CUDA device")
def test_noalloc_route_equals_moe_route_on_two_calls():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call, (T, E, k, G) in enumerate([(5000, 64, 8, 4), (777, 16, 2, 2)]):
        z = workloads.make_logits(T, E, device="cuda", seed=100 + call)
        rc, got = _noalloc(z, k, G, err)
        assert rc == N.MOE_OK, N.lib().moe_last_error()
        ref = N.moe_route(z, k, G)
        torch.cuda.synchronize()
        for name in ("topk_idx", "counts", "offsets", "group_counts", "group_offsets",
                     "row_of_pair", "pair_of_row"):
            assert torch.equal(got[name], ref[name]), (call, name)
        # same kernels: the gate weights agree to the bit, far inside the 1e-6 used elsewhere
        assert (got["topk_w"] - ref["topk_w"]).abs().max().item() <= 1e-6
    assert err.item() == 0


@pytest.mark.skipif(not torch.cuda.is_available(), reason="no CUDA device")
def test_noalloc_route_reports_flags_and_limits():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    z = workloads.make_logits(300, 8, device="cuda", seed=7)
    z[3, :] = float("nan")
    rc, got = _noalloc(z, 2, 1, err)
    assert rc == N.MOE_OK
    torch.cuda.synchronize()
    assert err.item() & N.MOE_DEVERR_NONFINITE_LOGIT
    assert np.allclose(got["topk_w"][3].cpu().numpy(), 0.5)
    # beyond the fixed array: rejected before any work, with a message
    big = torch.empty((256 * 300, 1024), dtype=torch.float32, device="cuda")
    rc, _ = _noalloc(big, 2, 1, None)
    assert rc == N.MOE_ERR_UNSUPPORTED
    assert b"MOE_ROUTE_NOALLOC_MAX_SLOTS" in N.lib().moe_last_error()


@pytest.mark.skipif(not torch.cuda.is_available(), reason="no CUDA device")
def test_noalloc_route_in_a_fresh_process():
    here = os.path.dirname(os.path.abspath(__file__))
    code = ("import sys; sys.path[:0] = [%r, %r]; "
            "import test_zz_no_alloc as t; t.test_noalloc_route_equals_moe_route_on_two_calls(); "
            "print('fresh process ok')" % (here, os.path.dirname(here)))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "fresh process ok" in r.stdout
