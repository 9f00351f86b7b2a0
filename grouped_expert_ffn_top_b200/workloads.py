"""Seeded synthetic inputs for the MoE layer hot path.

This module only draws random numbers and lays them out. It holds none of the
layer's arithmetic (no routing, no softmax, no expert FFN), so both the CUDA
path and the CPU oracle can take their inputs from it without sharing any of
the method.

The workloads stand in for the data the pages train on: "packed 32k
sequences" with expert-parallel dispatch (leap-finetune PR #26 "Add MoE expert
parallel training runtime", the comment on DP4/EP2 and DP4/EP4 runs), with
uneven and empty work per microbatch and per expert (ART issue #917 "Support
combined expert and data parallelism in TrainerRank", Desired behavior and
Acceptance). No dataset or checkpoint is used; every tensor is drawn here.

Recipe per tensor (all N(mean, std) draws are Gaussian):
  x  ~ N(0, 1)                    activations [T, d]
  Wr ~ N(0, 0.02)                 router weight [E, d]
  b                               router bias [E], fp32, per workload (below)
  Wg, Wu ~ N(0, 0.02)             gate / up projections [E, f, d]
  Wd ~ N(0, 0.02)                 down projection [E, d, f]
  dY ~ N(0, 1)                    upstream gradient [T, d]
Router bias kinds:
  "expert3_off"  (0, ..., 0, -1e4) on the last expert, so it receives no token
  ("normal", s)  N(0, s) per expert: uneven load
  "zipf"         -1.2 * ln(rank_e), rank a seeded permutation of 1..E, with the
                 four worst ranks pushed to -1e4 so that exactly four experts
                 receive no token (k < E - 4 keeps them out of every top-k)
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch

BF16 = "bf16"
F32 = "f32"


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: List[int]          # tokens per microbatch (one entry = one microbatch)
    d: int                # d_model
    E: int                # experts
    k: int                # top-k
    f: int                # SwiGLU ffn width
    dtype: str            # "bf16" or "f32"
    bias: object          # see module docstring
    backward: bool        # forward only, or forward + backward
    ep_groups: int        # destination groups of the send layout
    description: str = ""

    @property
    def total_tokens(self) -> int:
        return sum(self.T)

    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == BF16 else torch.float32


WORKLOADS: Dict[str, Workload] = {
    "tiny_fp32": Workload(
        "tiny_fp32", [256], d=64, E=4, k=2, f=128, dtype=F32, bias="expert3_off",
        backward=True, ep_groups=2,
        description="tiny fp32 MoE layer, expert 3 starved, fwd+bwd"),
    "dense_fwd": Workload(
        "dense_fwd", [4096], d=1024, E=8, k=2, f=2816, dtype=BF16, bias=("normal", 0.5),
        backward=False, ep_groups=1,
        description="dense-ish bf16 forward, uneven load"),
    "fine_fwd_32k": Workload(
        "fine_fwd_32k", [32768], d=2048, E=64, k=8, f=1408, dtype=BF16, bias="zipf",
        backward=False, ep_groups=4,
        description="fine-grained bf16 forward on one packed 32k sequence, Zipf-skewed, EP=4 layout"),
    "fine_fwdbwd_32k": Workload(
        "fine_fwdbwd_32k", [32768], d=2048, E=64, k=8, f=1408, dtype=BF16, bias="zipf",
        backward=True, ep_groups=4,
        description="fine-grained bf16 forward+backward on one packed 32k sequence, Zipf-skewed"),
    "fine_fwdbwd_8k": Workload(
        "fine_fwdbwd_8k", [8192], d=2048, E=64, k=8, f=1408, dtype=BF16, bias="zipf",
        backward=True, ep_groups=4,
        description="the 32k workload's layer on 8192 tokens (kernel profiling: a few GB on the device)"),
    "sweep_profile": Workload(
        "sweep_profile", [4096], d=4096, E=2, k=2, f=14336, dtype=BF16,
        bias=("normal", 1.0), backward=True, ep_groups=1,
        description="the sweep's layer shapes with 2 experts and 4096 tokens at top-2: every "
                    "expert gets 4096 rows, the average of the sweep's 32768-token microbatch, "
                    "an eighth of its work (kernel counter captures: about 3.5 GB on the device)"),
    "uneven_sweep": Workload(
        "uneven_sweep", [32768, 9000, 1, 0], d=4096, E=16, k=2, f=14336, dtype=BF16,
        bias=("normal", 1.0), backward=True, ep_groups=1,
        description="uneven microbatch sweep T=32768,9000,1,0 with fp32 gradient accumulation"),
}


def custom(name: str, T, d: int, E: int, k: int, f: int, dtype: str = BF16,
           bias=("normal", 0.5), backward: bool = True, ep_groups: int = 1) -> Workload:
    """A workload with arbitrary sizes (parity tests use several)."""
    if isinstance(T, int):
        T = [T]
    return Workload(name, list(T), d, E, k, f, dtype, bias, backward, ep_groups)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, std, gen, device, dtype):
    # Draw in fp32 on the generator's device, then round once to the storage type.
    out = torch.empty(shape, dtype=torch.float32, device=device)
    out.normal_(0.0, std, generator=gen)
    return out.to(dtype)


def router_bias(w: Workload, device="cpu", seed: int = 0) -> torch.Tensor:
    """The fp32 router bias of a workload (see the module docstring)."""
    E = w.E
    if w.bias == "expert3_off":
        b = torch.zeros(E, dtype=torch.float32)
        b[E - 1] = -1.0e4
        return b.to(device)
    if w.bias == "zipf":
        g = _gen("cpu", seed + 7001)
        rank = torch.randperm(E, generator=g).to(torch.float64) + 1.0
        b = (-1.2 * torch.log(rank)).to(torch.float32)
        b[rank > E - 4] = -1.0e4
        return b.to(device)
    if isinstance(w.bias, tuple) and w.bias[0] == "normal":
        g = _gen("cpu", seed + 7002)
        b = torch.empty(E, dtype=torch.float32).normal_(0.0, float(w.bias[1]), generator=g)
        return b.to(device)
    if w.bias is None or w.bias == "zero":
        return torch.zeros(E, dtype=torch.float32, device=device)
    raise ValueError(f"unknown bias kind {w.bias!r}")


def make_params(w: Workload, device="cpu", seed: int = 0, std: float = 0.02) -> Dict[str, torch.Tensor]:
    """Router and expert parameters: Wr [E,d], b [E] fp32, Wg/Wu [E,f,d], Wd [E,d,f]."""
    dt = w.torch_dtype()
    g = _gen(device, seed + 1)
    p = {
        "Wr": _normal((w.E, w.d), std, g, device, dt),
        "Wg": _normal((w.E, w.f, w.d), std, g, device, dt),
        "Wu": _normal((w.E, w.f, w.d), std, g, device, dt),
        "Wd": _normal((w.E, w.d, w.f), std, g, device, dt),
    }
    p["b"] = router_bias(w, device, seed)
    return p


def make_batch(w: Workload, mb: int = 0, device="cpu", seed: int = 0) -> Dict[str, torch.Tensor]:
    """Activations x [T,d] and upstream gradient dY [T,d] of microbatch `mb`."""
    dt = w.torch_dtype()
    T = w.T[mb]
    g = _gen(device, seed + 101 + 17 * mb)
    return {
        "x": _normal((T, w.d), 1.0, g, device, dt),
        "dY": _normal((T, w.d), 1.0, g, device, dt),
    }


def make_logits(T: int, E: int, device="cpu", seed: int = 0, tie_fraction: float = 0.5,
                specials: bool = False) -> torch.Tensor:
    """Router logits [T,E] fp32 with many exact ties (values on a coarse grid).

    Routing parity runs on these directly: a coarse grid makes equal logits
    common, so the lower-index tie-break is exercised on every token.
    With `specials`, some entries are +inf / -inf (non-finite inputs)."""
    g = _gen("cpu", seed + 303)
    z = torch.randn((T, E), generator=g, dtype=torch.float32)
    grid = torch.round(z * 4.0) / 4.0
    pick = torch.rand((T, E), generator=g) < tie_fraction
    z = torch.where(pick, grid, z)
    if specials and T > 0:
        rows = torch.randint(0, T, (max(1, T // 16),), generator=g)
        cols = torch.randint(0, E, (rows.numel(),), generator=g)
        z[rows, cols] = -math.inf
    return z.to(device)


def sample_tokens(T: int, n: int, seed: int = 0, must_include: Optional[torch.Tensor] = None) -> torch.Tensor:
    """A deterministic sorted sample of token indices (plus any required ones)."""
    g = _gen("cpu", seed + 505)
    n = min(n, T)
    idx = torch.randperm(T, generator=g)[:n]
    if must_include is not None and must_include.numel():
        idx = torch.cat([idx, must_include.to(torch.int64).cpu()])
    return torch.unique(idx).sort().values
