"""Seeded synthetic workloads shared by the tests, the smoke entry and the benchmark.

This module only draws inputs.  It holds none of the method's arithmetic, so the CUDA
path and the CPU oracle can both use it without sharing any computation.

Each workload mirrors a shape the pages measure on: sequence lengths from the 2K-131K
range the scan page asks to test ("Log-Depth Chunked Linear-Attention Scan",
"Implementation notes"), chunk sizes 32 or 64 (same passage), the ELU+1 feature map
("Linear Attention and Retentive Networks ...", "The Associative Property and Linear
Kernel Formulation") and a retention-style per-head decay of the form 1 - 2^(-5 - x)
(same page, "1. Multi-Scale Decay Formulation").  No dataset is involved; every tensor
is Gaussian noise from a fixed seed.

Recipe: q, then k, then v, each ``randn([B, H, T, d])`` in float32 from one generator
seeded with ``seed``, multiplied by the workload's scale in float32, then rounded to the
workload dtype (round-to-nearest-even for bf16).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    C: int
    dtype: str            # "f32" or "bf16"
    scale: float          # multiplies the N(0, 1) draws
    feature_map: str      # "elu1" or "identity"
    decay: bool           # per-head gamma_h = 1 - 2^(-5 - 3h/31)
    normalize: bool
    description: str = field(default="", compare=False)

    @property
    def tokens_heads(self) -> int:
        return self.B * self.H * self.T

    @property
    def n_chunks(self) -> int:
        return -(-self.T // self.C)

    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def gammas(self) -> list[float] | None:
        """Per-head decays as float32 values (None when the workload has no decay)."""
        if not self.decay:
            return None
        return [float(torch.tensor(1.0 - 2.0 ** (-5.0 - 3.0 * h / 31.0), dtype=torch.float32))
                for h in range(self.H)]

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS: dict[str, Workload] = {
    "pr1_ref": Workload(
        "pr1_ref", B=1, H=2, T=256, dk=32, dv=32, C=32, dtype="f32", scale=1.0,
        feature_map="elu1", decay=False, normalize=True,
        description="normalised, B1 H2 T256 d32 C32, fp32 N(0,1) seed 0, elu+1"),
    "norm_b4h16": Workload(
        "norm_b4h16", B=4, H=16, T=4096, dk=64, dv=64, C=64, dtype="bf16", scale=0.5,
        feature_map="elu1", decay=False, normalize=True,
        description="normalised, B4 H16 T4096 d64 C64, bf16 N(0,1)*0.5, elu+1"),
    "ragged_b2h32": Workload(
        "ragged_b2h32", B=2, H=32, T=16000, dk=128, dv=128, C=64, dtype="bf16", scale=0.5,
        feature_map="elu1", decay=False, normalize=True,
        description="normalised, B2 H32 T16000 d128 C64, bf16 N(0,1)*0.5, elu+1"),
    "ragged_b2h32_t15990": Workload(
        "ragged_b2h32_t15990", B=2, H=32, T=15990, dk=128, dv=128, C=64, dtype="bf16",
        scale=0.5, feature_map="elu1", decay=False, normalize=True,
        description="ragged companion: T15990 (last chunk 54 of 64 tokens)"),
    "retention_128k": Workload(
        "retention_128k", B=1, H=32, T=131072, dk=128, dv=128, C=64, dtype="bf16",
        scale=1.0 / math.sqrt(128.0), feature_map="identity", decay=True, normalize=False,
        description="retention-style decayed, unnormalised, B1 H32 T131072 d128 C64, "
                    "bf16 N(0,1)/sqrt(128), identity, gamma_h = 1 - 2^(-5-3h/31)"),
    "scan_depth_1m": Workload(
        "scan_depth_1m", B=1, H=8, T=1048576, dk=64, dv=64, C=64, dtype="bf16", scale=0.5,
        feature_map="elu1", decay=False, normalize=True,
        description="scan-depth stress, B1 H8 T1048576 d64 C64 (16384 chunks), bf16, elu+1"),
}


# Gated linear attention (data-dependent decay, "Linear Attention and Retentive Networks ...",
# Gated Linear Attention (GLA) and Hardware-Software Co-Design) on the retention workload's
# shape: gates alpha = sigmoid(x) per token and key feature, the page's parameterisation,
# with x ~ N(4, 1) (gates mostly 0.95-0.99, some near 0.8).
GLA_WORKLOADS: dict[str, Workload] = {
    "gla_128k": Workload(
        "gla_128k", B=1, H=32, T=131072, dk=128, dv=128, C=64, dtype="bf16",
        scale=1.0 / math.sqrt(128.0), feature_map="identity", decay=False, normalize=False,
        description="gated linear attention, B1 H32 T131072 d128 C64, bf16 N(0,1)/sqrt(128), "
                    "gates sigmoid(N(4, 1)) in float32"),
}


def make_gates(w: Workload, seed: int = 0, device: str | torch.device = "cpu",
               gen_device: str | torch.device | None = None, mean: float = 4.0,
               std: float = 1.0) -> torch.Tensor:
    """Draw the gates [B, H, T, dk] (float32) of a gated workload: sigmoid of N(mean, std)
    from a generator seeded with ``seed`` + 1000003 (independent of q, k, v)."""
    gen_device = torch.device(gen_device if gen_device is not None else device)
    g = torch.Generator(device=gen_device)
    g.manual_seed(int(seed) + 1000003)
    x = torch.randn((w.B, w.H, w.T, w.dk), generator=g, device=gen_device, dtype=torch.float32)
    return torch.sigmoid(x * std + mean).to(device)


def make_inputs(w: Workload, seed: int = 0, device: str | torch.device = "cpu",
                gen_device: str | torch.device | None = None):
    """Draw (q, k, v) for workload ``w`` on ``device``.

    The draws happen on ``gen_device`` (default: ``device``) so that CPU-drawn inputs are
    portable across machines; they are then moved to ``device``.
    """
    gen_device = torch.device(gen_device if gen_device is not None else device)
    g = torch.Generator(device=gen_device)
    g.manual_seed(int(seed))
    out = []
    for d in (w.dk, w.dk, w.dv):
        x = torch.randn((w.B, w.H, w.T, d), generator=g, device=gen_device, dtype=torch.float32)
        if w.scale != 1.0:
            x.mul_(torch.tensor(w.scale, dtype=torch.float32, device=gen_device))
        x = x.to(w.torch_dtype())
        out.append(x.to(device))
    return tuple(out)
