"""Seeded synthetic inputs for the masked HLA forward workloads.

This module is the only code shared by the fp64 oracle side (``oracle/``, the
tests, the CPU baseline) and the CUDA side (the package, ``bench.py``).  It
holds no arithmetic of the method itself: it draws random numbers, applies the
per-workload input transform (scale, softplus) and rounds bf16 workloads once.

Recipe (one torch CPU generator per workload, so inputs are identical on every
machine and device):

* ``torch.Generator('cpu').manual_seed(seed)``;
* draw ``z_q, z_k, z_v`` in that order, each ``randn([B,H,T,d])`` in fp32;
* then, only for the decayed workload, ``u = rand([H])`` and
  ``gamma = lo + (hi - lo) * u``;
* transform: ``q = f(z_q)``, ``k = f(z_k)``, ``v = g(z_v)`` as the workload
  table below says;
* bf16 workloads are rounded once, round-to-nearest-even (``.to(bfloat16)``),
  after the transform; the oracle consumes exactly those rounded values,
  widened to fp64, so a parity error measures the GPU arithmetic and not the
  input quantisation.

The five workloads are the masked second-order HLA (plain, ratio-normalised,
per-head decay), the asymmetric AHLA and the third-order HLA forward of the
"Higher-order Linear Attention" summary (page 2510.27258, sections
Metodología 1-3).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "workload"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    op: str            # "hla2", "hla2n" (ratio-normalised), "hla2d" (decay), "ahla", "hla3"
    dtype: str         # "f32" or "bf16": the element type handed to the kernels
    B: int
    H: int
    T: int
    d: int
    dv: int
    qk_transform: str  # "scaled" = z/sqrt(d); "softplus" = softplus(z)/sqrt(d)
    v_transform: str   # "scaled" = z/sqrt(d); "unit" = z
    eps: float = 1e-6
    gamma_range: Optional[tuple] = None
    seed: int = 0

    @property
    def tokens(self) -> int:
        return self.B * self.H * self.T

    def scaled(self, **kw) -> "Workload":
        """Same recipe with other sizes (small parity cases)."""
        return dataclasses.replace(self, **kw)


# The five workloads of the problem list (sizes, distributions, dtypes), plus three for the
# widened operators; the names say what each one is.
WORKLOADS = {
    "hla2_f32_1x2x256x32": Workload(
        "hla2_f32_1x2x256x32", "hla2", "f32", 1, 2, 256, 32, 32, "scaled", "scaled"),
    "hla2n_bf16_4x16x4096x64": Workload(
        "hla2n_bf16_4x16x4096x64", "hla2n", "bf16", 4, 16, 4096, 64, 64, "softplus", "unit",
        eps=1e-6),
    "hla2d_bf16_2x16x16384x64": Workload(
        "hla2d_bf16_2x16x16384x64", "hla2d", "bf16", 2, 16, 16384, 64, 64, "scaled", "scaled",
        gamma_range=(0.95, 0.999)),
    "ahla_bf16_4x16x8192x64": Workload(
        "ahla_bf16_4x16x8192x64", "ahla", "bf16", 4, 16, 8192, 64, 64, "scaled", "scaled"),
    "hla3_f32_2x8x4096x32": Workload(
        "hla3_f32_2x8x4096x32", "hla3", "f32", 2, 8, 4096, 32, 32, "scaled", "scaled"),
    # not among the five: the unmasked second order at the headline's shape, and the
    # ratio-normalised AHLA / third order at the shapes of their plain workloads
    "hla2u_bf16_4x16x4096x64": Workload(
        "hla2u_bf16_4x16x4096x64", "hla2u", "bf16", 4, 16, 4096, 64, 64, "scaled", "scaled"),
    "ahlan_bf16_4x16x8192x64": Workload(
        "ahlan_bf16_4x16x8192x64", "ahlan", "bf16", 4, 16, 8192, 64, 64, "softplus", "unit"),
    "hla3n_f32_2x8x4096x32": Workload(
        "hla3n_f32_2x8x4096x32", "hla3n", "f32", 2, 8, 4096, 32, 32, "softplus", "unit"),
    # the decayed AHLA and third order at the shapes of their plain workloads, gamma as for the
    # decayed second order
    "ahlad_bf16_4x16x8192x64": Workload(
        "ahlad_bf16_4x16x8192x64", "ahlad", "bf16", 4, 16, 8192, 64, 64, "scaled", "scaled",
        gamma_range=(0.95, 0.999)),
    "hla3d_f32_2x8x4096x32": Workload(
        "hla3d_f32_2x8x4096x32", "hla3d", "f32", 2, 8, 4096, 32, 32, "scaled", "scaled",
        gamma_range=(0.95, 0.999)),
    # the ratio-normalised AHLA with decay (op "ahlan" with a gamma per head)
    "ahlan_decayed_bf16_4x16x8192x64": Workload(
        "ahlan_decayed_bf16_4x16x8192x64", "ahlan", "bf16", 4, 16, 8192, 64, 64, "softplus", "unit",
        gamma_range=(0.95, 0.999)),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def _qk(z: torch.Tensor, how: str, d: int) -> torch.Tensor:
    if how == "scaled":
        return z / math.sqrt(d)
    if how == "softplus":
        return torch.nn.functional.softplus(z) / math.sqrt(d)
    raise ValueError(how)


def _v(z: torch.Tensor, how: str, d: int) -> torch.Tensor:
    if how == "scaled":
        return z / math.sqrt(d)
    if how == "unit":
        return z
    raise ValueError(how)


def make_inputs(w: Workload):
    """Return ``(q, k, v, gamma)`` as CPU tensors in the workload's dtype.

    ``q, k``: [B,H,T,d]; ``v``: [B,H,T,dv]; ``gamma``: fp32 [H] or None.
    """
    g = torch.Generator("cpu").manual_seed(w.seed)
    zq = torch.randn([w.B, w.H, w.T, w.d], generator=g, dtype=torch.float32)
    zk = torch.randn([w.B, w.H, w.T, w.d], generator=g, dtype=torch.float32)
    zv = torch.randn([w.B, w.H, w.T, w.dv], generator=g, dtype=torch.float32)
    gamma = None
    if w.gamma_range is not None:
        lo, hi = w.gamma_range
        u = torch.rand([w.H], generator=g, dtype=torch.float32)
        gamma = (lo + (hi - lo) * u).to(torch.float32)
    q = _qk(zq, w.qk_transform, w.d)
    k = _qk(zk, w.qk_transform, w.d)
    v = _v(zv, w.v_transform, w.d)
    if w.dtype == "bf16":
        q, k, v = (x.to(torch.bfloat16) for x in (q, k, v))
    elif w.dtype != "f32":
        raise ValueError(w.dtype)
    return q.contiguous(), k.contiguous(), v.contiguous(), gamma
