"""Seeded synthetic inputs for the Gecko SCA + AWM forward.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests. It holds none of the method's arithmetic: it only draws the five
per-head input tensors (Q, K, V, Q_m, K_m) with the shapes and value
distributions of the projections that feed the layer ("Gecko: An Efficient
Neural Architecture ...", method step details, steps 2 and 4): a shared
representation Z' normalised to unit L2 norm per token, per-(head, dim)
affine maps for the queries and keys, and SiLU values.

Recipe, per tensor and per (b, h, t):
  g ~ N(0, 1)^d,  Z' = g / ||g||_2
  Q   = kappa_q * Z' + nu_q      K   = kappa_k * Z' + nu_k
  Q_m = eta_q   * Z' + rho_q     K_m = eta_k   * Z' + rho_k
  scales ~ N(1, 0.1^2), offsets ~ N(0, 0.1^2) (per head and dim)
  V = SiLU(N(0, 1)) elementwise
Everything is drawn in fp32 and then cast (round-to-nearest-even) to the
workload's dtype.  The small fp32 workload shares one Z' across Q, K, Q_m,
K_m (seed 0); the others draw each tensor from its own seed
100 * workload_id + {Q: 0, K: 1, V: 2, Q_m: 3, K_m: 4}.
"""
from __future__ import annotations

import dataclasses
import torch

TENSORS = ("q", "k", "v", "qm", "km")


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shape, dtype and generator options."""
    name: str
    wid: int                 # workload id used in the seed formula
    dtype: str               # "f32" or "bf16"
    B: int
    H: int
    T: int
    d: int
    c: int
    shared_z: bool = False   # one Z' for Q, K, Q_m, K_m (small fp32 case)
    key_offset_std: float = 0.1  # std of nu_k and rho_k

    @property
    def S(self) -> int:
        return self.T // self.c

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The workloads: a small fp32 case, a many-chunk bf16 case, the 7B-layer-shaped
# headline case (H=32, d=128, c=4096), the chunk-size sweep with wide key
# offsets, and the 4M-token case.
WORKLOADS = {
    "fp32_small": Workload("fp32_small", 1, "f32", 1, 1, 512, 64, 64, shared_z=True),
    "bf16_many_chunks": Workload("bf16_many_chunks", 2, "bf16", 2, 8, 4096, 64, 256),
    "bf16_h32_c4096": Workload("bf16_h32_c4096", 3, "bf16", 1, 32, 32768, 128, 4096),
    "bf16_sweep_c512": Workload("bf16_sweep_c512", 4, "bf16", 1, 32, 65536, 128, 512, key_offset_std=1.0),
    "bf16_sweep_c1024": Workload("bf16_sweep_c1024", 4, "bf16", 1, 32, 65536, 128, 1024, key_offset_std=1.0),
    "bf16_sweep_c2048": Workload("bf16_sweep_c2048", 4, "bf16", 1, 32, 65536, 128, 2048, key_offset_std=1.0),
    "bf16_sweep_c4096": Workload("bf16_sweep_c4096", 4, "bf16", 1, 32, 65536, 128, 4096, key_offset_std=1.0),
    "bf16_4m_tokens": Workload("bf16_4m_tokens", 5, "bf16", 1, 8, 4194304, 128, 4096),
    # the headline shape with 4 heads: small enough for profiler captures,
    # inputs (168 MB) still larger than L2
    "bf16_h4_c4096": Workload("bf16_h4_c4096", 6, "bf16", 1, 4, 32768, 128, 4096),
}


def _unit_rows(gen: torch.Generator, n: int, d: int, device) -> torch.Tensor:
    g = torch.randn(n, d, generator=gen, device=device, dtype=torch.float32)
    return g / g.norm(dim=1, keepdim=True)


def _affine(gen: torch.Generator, H: int, d: int, off_std: float, device):
    scale = 1.0 + 0.1 * torch.randn(H, d, generator=gen, device=device, dtype=torch.float32)
    off = off_std * torch.randn(H, d, generator=gen, device=device, dtype=torch.float32)
    return scale, off


def _silu(x: torch.Tensor) -> torch.Tensor:
    return x * torch.sigmoid(x)


def make_inputs(w: Workload, device="cpu", seed_offset: int = 0) -> dict:
    """Draw q, k, v, qm, km as [B, H, T, d] tensors of the workload's dtype.

    Large workloads are drawn one (b, h) slab at a time so the fp32
    temporaries stay small; each slab has its own generator seeded from the
    tensor seed and the slab index, so results do not depend on slab order.
    """
    B, H, T, d = w.B, w.H, w.T, w.d
    dt = w.torch_dtype
    out = {n: torch.empty(B, H, T, d, dtype=dt, device=device) for n in TENSORS}
    if w.shared_z:
        gen = torch.Generator(device=device).manual_seed(0 + seed_offset)
        z = _unit_rows(gen, B * H * T, d, device).view(B, H, T, d)
        for name in ("q", "k", "qm", "km"):
            std = w.key_offset_std if name in ("k", "km") else 0.1
            sc, off = _affine(gen, H, d, std, device)
            out[name].copy_((sc[None, :, None, :] * z + off[None, :, None, :]).to(dt))
        out["v"].copy_(_silu(torch.randn(B, H, T, d, generator=gen, device=device)).to(dt))
        return out
    for idx, name in enumerate(TENSORS):
        seed = 100 * w.wid + idx + seed_offset
        gen = torch.Generator(device=device).manual_seed(seed)
        if name != "v":
            std = w.key_offset_std if name in ("k", "km") else 0.1
            sc, off = _affine(gen, H, d, std, device)
        for b in range(B):
            for h in range(H):
                sg = torch.Generator(device=device).manual_seed(seed * 1000003 + b * H + h)
                if name == "v":
                    slab = _silu(torch.randn(T, d, generator=sg, device=device, dtype=torch.float32))
                else:
                    slab = sc[h] * _unit_rows(sg, T, d, device) + off[h]
                out[name][b, h].copy_(slab.to(dt))
    return out


# --------------------------------------------------------------------------
# CEMA (the complex damped EMA that produces the layer input): seeded
# synthetic inputs.  x is the layer input (standard normal); the per-(d, j)
# parameters are drawn as a trained layer would hold them after its sigmoids
# (alpha, delta in (0, 1)); document starts, where the recurrence restarts,
# are Bernoulli with mean document length `mean_doc` (0: one document).
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class CemaWorkload:
    """One synthetic CEMA workload: x [B, L, D], h hidden dimensions per feature."""
    name: str
    wid: int
    dtype: str               # "f32" or "bf16"
    B: int
    L: int
    D: int
    h: int = 16
    mean_doc: int = 0        # mean document length for resets (0 = no resets)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# small parity cases (ragged D, resets) and the 7B-width case (D = 4096, h = 16)
# over the same 32K tokens as the attention workload
CEMA_WORKLOADS = {
    "cema_f32_small": CemaWorkload("cema_f32_small", 21, "f32", 2, 1000, 96, 16, mean_doc=300),
    "cema_bf16_small": CemaWorkload("cema_bf16_small", 22, "bf16", 2, 2304, 160, 16, mean_doc=700),
    "cema_bf16_7b_32k": CemaWorkload("cema_bf16_7b_32k", 23, "bf16", 1, 32768, 4096, 16),
}


def make_cema_inputs(w: CemaWorkload, device="cpu", seed_offset: int = 0) -> dict:
    """x [B, L, D] (workload dtype); alpha, delta, theta, beta [D, h] fp32;
    eta [D, h, 2] fp32 (real, imaginary); reset [B, L] uint8 (1 = a document
    starts at this token)."""
    gen = torch.Generator(device=device).manual_seed(100 * w.wid + seed_offset)
    f32 = dict(generator=gen, device=device, dtype=torch.float32)
    out = {
        "x": torch.randn(w.B, w.L, w.D, **f32).to(w.torch_dtype),
        "alpha": torch.sigmoid(torch.randn(w.D, w.h, **f32) - 2.0),
        "delta": torch.sigmoid(torch.randn(w.D, w.h, **f32)),
        "theta": torch.rand(w.D, w.h, **f32) * 3.141592653589793,
        "beta": torch.randn(w.D, w.h, **f32),
        "eta": torch.randn(w.D, w.h, 2, **f32) / w.h ** 0.5,
    }
    if w.mean_doc > 0:
        out["reset"] = (torch.rand(w.B, w.L, **f32) < 1.0 / w.mean_doc).to(torch.uint8)
    else:
        out["reset"] = None
    return out


# --------------------------------------------------------------------------
# Timestep decay normalisation: x is the layer input (standard normal with a
# slowly drifting per-group offset and scale, so the decayed statistics have
# something to track); gamma, bias per feature; G groups of D / G features.
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class NormWorkload:
    """One synthetic timestep-decay-normalisation workload."""
    name: str
    wid: int
    dtype: str
    B: int
    L: int
    D: int
    G: int
    beta1: float = 0.99
    beta2: float = 0.999
    eps: float = 1e-5

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


NORM_WORKLOADS = {
    "tdnorm_f32_small": NormWorkload("tdnorm_f32_small", 51, "f32", 2, 700, 96, 4),
    "tdnorm_bf16_small": NormWorkload("tdnorm_bf16_small", 52, "bf16", 2, 1500, 256, 8, beta1=0.9, beta2=0.99),
    "tdnorm_bf16_7b_32k": NormWorkload("tdnorm_bf16_7b_32k", 53, "bf16", 1, 32768, 4096, 32),
}


def make_norm_inputs(w: NormWorkload, device="cpu", seed_offset: int = 0) -> dict:
    """x [B, L, D] (workload dtype); gamma, bias [D] fp32."""
    gen = torch.Generator(device=device).manual_seed(100 * w.wid + seed_offset)
    f32 = dict(generator=gen, device=device, dtype=torch.float32)
    t = torch.arange(w.L, device=device, dtype=torch.float32)[None, :, None]
    drift_off = 0.5 * torch.sin(t / 997.0 + torch.rand(w.B, 1, w.G, **f32) * 6.283)
    drift_scl = 1.0 + 0.3 * torch.cos(t / 1777.0 + torch.rand(w.B, 1, w.G, **f32) * 6.283)
    x = torch.randn(w.B, w.L, w.G, w.D // w.G, **f32) * drift_scl[..., None] + drift_off[..., None]
    return {
        "x": x.reshape(w.B, w.L, w.D).to(w.torch_dtype),
        "gamma": 1.0 + 0.1 * torch.randn(w.D, **f32),
        "bias": 0.1 * torch.randn(w.D, **f32),
    }
