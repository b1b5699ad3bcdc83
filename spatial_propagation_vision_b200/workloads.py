"""Seeded synthetic Prop2D workloads.

This module only draws random tensors of the right shapes; it holds none of
the method's arithmetic.  It is the one module that both the CUDA path's
tests/benchmark and the CPU oracle's tests use.

The shapes follow the workloads of "Scaling Parallel Sequence Models to
Foundation-Scale Vision Encoders": ViT patch grids (patch 14) at 518, 1036
and 2072 px, latent width Cc = C / s with C = 1152 and s = 18 (Sec. 5.1,
Sec. 6.3 "C-GSPN System Efficiency", batch 32), and the 256 x 256 x 1024
input of the original GSPN kernel (Sec. 1).  No real activations are
available, so seeded draws stand in for them.

Draw order (fixed): x ~ N(0, 1); lambda ~ U(0, 1); wlogit ~ N(0, sigma_w);
u ~ U(0, 1), all drawn in fp32 from ``torch.Generator('cpu')`` seeded with
``seed``, then cast to the workload dtype.
"""
from __future__ import annotations

from dataclasses import dataclass, asdict

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Cc: int
    H: int
    W: int
    dtype: str          # "f32" or "bf16": input and output dtype (state is fp32)
    share_w: int        # 1: one logit field per (batch, direction), shared by all Cc channels
    sigma_w: float      # standard deviation of the logits
    dirs: int = 15

    @property
    def elems(self) -> int:
        return self.B * self.Cc * self.H * self.W

    @property
    def planes(self) -> int:
        return self.B * self.Cc

    @property
    def in_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def algorithmic_bytes(self) -> int:
        """Bytes that must cross HBM once: x once; lambda, u, logits once per
        direction; y written once."""
        s = self.in_bytes
        nd = bin(self.dirs).count("1")
        E = self.elems
        if self.share_w:
            return E * (s + 2 * nd * s + s) + 3 * nd * self.B * self.H * self.W * s
        return E * (s + 5 * nd * s + s)

    def asdict(self) -> dict:
        return asdict(self)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 4, 16, 16, "f32", 0, 1.0),
    "mid": Workload("mid", 8, 64, 37, 37, "f32", 0, 2.0),
    "1k": Workload("1k", 32, 64, 74, 74, "bf16", 0, 2.0),
    "orig": Workload("orig", 1, 1024, 256, 256, "f32", 0, 1.0),
    "2k": Workload("2k", 8, 64, 148, 148, "bf16", 1, 1.0),
}

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def make_inputs(B: int, Cc: int, H: int, W: int, *, share_w: int = 0,
                sigma_w: float = 1.0, dtype: str = "f32", seed: int = 0,
                device: str | torch.device = "cpu") -> dict:
    """Seeded inputs in the C-ABI layouts.

    Returns a dict with x [B,Cc,H,W], lam [B,4,Cc,H,W], wlogit [B,4,Cw,3,H,W]
    (Cw = 1 if share_w else Cc) and u [B,4,Cc,H,W], in ``dtype``.  Drawing
    always happens on the CPU so that every device sees identical values.
    """
    g = torch.Generator("cpu").manual_seed(seed)
    Cw = 1 if share_w else Cc
    x = torch.randn((B, Cc, H, W), generator=g, dtype=torch.float32)
    lam = torch.rand((B, 4, Cc, H, W), generator=g, dtype=torch.float32)
    wl = torch.randn((B, 4, Cw, 3, H, W), generator=g, dtype=torch.float32) * float(sigma_w)
    u = torch.rand((B, 4, Cc, H, W), generator=g, dtype=torch.float32)
    td = TORCH_DTYPE[dtype]
    out = {"x": x, "lam": lam, "wlogit": wl, "u": u}
    return {k: v.to(td).to(device) for k, v in out.items()}


def workload_inputs(w: Workload, seed: int = 0, device="cpu") -> dict:
    return make_inputs(w.B, w.Cc, w.H, w.W, share_w=w.share_w, sigma_w=w.sigma_w,
                       dtype=w.dtype, seed=seed, device=device)
